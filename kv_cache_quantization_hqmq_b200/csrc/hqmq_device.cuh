// hqmq_device.cuh -- device helpers shared by the libhqmq kernels (sm_100a).
//
// Every fp32 step that decides a stored bit pattern (chunk norm, radius,
// codeword, decoded value) is written with explicit IEEE round-to-nearest
// intrinsics so that no FMA contraction or reassociation can change it.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/hqmq.h"

namespace hqmq {

constexpr unsigned FULL = 0xFFFFFFFFu;

struct DevStatus {  // same layout as hqmq_status
    unsigned int flags;
    unsigned int reserved;
    unsigned long long n_outliers;
    unsigned long long n_saturated;
    unsigned long long n_nonfinite;
};
static_assert(sizeof(DevStatus) == sizeof(hqmq_status), "status layout");

// Norm of a chunk (w, i, j, k): r2 = fma(x3,x3, fma(x2,x2, fma(x1,x1, x0*x0))),
// r = sqrt(r2), every step IEEE round-to-nearest.
__device__ __forceinline__ float chunk_norm(float x0, float x1, float x2, float x3) {
    float r2 = __fmul_rn(x0, x0);
    r2 = __fmaf_rn(x1, x1, r2);
    r2 = __fmaf_rn(x2, x2, r2);
    r2 = __fmaf_rn(x3, x3, r2);
    return __fsqrt_rn(r2);
}

// Order key of a non-negative magnitude: its bits; every NaN -> 0x7FFFFFFF.
__device__ __forceinline__ uint32_t mag_key(float v) {
    return (v != v) ? 0x7FFFFFFFu : __float_as_uint(v);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h16) {
    return __uint_as_float(h16 << 16);
}

// fp32 -> fp16 bits, round-to-nearest-even; finite values that would round to
// inf saturate to +-65504 (*sat = 1); NaN -> sign | 0x7E00.
__device__ __forceinline__ uint16_t f32_to_f16_sat(float v, int &sat) {
    uint16_t sign = (uint16_t)((__float_as_uint(v) >> 16) & 0x8000u);
    if (v != v) return (uint16_t)(sign | 0x7E00u);
    uint16_t h = __half_as_ushort(__float2half_rn(v));
    if ((h & 0x7FFFu) == 0x7C00u && fabsf(v) != __int_as_float(0x7F800000)) {
        sat = 1;
        return (uint16_t)(sign | 0x7BFFu);
    }
    return h;
}

// Two values to packed fp16 bits (a in the low half), same rules as
// f32_to_f16_sat; the common in-range case is one packed conversion.
__device__ __forceinline__ uint32_t f32x2_to_f16x2_sat(float a, float b, int &sat) {
    if (fabsf(a) < 65504.0f && fabsf(b) < 65504.0f) {      // (false for NaN)
        const __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<const uint32_t *>(&h);
    }
    int s0 = 0, s1 = 0;
    const uint32_t lo = f32_to_f16_sat(a, s0), hi = f32_to_f16_sat(b, s1);
    sat += s0 + s1;
    return lo | (hi << 16);
}

// A finite, non-negative radius to fp16 bits: round to nearest even,
// saturating at 65504 (values from 65520 up would round to inf).
__device__ __forceinline__ uint16_t radius_to_f16(float r, int &sat) {
    if (r >= 65520.0f) {
        sat = 1;
        return 0x7BFFu;
    }
    return __half_as_ushort(__float2half_rn(r));
}

__device__ __forceinline__ float f16_bits_to_f32(uint32_t h) {
    return __half2float(__ushort_as_half((unsigned short)h));
}

// Element e of the input (bf16 bits or fp32).
template <int DT>
__device__ __forceinline__ void load_chunk(const void *x, size_t j, float &x0, float &x1,
                                           float &x2, float &x3) {
    if (DT == HQMQ_BF16) {
        uint2 v = __ldg(reinterpret_cast<const uint2 *>(x) + j);
        x0 = __uint_as_float(v.x << 16);
        x1 = __uint_as_float(v.x & 0xFFFF0000u);
        x2 = __uint_as_float(v.y << 16);
        x3 = __uint_as_float(v.y & 0xFFFF0000u);
    } else {
        float4 v = __ldg(reinterpret_cast<const float4 *>(x) + j);
        x0 = v.x; x1 = v.y; x2 = v.z; x3 = v.w;
    }
}

// Streaming (read-once) variant: evict-first hint for data not reused soon.
template <int DT>
__device__ __forceinline__ void load_chunk_stream(const void *x, size_t j, float &x0, float &x1,
                                                  float &x2, float &x3) {
    if (DT == HQMQ_BF16) {
        uint2 v = __ldcs(reinterpret_cast<const uint2 *>(x) + j);
        x0 = __uint_as_float(v.x << 16);
        x1 = __uint_as_float(v.x & 0xFFFF0000u);
        x2 = __uint_as_float(v.y << 16);
        x3 = __uint_as_float(v.y & 0xFFFF0000u);
    } else {
        float4 v = __ldcs(reinterpret_cast<const float4 *>(x) + j);
        x0 = v.x; x1 = v.y; x2 = v.z; x3 = v.w;
    }
}

// Raw chunk storage (8 bytes for bf16, 16 for fp32) to keep several chunks
// in flight per thread at a low register cost.
template <int DT> struct RawChunk;
template <> struct RawChunk<HQMQ_BF16> {
    uint2 v;
    __device__ __forceinline__ void load(const void *x, size_t j) {
        v = __ldcs(reinterpret_cast<const uint2 *>(x) + j);
    }
    __device__ __forceinline__ void zero() { v = make_uint2(0u, 0u); }
    __device__ __forceinline__ float e(int i) const {
        uint32_t w = (i < 2) ? v.x : v.y;
        return (i & 1) ? __uint_as_float(w & 0xFFFF0000u) : __uint_as_float(w << 16);
    }
};
template <> struct RawChunk<HQMQ_F32> {
    float4 v;
    __device__ __forceinline__ void load(const void *x, size_t j) {
        v = __ldcs(reinterpret_cast<const float4 *>(x) + j);
    }
    __device__ __forceinline__ void zero() { v = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ float e(int i) const {
        return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
    }
};

// 2T element p as fp32 (w, i, j, k).
__device__ __forceinline__ void element_2t(int p, float &a0, float &a1, float &a2, float &a3) {
    if (p < 8) {
        float sg = (p & 1) ? -1.0f : 1.0f;
        int ax = p >> 1;
        a0 = ax == 0 ? sg : 0.0f;
        a1 = ax == 1 ? sg : 0.0f;
        a2 = ax == 2 ? sg : 0.0f;
        a3 = ax == 3 ? sg : 0.0f;
    } else {
        int m = p - 8;
        a0 = (m & 1) ? -0.5f : 0.5f;
        a1 = (m & 2) ? -0.5f : 0.5f;
        a2 = (m & 4) ? -0.5f : 0.5f;
        a3 = (m & 8) ? -0.5f : 0.5f;
    }
}

// Codeword q_p q_s in fp32: each component the left-to-right sum of its four
// Hamilton terms (ij = k), each term one fp32 product.
__device__ __forceinline__ float4 codeword(int p, float4 q) {
    float a0, a1, a2, a3;
    element_2t(p, a0, a1, a2, a3);
    float4 c;
    float t;
    t = __fmul_rn(a0, q.x); t = __fsub_rn(t, __fmul_rn(a1, q.y));
    t = __fsub_rn(t, __fmul_rn(a2, q.z)); t = __fsub_rn(t, __fmul_rn(a3, q.w)); c.x = t;
    t = __fmul_rn(a0, q.y); t = __fadd_rn(t, __fmul_rn(a1, q.x));
    t = __fadd_rn(t, __fmul_rn(a2, q.w)); t = __fsub_rn(t, __fmul_rn(a3, q.z)); c.y = t;
    t = __fmul_rn(a0, q.z); t = __fsub_rn(t, __fmul_rn(a1, q.w));
    t = __fadd_rn(t, __fmul_rn(a2, q.x)); t = __fadd_rn(t, __fmul_rn(a3, q.y)); c.z = t;
    t = __fmul_rn(a0, q.w); t = __fadd_rn(t, __fmul_rn(a1, q.z));
    t = __fsub_rn(t, __fmul_rn(a2, q.y)); t = __fadd_rn(t, __fmul_rn(a3, q.x)); c.w = t;
    return c;
}

// Quantized-radius mode: the step delta = fl32(thr / (L - 1)) of a head
// (0 unless thr is a positive finite value), and the radius fl32(k delta) of
// level k (codes >= L read as L - 1).
__device__ __forceinline__ float qr_delta(float thr, uint32_t L) {
    if (!(thr > 0.0f) || isinf(thr) || L < 2u) return 0.0f;
    return __fdiv_rn(thr, (float)(L - 1u));
}
__device__ __forceinline__ float qr_radius(uint32_t k, uint32_t L, float delta) {
    return __fmul_rn((float)(k < L ? k : L - 1u), delta);
}

__device__ __forceinline__ void status_add(DevStatus *st, unsigned flag,
                                           unsigned long long *ctr, unsigned long long n) {
    if (st && n) {
        atomicOr(&st->flags, flag);
        atomicAdd(ctr, n);
    }
}

// Programmatic dependent launch (sm_90 and later): a kernel launched with
// launch_pdl may be scheduled while the previous kernel on its stream is
// still running; it executes pdl_wait() before its first access to global
// memory, which returns once that kernel has completed and its writes are
// visible, so any predecessor is safe.  pdl_trigger() lets the next such
// kernel be scheduled before this one ends.  Only the launch latency and the
// CTAs' start overlap the predecessor.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace hqmq
