// decode.cu -- HQMQ decode: unpack -> quaternion product -> scale -> outliers.
//
// x_hat = r (q_p q_s): the stored fp16 radius times the effective codeword
// (gist.science/nl, Technische Samenvatting, Methodologie and section 1); the
// Med3x outliers kept in fp16 (section 3) are restored.  The pages run this
// inside their attention kernel ("Memory en Latentie"); here it is a
// standalone streaming kernel that writes the dense bf16 (or fp32) tensor.
//
// Each CTA owns one slab (b, h) and builds that head's 24 S codeword table in
// shared memory once (for S <= 170; larger S recomputes the codeword per
// chunk).  Threads decode 2 consecutive chunks per step, so every output
// store is one aligned 16-byte vector (8 bf16).  The slab is cut into
// ranges of RANGE chunks; after a range's main pass the CTA applies that
// range's outliers (chunk mode: overwrite after a barrier; element mode: an
// add-back buffer in shared memory, pre-filled with -0.0, the exact additive
// identity).
#include "hqmq_device.cuh"

namespace hqmq {

constexpr int DEC_THREADS = 256;
constexpr int RANGE = 2048;          // chunks per range (8 per thread)
constexpr int MODE_NONE = 0, MODE_CHUNK = 1, MODE_ELEM = 2;

__device__ __forceinline__ uint32_t get_index(const uint32_t *__restrict__ words, uint64_t grp,
                                              uint32_t k, uint32_t b) {
    const uint32_t *w = words + grp * b;
    uint32_t bit = k * b;
    uint32_t o = bit & 31u;
    uint64_t v = __ldg(w + (bit >> 5));
    if (o + b > 32u) v |= (uint64_t)__ldg(w + (bit >> 5) + 1) << 32;
    return (uint32_t)(v >> o) & ((1u << b) - 1u);
}

// First position in [lo, hi) with key >= v (keys ascending).
__device__ __forceinline__ uint32_t lower_bound(const uint32_t *__restrict__ keys, uint32_t lo,
                                                uint32_t hi, uint32_t v) {
    while (lo < hi) {
        uint32_t mid = lo + ((hi - lo) >> 1);
        if (__ldg(keys + mid) < v) lo = mid + 1; else hi = mid;
    }
    return lo;
}

template <int OUT_DT, int MODE, bool TABLE>
__global__ void __launch_bounds__(DEC_THREADS)
k_decode(const uint32_t *__restrict__ words, const uint16_t *__restrict__ radius,
         const float4 *__restrict__ cb_all, uint32_t S, uint32_t b,
         const uint32_t *__restrict__ out_idx, const uint16_t *__restrict__ out_val,
         const uint32_t *__restrict__ slab_off, uint64_t cap, int H, uint32_t chunks_per_slab,
         void *__restrict__ y, DevStatus *st) {
    extern __shared__ float4 smem[];
    float4 *s_tab = smem;                                            // [24 S] if TABLE
    float *s_add = reinterpret_cast<float *>(smem + (TABLE ? 24 * S : 0));  // [RANGE*4]
    __shared__ uint32_t s_rng[2];

    const int slab = blockIdx.y;
    const int h = slab % H;
    const float4 *cb = cb_all + (size_t)h * S;
    const uint32_t n_words = 24u * S;
    if (TABLE) {
        for (uint32_t i = threadIdx.x; i < n_words; i += DEC_THREADS)
            s_tab[i] = codeword((int)(i % 24u), __ldg(cb + i / 24u));
        __syncthreads();
    }
    const uint64_t chunk0 = (uint64_t)slab * chunks_per_slab;     // first chunk of the slab
    uint32_t o_lo = 0, o_hi = 0;                                     // this slab's list entries
    if (MODE != MODE_NONE) {
        uint64_t a = slab_off[slab], e = slab_off[slab + 1];
        o_lo = (uint32_t)(a < cap ? a : cap);
        o_hi = (uint32_t)(e < cap ? e : cap);
    }
    unsigned n_bad = 0;
    const uint32_t n_ranges = (chunks_per_slab + RANGE - 1) / RANGE;
    for (uint32_t rg = blockIdx.x; rg < n_ranges; rg += gridDim.x) {
        const uint32_t c0 = rg * RANGE;
        const uint32_t c1 = min(c0 + RANGE, chunks_per_slab);
        if (MODE != MODE_NONE) {
            if (threadIdx.x == 0) {
                uint32_t base = (uint32_t)(MODE == MODE_ELEM ? 4 : 1);
                uint32_t lo_key = (uint32_t)((chunk0 + c0) * base);
                uint32_t hi_key = (uint32_t)((chunk0 + c1) * base);
                uint32_t lo = lower_bound(out_idx, o_lo, o_hi, lo_key);
                s_rng[0] = lo;
                s_rng[1] = lower_bound(out_idx, lo, o_hi, hi_key);
            }
            if (MODE == MODE_ELEM)
                for (int i = threadIdx.x; i < RANGE * 4; i += DEC_THREADS) s_add[i] = -0.0f;
            __syncthreads();
            if (MODE == MODE_ELEM) {
                const uint32_t e0 = (uint32_t)((chunk0 + c0) * 4);
                const uint32_t n_e = (c1 - c0) * 4;
                for (uint32_t q = s_rng[0] + threadIdx.x; q < s_rng[1]; q += DEC_THREADS) {
                    const uint32_t e = __ldg(out_idx + q) - e0;
                    if (e < n_e) s_add[e] = f16_bits_to_f32(__ldg(out_val + q));   // unsorted list guard
                }
                __syncthreads();
            }
        }
        for (uint32_t c = c0 + 2 * threadIdx.x; c < c1; c += 2 * DEC_THREADS) {
            const uint64_t j = chunk0 + c;                 // even: (T*D/4) % 32 == 0
            const uint32_t rr2 = __ldg(reinterpret_cast<const uint32_t *>(radius) + (j >> 1));
            const uint64_t grp = j >> 5;
            const uint32_t k = (uint32_t)(j & 31u);
            float out[8];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                uint32_t idx = get_index(words, grp, k + u, b);
                float r = f16_bits_to_f32(u ? (rr2 >> 16) : (rr2 & 0xFFFFu));
                float4 cw;
                if (idx < n_words) {
                    cw = TABLE ? s_tab[idx] : codeword((int)(idx % 24u), __ldg(cb + idx / 24u));
                } else {
                    cw = make_float4(0.f, 0.f, 0.f, 0.f);
                    r = 0.0f;
                    ++n_bad;
                }
                out[4 * u + 0] = __fmul_rn(r, cw.x);
                out[4 * u + 1] = __fmul_rn(r, cw.y);
                out[4 * u + 2] = __fmul_rn(r, cw.z);
                out[4 * u + 3] = __fmul_rn(r, cw.w);
            }
            if (MODE == MODE_ELEM) {
                const float *ad = s_add + (c - c0) * 4;
#pragma unroll
                for (int i = 0; i < 8; ++i) out[i] = __fadd_rn(out[i], ad[i]);
            }
            if (OUT_DT == HQMQ_BF16) {
                uint4 v;
                __nv_bfloat162 p0 = __floats2bfloat162_rn(out[0], out[1]);
                __nv_bfloat162 p1 = __floats2bfloat162_rn(out[2], out[3]);
                __nv_bfloat162 p2 = __floats2bfloat162_rn(out[4], out[5]);
                __nv_bfloat162 p3 = __floats2bfloat162_rn(out[6], out[7]);
                v.x = *reinterpret_cast<uint32_t *>(&p0);
                v.y = *reinterpret_cast<uint32_t *>(&p1);
                v.z = *reinterpret_cast<uint32_t *>(&p2);
                v.w = *reinterpret_cast<uint32_t *>(&p3);
                __stcs(reinterpret_cast<uint4 *>(y) + (j >> 1), v);
            } else {
                float4 *yp = reinterpret_cast<float4 *>(y) + j;
                __stcs(yp, make_float4(out[0], out[1], out[2], out[3]));
                __stcs(yp + 1, make_float4(out[4], out[5], out[6], out[7]));
            }
        }
        if (MODE == MODE_CHUNK) {
            __syncthreads();   // main-pass stores of this range precede the overwrite
            for (uint32_t q = s_rng[0] + threadIdx.x; q < s_rng[1]; q += DEC_THREADS) {
                const uint64_t j = __ldg(out_idx + q);
                if (j < chunk0 + c0 || j >= chunk0 + c1) continue;   // unsorted list guard
                const uint32_t *vv = reinterpret_cast<const uint32_t *>(out_val + (size_t)q * 4);
                uint32_t v01 = __ldg(vv), v23 = __ldg(vv + 1);
                float f0 = f16_bits_to_f32(v01 & 0xFFFFu), f1 = f16_bits_to_f32(v01 >> 16);
                float f2 = f16_bits_to_f32(v23 & 0xFFFFu), f3 = f16_bits_to_f32(v23 >> 16);
                if (OUT_DT == HQMQ_BF16) {
                    __nv_bfloat162 p0 = __floats2bfloat162_rn(f0, f1);
                    __nv_bfloat162 p1 = __floats2bfloat162_rn(f2, f3);
                    uint2 v;
                    v.x = *reinterpret_cast<uint32_t *>(&p0);
                    v.y = *reinterpret_cast<uint32_t *>(&p1);
                    reinterpret_cast<uint2 *>(y)[j] = v;
                } else {
                    reinterpret_cast<float4 *>(y)[j] = make_float4(f0, f1, f2, f3);
                }
            }
        }
        if (MODE != MODE_NONE) __syncthreads();   // s_rng / s_add reuse by the next range
    }
    unsigned nb = __reduce_add_sync(FULL, n_bad);
    if ((threadIdx.x & 31) == 0 && nb && st) atomicOr(&st->flags, HQMQ_FLAG_BAD_INDEX);
}

template <int OUT_DT, int MODE, bool TABLE>
static int launch_t(const uint32_t *words, const uint16_t *radius, const float *cb, uint32_t S,
                    uint32_t b, const uint32_t *out_idx, const uint16_t *out_val,
                    const uint32_t *slab_off, uint64_t cap, int B, int H,
                    uint32_t chunks_per_slab, void *y, hqmq_status *st, int sm_count,
                    cudaStream_t stream) {
    auto kern = k_decode<OUT_DT, MODE, TABLE>;
    size_t smem = (TABLE ? (size_t)24 * S * sizeof(float4) : 0) +
                  (MODE == MODE_ELEM ? (size_t)RANGE * 4 * sizeof(float) : 0);
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return HQMQ_ERR_CUDA;
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, DEC_THREADS, smem) !=
            cudaSuccess || occ < 1)
        occ = 1;
    int n_slabs = B * H;
    uint64_t ranges = (chunks_per_slab + RANGE - 1) / RANGE;
    uint64_t fill = ((uint64_t)sm_count * occ + n_slabs - 1) / n_slabs;
    uint64_t gx = ranges < fill ? ranges : fill;
    if (gx < 1) gx = 1;
    dim3 grid((unsigned)gx, (unsigned)n_slabs);
    kern<<<grid, DEC_THREADS, smem, stream>>>(words, radius, reinterpret_cast<const float4 *>(cb),
                                              S, b, out_idx, out_val, slab_off, cap, H,
                                              chunks_per_slab, y,
                                              reinterpret_cast<DevStatus *>(st));
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

template <int OUT_DT, int MODE>
static int launch_m(bool table, const uint32_t *words, const uint16_t *radius, const float *cb,
                    uint32_t S, uint32_t b, const uint32_t *out_idx, const uint16_t *out_val,
                    const uint32_t *slab_off, uint64_t cap, int B, int H, uint32_t cps, void *y,
                    hqmq_status *st, int sm, cudaStream_t stream) {
    return table ? launch_t<OUT_DT, MODE, true>(words, radius, cb, S, b, out_idx, out_val, slab_off,
                                                cap, B, H, cps, y, st, sm, stream)
                 : launch_t<OUT_DT, MODE, false>(words, radius, cb, S, b, out_idx, out_val,
                                                 slab_off, cap, B, H, cps, y, st, sm, stream);
}

template <int OUT_DT>
static int launch_o(int mode, bool table, const uint32_t *words, const uint16_t *radius,
                    const float *cb, uint32_t S, uint32_t b, const uint32_t *out_idx,
                    const uint16_t *out_val, const uint32_t *slab_off, uint64_t cap, int B, int H,
                    uint32_t cps, void *y, hqmq_status *st, int sm, cudaStream_t stream) {
    if (mode == MODE_CHUNK)
        return launch_m<OUT_DT, MODE_CHUNK>(table, words, radius, cb, S, b, out_idx, out_val,
                                            slab_off, cap, B, H, cps, y, st, sm, stream);
    if (mode == MODE_ELEM)
        return launch_m<OUT_DT, MODE_ELEM>(table, words, radius, cb, S, b, out_idx, out_val,
                                           slab_off, cap, B, H, cps, y, st, sm, stream);
    return launch_m<OUT_DT, MODE_NONE>(table, words, radius, cb, S, b, out_idx, out_val, slab_off,
                                       cap, B, H, cps, y, st, sm, stream);
}

}  // namespace hqmq

extern "C" int hqmq_launch_decode(const uint32_t *words, const uint16_t *radius, const float *cb,
                                  uint32_t S, uint32_t b, const uint32_t *out_idx,
                                  const uint16_t *out_val, const uint32_t *slab_off, uint64_t cap,
                                  int gran, int B, int H, int T, int D, void *y, int out_dtype,
                                  hqmq_status *st, int sm_count, cudaStream_t stream) {
    using namespace hqmq;
    uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    int mode = out_idx == nullptr ? MODE_NONE : (gran == HQMQ_GRAN_CHUNK ? MODE_CHUNK : MODE_ELEM);
    bool table = S <= 170;
    if (out_dtype == HQMQ_BF16)
        return launch_o<HQMQ_BF16>(mode, table, words, radius, cb, S, b, out_idx, out_val, slab_off,
                                   cap, B, H, cps, y, st, sm_count, stream);
    return launch_o<HQMQ_F32>(mode, table, words, radius, cb, S, b, out_idx, out_val, slab_off,
                              cap, B, H, cps, y, st, sm_count, stream);
}
