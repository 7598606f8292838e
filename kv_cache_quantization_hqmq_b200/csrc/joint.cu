// joint.cu -- the pages' bit budget: one mixed-radix code for a chunk's
// (index, radius level) pair, and the per-chunk outlier flag.
//
// The pages give 3.79 bits per element at S = 8 and about 5 at S = 32
// (signal-ia-rouge, "La mecanique"; abstract): two digits of 24 S values per
// chunk of four elements.  With the quantized radius (qradius.cu: level k of
// L = 24 S on [0, thr_h]) each chunk carries the digit D = idx * L + k in
// base L^2; n consecutive chunks of a slab form one block value
// V = sum_c D_c (L^2)^c (least significant chunk first), n the largest count
// with L^(2n) < 2^64, stored in w = bit length of L^(2n) - 1 bits.  Every
// slab's blocks (its last one padded with zero digits) are packed LSB-first
// into its own run of 32-bit words: 3.8125 bits per element at S = 8
// (n = 4, w = 61), 4.833 at S = 32 (n = 3, w = 58).
//
// Outliers (chunk mode) keep their fp16 values in the list's order; the
// pages mark them with a 1-bit flag (gist.science/nl, Technische
// Samenvatting, section 3): bit c of flag word g is set for chunk 32 g + c.
// A chunk's value is the q-th of its list tile (1024 chunks), q = its rank
// among the tile's set flags; the list's tile offsets give each tile's first
// value.
//
// k_pack_joint   one thread per output word: the (at most two, w > 32)
//                blocks that overlap it, each from its chunks' b-bit index and
//                level fields.
// k_decode_joint one thread per block: V -> digits -> (idx, k) -> r k-th
//                level times the codeword (table in shared memory) -> bf16.
// k_list_flags   one thread per list entry: sets the entry's flag bit.
// k_apply_flags  one warp per list tile: each flagged chunk becomes its fp16
//                values (after k_decode_joint, on the same stream).
#include "med3_window.cuh"

namespace hqmq {

constexpr int JT_THREADS = 256;

struct JointGeom {
    uint32_t L, n, w;          // levels (= codewords), chunks per block, bits per block
    uint64_t m;                // L^2
    uint64_t cps, nb, wps;     // chunks, blocks and words per slab
};

inline JointGeom joint_geom(int T, int D, uint32_t S) {
    JointGeom g;
    g.L = 24u * S;
    g.m = (uint64_t)g.L * g.L;
    uint64_t p = 1;
    g.n = 0;
    while (p <= ~0ull / g.m) { p *= g.m; ++g.n; }            // p = L^(2n) < 2^64
    const uint64_t top = p - 1;
    g.w = 0;
    while (g.w < 64 && (top >> g.w) != 0) ++g.w;
    g.cps = (uint64_t)T * D / 4;
    g.nb = (g.cps + g.n - 1) / g.n;
    g.wps = (g.nb * g.w + 31) / 32;
    return g;
}

// b-bit field of chunk j (LSB-first, groups of 32 chunks in b words)
__device__ __forceinline__ uint32_t field(const uint32_t *__restrict__ words, uint64_t j,
                                          uint32_t b) {
    const uint32_t *w = words + (j >> 5) * b;
    const uint32_t bit = (uint32_t)(j & 31u) * b, o = bit & 31u;
    const uint32_t lo = __ldg(w + (bit >> 5));
    const uint32_t hi = o + b > 32u ? __ldg(w + (bit >> 5) + 1) : 0u;
    return __funnelshift_r(lo, hi, o) & ((1u << b) - 1u);
}

// V = q * m + r for m < 2^32 (here m = L^2 < 2^21): the high word by a 32-bit
// division, the rest (below m 2^32 < 2^53) in fp64 and one integer correction
__device__ __forceinline__ uint64_t divmod_m(uint64_t v, uint32_t m, double inv_m, uint32_t &r) {
    const uint32_t hi = (uint32_t)(v >> 32);
    const uint32_t qh = hi / m;
    const uint64_t t = ((uint64_t)(hi - qh * m) << 32) | (uint32_t)v;   // < m 2^32
    uint64_t ql = (uint64_t)__dmul_rz((double)t, inv_m);
    int64_t rr = (int64_t)(t - ql * m);
    if (rr < 0) { --ql; rr += m; }
    if (rr >= (int64_t)m) { ++ql; rr -= m; }
    r = (uint32_t)rr;
    return ((uint64_t)qh << 32) + ql;
}

// Block q of slab s: its value from its chunks' fields (0 past the slab;
// an index or level not below L counts as bad and gives digit 0).
__device__ __forceinline__ uint64_t block_value(const uint32_t *__restrict__ iw,
                                                const uint32_t *__restrict__ kw, uint32_t b,
                                                const JointGeom &g, uint64_t s, uint64_t q,
                                                unsigned &bad) {
    uint64_t v = 0, p = 1;
    for (uint32_t c = 0; c < g.n; ++c) {
        const uint64_t jl = q * g.n + c;
        uint64_t d = 0;
        if (jl < g.cps) {
            const uint64_t j = s * g.cps + jl;
            const uint32_t idx = field(iw, j, b), k = field(kw, j, b);
            if (idx < g.L && k < g.L) d = (uint64_t)idx * g.L + k;
            else ++bad;
        }
        v += d * p;
        p *= g.m;
    }
    return v;
}

__global__ void __launch_bounds__(JT_THREADS)
k_pack_joint(const uint32_t *__restrict__ iw, const uint32_t *__restrict__ kw, uint32_t b,
             JointGeom g, uint64_t n_words, uint32_t *__restrict__ joint, DevStatus *st) {
    unsigned bad = 0;
    for (uint64_t t = (uint64_t)blockIdx.x * JT_THREADS + threadIdx.x; t < n_words;
         t += (uint64_t)gridDim.x * JT_THREADS) {
        const uint64_t s = t / g.wps, wi = t % g.wps;
        const uint64_t bit0 = wi * 32;                       // this word's first bit
        uint64_t word = 0;
        for (uint64_t q = bit0 / g.w; q < g.nb && q * g.w < bit0 + 32; ++q) {
            unsigned bq = 0;
            const uint64_t v = block_value(iw, kw, b, g, s, q, bq);
            const uint64_t qb = q * g.w;                     // the block's first bit
            if (qb >= bit0) {
                word |= v << (qb - bit0);                    // (qb - bit0 < 32)
                bad += bq;                                   // (counted by the word it starts in)
            } else {
                word |= v >> (bit0 - qb);                    // (bit0 - qb < w <= 64)
            }
        }
        joint[t] = (uint32_t)word;
    }
    const unsigned tot = __reduce_add_sync(FULL, bad);
    if ((threadIdx.x & 31) == 0 && tot && st) atomicOr(&st->flags, HQMQ_FLAG_BAD_INDEX);
}

template <int OUT_DT>
__global__ void __launch_bounds__(JT_THREADS)
k_decode_joint(const uint32_t *__restrict__ joint, JointGeom g, int H,
               const float *__restrict__ thr, const float4 *__restrict__ cb_all, uint32_t S,
               uint32_t blocks_per_cta, void *__restrict__ y) {
    extern __shared__ float4 s_tab[];                   // [24 S] this slab's codewords
    const uint64_t s = blockIdx.y;                      // slab
    const int h = (int)(s % (uint64_t)H);
    const float4 *cb = cb_all + (size_t)h * S;
    for (uint32_t i = threadIdx.x; i < g.L; i += JT_THREADS)
        s_tab[i] = codeword((int)(i % 24u), __ldg(cb + i / 24u));
    __syncthreads();
    const float delta = qr_delta(__ldg(thr + h), g.L);
    const double inv_m = 1.0 / (double)g.m;
    const uint32_t *run = joint + s * g.wps;
    const uint64_t q_lim = (uint64_t)(blockIdx.x + 1) * blocks_per_cta;
    const uint64_t q_end = g.nb < q_lim ? g.nb : q_lim;
    for (uint64_t q = (uint64_t)blockIdx.x * blocks_per_cta + threadIdx.x; q < q_end;
         q += JT_THREADS) {
        const uint64_t bit0 = q * g.w;
        const uint64_t wi = bit0 >> 5;
        const uint32_t o = (uint32_t)(bit0 & 31u);
        const uint64_t lo = (uint64_t)__ldg(run + wi) | ((wi + 1 < g.wps ? (uint64_t)__ldg(run + wi + 1) : 0ull) << 32);
        uint64_t v = lo >> o;
        if (o + g.w > 64u && wi + 2 < g.wps)
            v |= (uint64_t)__ldg(run + wi + 2) << (64u - o);
        if (g.w < 64u) v &= (1ull << g.w) - 1ull;
        for (uint32_t c = 0; c < g.n; ++c) {
            const uint64_t jl = q * g.n + c;
            uint32_t d;
            v = divmod_m(v, (uint32_t)g.m, inv_m, d);
            if (jl >= g.cps) break;
            const uint32_t idx = d / g.L, k = d - idx * g.L;
            const float r = qr_radius(k, g.L, delta);
            const float4 cw = s_tab[idx];
            const float o0 = __fmul_rn(r, cw.x), o1 = __fmul_rn(r, cw.y);
            const float o2 = __fmul_rn(r, cw.z), o3 = __fmul_rn(r, cw.w);
            const uint64_t j = s * g.cps + jl;
            if (OUT_DT == HQMQ_BF16) {
                __nv_bfloat162 a0 = __floats2bfloat162_rn(o0, o1);
                __nv_bfloat162 a1 = __floats2bfloat162_rn(o2, o3);
                uint2 out;
                out.x = *reinterpret_cast<uint32_t *>(&a0);
                out.y = *reinterpret_cast<uint32_t *>(&a1);
                reinterpret_cast<uint2 *>(y)[j] = out;
            } else {
                reinterpret_cast<float4 *>(y)[j] = make_float4(o0, o1, o2, o3);
            }
        }
    }
}

__global__ void __launch_bounds__(JT_THREADS)
k_list_flags(const uint32_t *__restrict__ out_idx, const uint32_t *__restrict__ total,
             uint64_t cap, uint64_t n_chunks, uint32_t *__restrict__ flags) {
    uint64_t n = *total;
    if (n > cap) n = cap;
    for (uint64_t q = (uint64_t)blockIdx.x * JT_THREADS + threadIdx.x; q < n;
         q += (uint64_t)gridDim.x * JT_THREADS) {
        const uint32_t j = __ldg(out_idx + q);
        if (j < n_chunks) atomicOr(flags + (j >> 5), 1u << (j & 31u));
    }
}

template <int OUT_DT>
__global__ void __launch_bounds__(JT_THREADS)
k_apply_flags(const uint32_t *__restrict__ flags, const uint16_t *__restrict__ out_val,
              const uint32_t *__restrict__ tile_off, uint32_t cap32, uint32_t gps,
              uint32_t tps, uint64_t n_tiles, void *__restrict__ y) {
    const int lane = threadIdx.x & 31;
    const uint64_t warp_g = (uint64_t)blockIdx.x * (JT_THREADS / 32) + (threadIdx.x >> 5);
    const uint64_t n_warps = (uint64_t)gridDim.x * (JT_THREADS / 32);
    for (uint64_t t = warp_g; t < n_tiles; t += n_warps) {
        const uint64_t slab = t / tps;
        const uint32_t g0 = (uint32_t)(t % tps) * TILE_GROUPS;
        const uint32_t ng = min((uint32_t)TILE_GROUPS, gps - g0);
        const uint64_t G = slab * gps + g0 + lane;       // this lane's packing group
        const uint32_t f = (uint32_t)lane < ng ? __ldg(flags + G) : 0u;
        const uint32_t cnt = __popc(f);
        uint32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(FULL, incl, o);
            if (lane >= o) incl += u;
        }
        uint32_t pos = __ldg(tile_off + t) + incl - cnt;  // the lane's first value
        for (uint32_t m = f; m; m &= m - 1u, ++pos) {
            if (pos >= cap32) break;
            const uint32_t c = __ffs(m) - 1u;
            const uint64_t j = G * 32 + c;
            const uint32_t *vv = reinterpret_cast<const uint32_t *>(out_val + (uint64_t)pos * 4);
            const uint32_t v01 = __ldg(vv), v23 = __ldg(vv + 1);
            const float f0 = f16_bits_to_f32(v01 & 0xFFFFu), f1 = f16_bits_to_f32(v01 >> 16);
            const float f2 = f16_bits_to_f32(v23 & 0xFFFFu), f3 = f16_bits_to_f32(v23 >> 16);
            if (OUT_DT == HQMQ_BF16) {
                __nv_bfloat162 a0 = __floats2bfloat162_rn(f0, f1);
                __nv_bfloat162 a1 = __floats2bfloat162_rn(f2, f3);
                uint2 out;
                out.x = *reinterpret_cast<uint32_t *>(&a0);
                out.y = *reinterpret_cast<uint32_t *>(&a1);
                reinterpret_cast<uint2 *>(y)[j] = out;
            } else {
                reinterpret_cast<float4 *>(y)[j] = make_float4(f0, f1, f2, f3);
            }
        }
    }
}

static int grid_for(uint64_t items, int sm_count) {
    uint64_t b = (items + JT_THREADS - 1) / JT_THREADS;
    const uint64_t cap = (uint64_t)sm_count * 16;
    if (b > cap) b = cap;
    return (int)(b < 1 ? 1 : b);
}

}  // namespace hqmq

extern "C" uint64_t hqmq_launch_joint_words(int B, int H, int T, int D, uint32_t S) {
    return (uint64_t)B * H * hqmq::joint_geom(T, D, S).wps;
}

extern "C" void hqmq_launch_joint_block(uint32_t S, uint32_t *n, uint32_t *w) {
    const hqmq::JointGeom g = hqmq::joint_geom(32, 128, S);
    *n = g.n;
    *w = g.w;
}

extern "C" int hqmq_launch_pack_joint(const uint32_t *iw, const uint32_t *kw, uint32_t S, int B,
                                      int H, int T, int D, uint32_t *joint, hqmq_status *st,
                                      int sm_count, cudaStream_t stream) {
    using namespace hqmq;
    const JointGeom g = joint_geom(T, D, S);
    const uint64_t n_words = (uint64_t)B * H * g.wps;
    uint32_t b = 0;
    while ((1u << b) < g.L) ++b;
    k_pack_joint<<<grid_for(n_words, sm_count), JT_THREADS, 0, stream>>>(
        iw, kw, b, g, n_words, joint, reinterpret_cast<DevStatus *>(st));
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

extern "C" int hqmq_launch_list_flags(const uint32_t *out_idx, const uint32_t *total,
                                      uint64_t cap, uint64_t n_chunks, uint32_t *flags,
                                      int sm_count, cudaStream_t stream) {
    using namespace hqmq;
    if (cudaMemsetAsync(flags, 0, (n_chunks / 32) * sizeof(uint32_t), stream) != cudaSuccess)
        return HQMQ_ERR_CUDA;
    k_list_flags<<<grid_for(cap, sm_count), JT_THREADS, 0, stream>>>(out_idx, total, cap,
                                                                     n_chunks, flags);
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

extern "C" int hqmq_launch_decode_joint(const uint32_t *joint, const float *thr, const float *cb,
                                        uint32_t S, const uint32_t *flags, const uint16_t *out_val,
                                        const uint32_t *tile_off, uint64_t cap, int B, int H,
                                        int T, int D, void *y, int out_dtype, int sm_count,
                                        cudaStream_t stream) {
    using namespace hqmq;
    const JointGeom g = joint_geom(T, D, S);
    const size_t smem = (size_t)g.L * sizeof(float4);
    const int n_slabs = B * H;
    // about four CTAs per SM in all, each a contiguous run of one slab's blocks
    uint64_t per_slab = ((uint64_t)sm_count * 4 + n_slabs - 1) / n_slabs;
    const uint64_t need = (g.nb + JT_THREADS - 1) / JT_THREADS;
    if (per_slab > need) per_slab = need;
    if (per_slab < 1) per_slab = 1;
    const uint32_t bpc = (uint32_t)((g.nb + per_slab - 1) / per_slab);
    dim3 grid((unsigned)per_slab, (unsigned)n_slabs);
    if (out_dtype == HQMQ_BF16) {
        if (smem > 48 * 1024 && cudaFuncSetAttribute(k_decode_joint<HQMQ_BF16>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)smem) != cudaSuccess)
            return HQMQ_ERR_CUDA;
        k_decode_joint<HQMQ_BF16><<<grid, JT_THREADS, smem, stream>>>(
            joint, g, H, thr, reinterpret_cast<const float4 *>(cb), S, bpc, y);
    } else {
        if (smem > 48 * 1024 && cudaFuncSetAttribute(k_decode_joint<HQMQ_F32>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)smem) != cudaSuccess)
            return HQMQ_ERR_CUDA;
        k_decode_joint<HQMQ_F32><<<grid, JT_THREADS, smem, stream>>>(
            joint, g, H, thr, reinterpret_cast<const float4 *>(cb), S, bpc, y);
    }
    if (cudaGetLastError() != cudaSuccess) return HQMQ_ERR_CUDA;
    if (!flags) return HQMQ_OK;
    const uint32_t gps = (uint32_t)(g.cps / 32);
    const uint32_t tps = (gps + TILE_GROUPS - 1) / TILE_GROUPS;
    const uint64_t n_tiles = (uint64_t)n_slabs * tps;
    const uint32_t cap32 = cap < 0xFFFFFFFFull ? (uint32_t)cap : 0xFFFFFFFFu;
    const int gb = grid_for(n_tiles * 32, sm_count);
    if (out_dtype == HQMQ_BF16)
        k_apply_flags<HQMQ_BF16><<<gb, JT_THREADS, 0, stream>>>(flags, out_val, tile_off, cap32,
                                                                gps, tps, n_tiles, y);
    else
        k_apply_flags<HQMQ_F32><<<gb, JT_THREADS, 0, stream>>>(flags, out_val, tile_off, cap32,
                                                               gps, tps, n_tiles, y);
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}
