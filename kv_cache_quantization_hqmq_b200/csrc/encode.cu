// encode.cu -- HQMQ encode: normalise -> search -> pack.
//
// Per chunk x (4 consecutive elements, gist.science/nl, Technische
// Samenvatting, Methodologie) the radius r = |x| is stored in fp16 and the
// direction is snapped to the codeword q_p q_s with the largest inner product
// (section 1 of the same summary).  The search uses
//     <x, q_p q_s> = <x conj(q_s), q_p>            (|q_s| = 1)
// so that per secondary codeword q_s one quaternion product y = x conj(q_s)
// (16 FMA) scores all 24 elements of 2T at once:
//     max_p <y, q_p> = max( max_i |y_i| , (|y_0|+|y_1|+|y_2|+|y_3|) / 2 ),
// the first term from the 8 units +-1,+-i,+-j,+-k, the second from the 16
// half units with the signs of y.  The kernel keeps the best s per chunk and
// resolves p for it in closed form afterwards.
//
// Layout: one warp owns a packing group of 32 consecutive chunks (lane =
// chunk); with CPT groups per warp iteration each lane carries CPT chunks so
// that one shared-memory load of q_s serves CPT chunks.  The b-bit indices of
// a group are assembled with warp shuffles and written as b coalesced words.
#include "hqmq_device.cuh"

namespace hqmq {

// y = x conj(q), conj(q) = (q.x, -q.y, -q.z, -q.w); fixed FMA order.
__device__ __forceinline__ void mul_conj(float x0, float x1, float x2, float x3, float4 q,
                                         float &y0, float &y1, float &y2, float &y3) {
    y0 = __fmaf_rn(x3, q.w, __fmaf_rn(x2, q.z, __fmaf_rn(x1, q.y, __fmul_rn(x0, q.x))));
    y1 = __fmaf_rn(x3, q.z, __fmaf_rn(-x2, q.w, __fmaf_rn(x1, q.x, __fmul_rn(-x0, q.y))));
    y2 = __fmaf_rn(-x3, q.y, __fmaf_rn(x2, q.x, __fmaf_rn(x1, q.w, __fmul_rn(-x0, q.z))));
    y3 = __fmaf_rn(x3, q.x, __fmaf_rn(x2, q.y, __fmaf_rn(-x1, q.z, __fmul_rn(-x0, q.w))));
}

// Twice the best 2T score of y: max(2 max_i |y_i|, sum_i |y_i|) (exact scaling
// of the score by 2, which keeps every comparison).
__device__ __forceinline__ float score2(float y0, float y1, float y2, float y3) {
    float a0 = fabsf(y0), a1 = fabsf(y1), a2 = fabsf(y2), a3 = fabsf(y3);
    float m = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
    float sum = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
    return fmaxf(__fadd_rn(m, m), sum);
}

// Nearest 2T element of y with ties to the lowest p: the axis family (p < 8)
// wins a tie with the half family; among axes the lowest axis; the sign of a
// zero coordinate is taken as +.
__device__ __forceinline__ int closest_2t(float y0, float y1, float y2, float y3) {
    float a0 = fabsf(y0), a1 = fabsf(y1), a2 = fabsf(y2), a3 = fabsf(y3);
    float m = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
    float sum = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
    if (__fadd_rn(m, m) >= sum) {
        int ax = (a0 == m) ? 0 : (a1 == m) ? 1 : (a2 == m) ? 2 : 3;
        float ya = ax == 0 ? y0 : ax == 1 ? y1 : ax == 2 ? y2 : y3;
        return 2 * ax + (ya < 0.0f ? 1 : 0);
    }
    return 8 + (y0 < 0.0f ? 1 : 0) + (y1 < 0.0f ? 2 : 0) + (y2 < 0.0f ? 4 : 0) +
           (y3 < 0.0f ? 8 : 0);
}

// Writes the b words of one group: lane w < b assembles word w from the
// (at most 8) chunks whose bits touch it.
__device__ __forceinline__ void pack_group(uint32_t idx, uint32_t b, int lane,
                                           uint32_t *__restrict__ dst) {
    int w = lane;
    int k0 = (32 * w) / (int)b;
    uint32_t word = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        int k = k0 + t;
        uint32_t v = __shfl_sync(FULL, idx, k & 31);
        int off = k * (int)b - 32 * w;
        if (w < (int)b && k < 32 && off < 32) word |= off >= 0 ? (v << off) : (v >> (-off));
    }
    if (w < (int)b) dst[w] = word;
}

template <int DT, int CPT, bool SMEM_CB>
__global__ void __launch_bounds__(256)
k_encode(const void *__restrict__ x, int H, uint32_t groups_per_slab,
         const float4 *__restrict__ cb_all, uint32_t S, uint32_t b,
         const float *__restrict__ thr, int gran, uint32_t *__restrict__ words,
         uint16_t *__restrict__ radius, DevStatus *st) {
    extern __shared__ float4 s_cb[];
    const int slab = blockIdx.y;
    const int h = slab % H;
    const float4 *cb = cb_all + (size_t)h * S;
    if (SMEM_CB) {
        for (uint32_t i = threadIdx.x; i < S; i += blockDim.x) s_cb[i] = cb[i];
        __syncthreads();
    }
    const float4 *qsrc = SMEM_CB ? s_cb : cb;
    const bool med3 = thr != nullptr;
    const float th = med3 ? thr[h] : 0.0f;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const uint64_t g_base = (uint64_t)slab * groups_per_slab;
    unsigned n_nf = 0, n_sat = 0;

    for (uint32_t unit = blockIdx.x * 8 + warp; unit * CPT < groups_per_slab;
         unit += gridDim.x * 8) {
        float xv[CPT][4];
        float r[CPT];
        bool valid[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            uint32_t gi = unit * CPT + c;
            valid[c] = gi < groups_per_slab;
            float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
            if (valid[c]) load_chunk_stream<DT>(x, (g_base + gi) * 32 + lane, x0, x1, x2, x3);
            if (med3) {
                if (gran == HQMQ_GRAN_CHUNK) {
                    if (chunk_norm(x0, x1, x2, x3) > th) x0 = x1 = x2 = x3 = 0.0f;
                } else {
                    if (fabsf(x0) > th) x0 = 0.0f;
                    if (fabsf(x1) > th) x1 = 0.0f;
                    if (fabsf(x2) > th) x2 = 0.0f;
                    if (fabsf(x3) > th) x3 = 0.0f;
                }
            }
            xv[c][0] = x0; xv[c][1] = x1; xv[c][2] = x2; xv[c][3] = x3;
            r[c] = chunk_norm(x0, x1, x2, x3);
        }
        float best[CPT];
        uint32_t bsel[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c) { best[c] = -1.0f; bsel[c] = 0; }
        for (uint32_t s = 0; s < S; ++s) {
            float4 q = qsrc[s];
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                float y0, y1, y2, y3;
                mul_conj(xv[c][0], xv[c][1], xv[c][2], xv[c][3], q, y0, y1, y2, y3);
                float sc = score2(y0, y1, y2, y3);
                if (sc > best[c]) { best[c] = sc; bsel[c] = s; }
            }
        }
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            float y0, y1, y2, y3;
            mul_conj(xv[c][0], xv[c][1], xv[c][2], xv[c][3], qsrc[bsel[c]], y0, y1, y2, y3);
            int p = closest_2t(y0, y1, y2, y3);
            float rr = r[c];
            bool finite = rr == rr && rr != __int_as_float(0x7F800000);
            uint32_t idx = (finite && rr > 0.0f) ? bsel[c] * 24u + (uint32_t)p : 0u;
            uint16_t rh;
            if (!finite) {
                rh = 0x7E00u;
                n_nf += valid[c] ? 1u : 0u;
            } else {
                int sat = 0;
                rh = f32_to_f16_sat(rr, sat);
                n_sat += (valid[c] && sat) ? 1u : 0u;
            }
            uint32_t gi = unit * CPT + c;
            if (valid[c]) radius[(g_base + gi) * 32 + lane] = rh;
            // `valid` is uniform across the warp: whole groups only
            if (valid[c]) pack_group(idx, b, lane, words + (g_base + gi) * b);
        }
    }
    // warp-aggregated status counters
    unsigned nf = __reduce_add_sync(FULL, n_nf);
    unsigned ns = __reduce_add_sync(FULL, n_sat);
    if (lane == 0 && st) {
        if (nf) status_add(st, HQMQ_FLAG_NONFINITE, &st->n_nonfinite, nf);
        if (ns) status_add(st, HQMQ_FLAG_SATURATED, &st->n_saturated, ns);
    }
}

template <int DT, int CPT, bool SMEM>
static int launch_t(const void *x, int B, int H, uint32_t groups_per_slab, const float *cb,
                    uint32_t S, uint32_t b, const float *thr, int gran, uint32_t *words,
                    uint16_t *radius, hqmq_status *st, int sm_count, cudaStream_t stream) {
    auto kern = k_encode<DT, CPT, SMEM>;
    size_t smem = SMEM ? (size_t)S * sizeof(float4) : 0;
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return HQMQ_ERR_CUDA;
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 256, smem) != cudaSuccess ||
        occ < 1)
        occ = 1;
    int n_slabs = B * H;
    uint64_t units = (groups_per_slab + CPT - 1) / CPT;
    uint64_t want = (units + 7) / 8;                       // CTAs to give every warp one unit
    uint64_t fill = ((uint64_t)sm_count * occ + n_slabs - 1) / n_slabs;
    uint64_t gx = want < fill ? want : fill;
    if (gx < 1) gx = 1;
    dim3 grid((unsigned)gx, (unsigned)n_slabs);
    kern<<<grid, 256, smem, stream>>>(x, H, groups_per_slab, reinterpret_cast<const float4 *>(cb),
                                      S, b, thr, gran, words, radius,
                                      reinterpret_cast<DevStatus *>(st));
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

}  // namespace hqmq

extern "C" int hqmq_launch_encode(const void *x, int dtype, int B, int H, int T, int D,
                                  const float *cb, uint32_t S, uint32_t b, const float *thr,
                                  int gran, uint32_t *words, uint16_t *radius, hqmq_status *st,
                                  int sm_count, cudaStream_t stream) {
    uint32_t groups_per_slab = (uint32_t)(((uint64_t)T * D / 4) / 32);
    const bool smem = (size_t)S * sizeof(float4) <= 96 * 1024;
    using namespace hqmq;
    if (dtype == HQMQ_BF16) {
        return smem ? launch_t<HQMQ_BF16, 2, true>(x, B, H, groups_per_slab, cb, S, b, thr, gran,
                                                   words, radius, st, sm_count, stream)
                    : launch_t<HQMQ_BF16, 2, false>(x, B, H, groups_per_slab, cb, S, b, thr, gran,
                                                    words, radius, st, sm_count, stream);
    }
    return smem ? launch_t<HQMQ_F32, 2, true>(x, B, H, groups_per_slab, cb, S, b, thr, gran, words,
                                              radius, st, sm_count, stream)
                : launch_t<HQMQ_F32, 2, false>(x, B, H, groups_per_slab, cb, S, b, thr, gran, words,
                                               radius, st, sm_count, stream);
}

namespace hqmq {

// ---------------------------------------------------------------------------
// Batched append: C small calls (e.g. one decode step's new tokens of every
// (layer, role)) in one launch, one CTA per call.  Per call c the outputs are
// those of hqmq_outlier_extract_given_thr (list under the given threshold,
// slab and list-tile offsets) followed by hqmq_encode with that threshold.
// ---------------------------------------------------------------------------
constexpr int APP_THREADS = 256;
constexpr int APP_LIST_TILE = 1024;              // chunks per list tile

// Exclusive block-wide scan of v (APP_THREADS threads); *total = the sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *s_warp, uint32_t *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(FULL, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) s_warp[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        const uint32_t w = lane < APP_THREADS / 32 ? s_warp[lane] : 0u;
        uint32_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(FULL, wi, o);
            if (lane >= o) wi += u;
        }
        if (lane < APP_THREADS / 32) s_warp[lane] = wi - w;
        if (lane == APP_THREADS / 32 - 1) s_warp[APP_THREADS / 32] = wi;
    }
    __syncthreads();
    const uint32_t excl = s_warp[wid] + inc - v;
    *total = s_warp[APP_THREADS / 32];
    __syncthreads();                                   // (s_warp reuse)
    return excl;
}

template <int DT, int GRAN>
__global__ void __launch_bounds__(APP_THREADS)
k_append(const void *__restrict__ x_all, int H, uint32_t cps, uint32_t n_slabs,
         const float *__restrict__ thr_all, const float4 *__restrict__ cb_all, uint32_t S,
         uint32_t b, uint32_t *__restrict__ words_all, uint16_t *__restrict__ radius_all,
         uint32_t *__restrict__ out_idx_all, uint16_t *__restrict__ out_val_all,
         uint32_t *__restrict__ slab_off_all, uint32_t *__restrict__ tile_off_all, uint32_t cap,
         DevStatus *st) {
    extern __shared__ float4 s_cb[];                   // this call's H * S secondary codewords
    __shared__ uint32_t s_warp[APP_THREADS / 32 + 1];
    const uint32_t c = blockIdx.x;
    const uint64_t n_chunks = (uint64_t)n_slabs * cps;
    const uint32_t tps = (cps + APP_LIST_TILE - 1) / APP_LIST_TILE;
    const uint32_t esz = DT == HQMQ_BF16 ? 2u : 4u;
    const char *x = reinterpret_cast<const char *>(x_all) + (size_t)c * n_chunks * 4 * esz;
    const float *thr = thr_all + (size_t)c * H;
    const float4 *cb = cb_all + (size_t)c * H * S;
    uint32_t *words = words_all + (size_t)c * (n_chunks / 32) * b;
    uint16_t *radius = radius_all + (size_t)c * n_chunks;
    uint32_t *out_idx = out_idx_all + (size_t)c * cap;
    uint16_t *out_val = out_val_all + (size_t)c * cap * (GRAN == HQMQ_GRAN_CHUNK ? 4 : 1);
    uint32_t *slab_off = slab_off_all + (size_t)c * (n_slabs + 1);
    uint32_t *tile_off = tile_off_all ? tile_off_all + (size_t)c * ((uint64_t)n_slabs * tps + 1)
                                      : nullptr;
    for (uint32_t i = threadIdx.x; i < (uint32_t)H * S; i += APP_THREADS) s_cb[i] = __ldg(cb + i);

    // ---- list: ascending flat index order, one chunk per thread per round ----
    uint64_t running = 0;
    unsigned n_sat = 0;
    for (uint64_t j0 = 0; j0 < n_chunks; j0 += APP_THREADS) {
        const uint64_t j = j0 + threadIdx.x;
        const bool ok = j < n_chunks;
        float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
        float th = 0.f;
        if (ok) {
            load_chunk<DT>(x, j, x0, x1, x2, x3);
            th = __ldg(thr + (uint32_t)((j / cps) % (uint64_t)H));
        }
        uint32_t mask = 0;
        if (ok) {
            if (GRAN == HQMQ_GRAN_CHUNK)
                mask = chunk_norm(x0, x1, x2, x3) > th ? 1u : 0u;
            else
                mask = (fabsf(x0) > th ? 1u : 0u) | (fabsf(x1) > th ? 2u : 0u) |
                       (fabsf(x2) > th ? 4u : 0u) | (fabsf(x3) > th ? 8u : 0u);
        }
        uint32_t tot;
        const uint32_t ex = block_excl_scan(__popc(mask), s_warp, &tot);
        const uint64_t pos = running + ex;
        if (ok) {
            const uint32_t cs = (uint32_t)(j % cps);
            if (cs == 0) slab_off[j / cps] = (uint32_t)pos;
            if (tile_off && cs % APP_LIST_TILE == 0)
                tile_off[(j / cps) * tps + cs / APP_LIST_TILE] = (uint32_t)pos;
        }
        if (GRAN == HQMQ_GRAN_CHUNK) {
            if (mask && pos < cap) {
                int sv = 0;
                const uint32_t h01 = f32x2_to_f16x2_sat(x0, x1, sv);
                const uint32_t h23 = f32x2_to_f16x2_sat(x2, x3, sv);
                n_sat += sv;
                out_idx[pos] = (uint32_t)j;
                reinterpret_cast<uint2 *>(out_val)[pos] = make_uint2(h01, h23);
            }
        } else {
            const float xs[4] = {x0, x1, x2, x3};
            uint64_t p = pos;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (mask & (1u << i)) {
                    if (p < cap) {
                        int sv = 0;
                        out_val[p] = f32_to_f16_sat(xs[i], sv);
                        n_sat += sv;
                        out_idx[p] = (uint32_t)(4 * j + i);
                    }
                    ++p;
                }
            }
        }
        running += tot;
    }
    if (threadIdx.x == 0) {
        slab_off[n_slabs] = (uint32_t)running;
        if (tile_off) tile_off[(uint64_t)n_slabs * tps] = (uint32_t)running;
        if (st) {
            atomicAdd(&st->n_outliers, (unsigned long long)running);
            if (running > cap) atomicOr(&st->flags, HQMQ_FLAG_OUTLIER_OVERFLOW);
        }
    }

    // ---- encode: a warp per packing group, the arithmetic of k_encode ----
    __syncthreads();                                   // s_cb ready
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned n_nf = 0;
    for (uint64_t g = warp; g < n_chunks / 32; g += APP_THREADS / 32) {
        const uint64_t j = g * 32 + lane;
        const int h = (int)((j / cps) % (uint64_t)H);
        const float th = __ldg(thr + h);
        float x0, x1, x2, x3;
        load_chunk<DT>(x, j, x0, x1, x2, x3);
        if (GRAN == HQMQ_GRAN_CHUNK) {
            if (chunk_norm(x0, x1, x2, x3) > th) x0 = x1 = x2 = x3 = 0.0f;
        } else {
            if (fabsf(x0) > th) x0 = 0.0f;
            if (fabsf(x1) > th) x1 = 0.0f;
            if (fabsf(x2) > th) x2 = 0.0f;
            if (fabsf(x3) > th) x3 = 0.0f;
        }
        const float r = chunk_norm(x0, x1, x2, x3);
        const float4 *qs = s_cb + (size_t)h * S;
        float best = -1.0f;
        uint32_t bsel = 0;
        for (uint32_t s = 0; s < S; ++s) {
            float y0, y1, y2, y3;
            mul_conj(x0, x1, x2, x3, qs[s], y0, y1, y2, y3);
            const float sc = score2(y0, y1, y2, y3);
            if (sc > best) { best = sc; bsel = s; }
        }
        float y0, y1, y2, y3;
        mul_conj(x0, x1, x2, x3, qs[bsel], y0, y1, y2, y3);
        const int p = closest_2t(y0, y1, y2, y3);
        const bool finite = r == r && r != __int_as_float(0x7F800000);
        const uint32_t idx = (finite && r > 0.0f) ? bsel * 24u + (uint32_t)p : 0u;
        uint16_t rh;
        if (!finite) {
            rh = 0x7E00u;
            ++n_nf;
        } else {
            int sat = 0;
            rh = f32_to_f16_sat(r, sat);
            n_sat += sat;
        }
        radius[j] = rh;
        pack_group(idx, b, lane, words + g * b);
    }
    const unsigned nf = __reduce_add_sync(FULL, n_nf), ns = __reduce_add_sync(FULL, n_sat);
    if (lane == 0 && st) {
        if (nf) status_add(st, HQMQ_FLAG_NONFINITE, &st->n_nonfinite, nf);
        if (ns) status_add(st, HQMQ_FLAG_SATURATED, &st->n_saturated, ns);
    }
}

}  // namespace hqmq

extern "C" int hqmq_launch_append(const void *x, int dtype, int n_calls, int B, int H, int T, int D,
                                  const float *thr, int gran, const float *cb, uint32_t S,
                                  uint32_t b, uint32_t *words, uint16_t *radius, uint32_t *out_idx,
                                  uint16_t *out_val, uint32_t *slab_off, uint32_t *tile_off,
                                  uint32_t cap, hqmq_status *st, cudaStream_t stream) {
    using namespace hqmq;
    const uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    const uint32_t n_slabs = (uint32_t)(B * H);
    const size_t smem = (size_t)H * S * sizeof(float4);
    DevStatus *ds = reinterpret_cast<DevStatus *>(st);
    const float4 *cb4 = reinterpret_cast<const float4 *>(cb);
#define HQMQ_APP(DT, GR)                                                                          \
    do {                                                                                          \
        auto kern = k_append<DT, GR>;                                                             \
        if (smem > 48 * 1024 &&                                                                   \
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != \
                cudaSuccess)                                                                      \
            return HQMQ_ERR_CUDA;                                                                 \
        kern<<<(unsigned)n_calls, APP_THREADS, smem, stream>>>(x, H, cps, n_slabs, thr, cb4, S, b, \
                                                               words, radius, out_idx, out_val,   \
                                                               slab_off, tile_off, cap, ds);      \
    } while (0)
    if (dtype == HQMQ_BF16) {
        if (gran == HQMQ_GRAN_CHUNK) HQMQ_APP(HQMQ_BF16, HQMQ_GRAN_CHUNK);
        else HQMQ_APP(HQMQ_BF16, HQMQ_GRAN_ELEMENT);
    } else {
        if (gran == HQMQ_GRAN_CHUNK) HQMQ_APP(HQMQ_F32, HQMQ_GRAN_CHUNK);
        else HQMQ_APP(HQMQ_F32, HQMQ_GRAN_ELEMENT);
    }
#undef HQMQ_APP
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}
