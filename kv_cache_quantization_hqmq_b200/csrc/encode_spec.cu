// encode_spec.cu -- the one-read Med3x encode pass (chunk mode, search tables).
//
// Med3x needs the exact median of a head's chunk norms before any chunk can
// be called an outlier (gist.science/nl, Technische Samenvatting, section 3),
// but the encode of a chunk does not depend on the median unless the chunk
// is an outlier.  This pass therefore reads x once and, per chunk:
//  * does the window bookkeeping of the median (keys below the sampled rank
//    window counted per head, keys inside it staged for the exact selection,
//    per 1024-chunk tile the count of chunks above every possible threshold
//    t_hi, and (tile, key) pairs of chunks inside the threshold's band
//    (t_lo, t_hi]);
//  * records per packing group which chunks lie above t_lo (the only ones
//    that can be outliers), for the fix-up pass after the exact threshold;
//  * encodes speculatively: a chunk above t_hi as an outlier (index 0,
//    radius 0), every other chunk as a bulk chunk: fp16 radius and the index
//    of the nearest of the 24 S codewords q_p q_s (section 1), found through
//    the per-face search table (search.cuh).
//
// Data flow (B200): one CTA of 32 warps per SM.  The call's work units (8
// packing groups, 256 chunks) are taken head by head (all batches of head 0,
// then head 1, ...) in rounds of up to 8 heads' units; every round is split
// into contiguous unit ranges over the CTAs, so that at any time the GPU
// works on at most 8 heads, whose search tables stay in L2.  Inside a slab's
// share of a range every warp takes a contiguous share of the units.  Each warp
// streams its chunks through a private cp.async ring in shared memory
// (7 groups = 1.75 KB ahead per warp, ~56 KB in flight per SM), so that HBM
// latency is hidden without registers; the head's codeword table sits in
// shared memory in R copies (lane l reads copy l mod R: the 8 lanes of a
// 16-byte phase hit distinct bank groups for R = 8).  Indices of a unit are
// staged in shared memory and packed into the unit's b-bit words with
// coalesced stores.
//
// The outputs equal those of k_encode_lut's speculative mode (search.cu) bit
// for bit; the per-tile counts are added atomically because a tile's four
// units may belong to different warps.
#include "search.cuh"

namespace hqmq {

constexpr int SPEC_THREADS = 1024;
constexpr int SPEC_WARPS = SPEC_THREADS / 32;
constexpr int UNIT_G = 8;                          // packing groups per work unit
constexpr int RING_BYTES = 2048;                   // input ring per warp
constexpr int SPEC_STAGE = 128;                    // window keys staged per warp
constexpr int WARP_SMEM = RING_BYTES + SPEC_STAGE * 4 + UNIT_G * 32 * 2 + UNIT_G * 4;
static_assert(WARP_SMEM % 16 == 0, "per-warp shared regions stay 16-byte aligned");
static_assert(TILE_GROUPS % UNIT_G == 0, "a unit lies inside one list tile");
constexpr size_t SPEC_SMEM_MAX = 227 * 1024;
constexpr int SPEC_ROUND_HEADS = 8;               // heads per round of the walk
// Steps of a unit unrolled per loop trip: 2 measured fastest on B200 (4 and 8
// run slower: the body no longer stays in the instruction cache).
constexpr int kSpecUnroll = 2;

template <int CB>
__device__ __forceinline__ void cp_async_chunk(uint32_t dst, const void *src) {
    if constexpr (CB == 8)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(dst), "l"(src) : "memory");
    else
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// <x, c> in fp32 (the order of the table encode)
__device__ __forceinline__ float score4(float x0, float x1, float x2, float x3, float4 c) {
    return __fmaf_rn(x3, c.w, __fmaf_rn(x2, c.z, __fmaf_rn(x1, c.y, __fmul_rn(x0, c.x))));
}

// Shared-memory accesses of the hot loop, by 32-bit shared address.
template <int CB> struct RingWord;
template <> struct RingWord<8> { using T = uint2; };
template <> struct RingWord<16> { using T = float4; };
__device__ __forceinline__ uint2 lds_u2(uint32_t a) {       // (ordered after cp.async waits)
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float4 lds_f4_ring(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float4 lds_cw(uint32_t a) {     // codeword table (read-only here)
    float4 v;
    asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
        : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts_u16(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"((unsigned short)v) : "memory");
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// SPEC = false: the plain table encode (no Med3x): no window bookkeeping, no
// candidate bits or values, status counts straight to st.
template <int DT, int BB, int R, bool SPEC>
__global__ void __launch_bounds__(SPEC_THREADS, 1)
k_encode_spec(const void *__restrict__ x, int B, int H, uint32_t gps, uint32_t ups, uint32_t tps,
              uint32_t n_units, uint32_t round_units, const float4 *__restrict__ cb_all, uint32_t S,
              const uint4 *__restrict__ tables, uint32_t *__restrict__ words,
              uint16_t *__restrict__ radius, SpecArgs sa, DevStatus *st) {
    constexpr int CB = DT == HQMQ_BF16 ? 8 : 16;       // bytes per chunk
    constexpr int NS = RING_BYTES / (32 * CB);         // ring slots (packing groups)
    static_assert(NS >= 2 && UNIT_G % NS == 0, "a unit's groups fill whole ring rounds");
    extern __shared__ __align__(16) unsigned char s_raw[];
    float4 *s_tab = reinterpret_cast<float4 *>(s_raw); // [24 S + 1][R]
    const uint32_t n_words = 24u * S;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    unsigned char *wsm = s_raw + (size_t)(n_words + 1) * R * sizeof(float4) +
                         (size_t)warp * WARP_SMEM;
    uint32_t *stage = reinterpret_cast<uint32_t *>(wsm + RING_BYTES);
    uint16_t *s_idx = reinterpret_cast<uint16_t *>(wsm + RING_BYTES + SPEC_STAGE * 4);
    uint32_t *s_cb = reinterpret_cast<uint32_t *>(wsm + RING_BYTES + SPEC_STAGE * 4 + UNIT_G * 64);
    // 32-bit shared addresses of this lane's ring chunk (slot 0), table copy,
    // index stage entry (group 0) and the warp's candidate-bit words
    const uint32_t a_ring = (uint32_t)__cvta_generic_to_shared(wsm) + (uint32_t)lane * CB;
    const uint32_t a_tab = (uint32_t)__cvta_generic_to_shared(s_tab) + (uint32_t)(lane & (R - 1)) * 16u;
    const uint32_t a_idx = (uint32_t)__cvta_generic_to_shared(s_idx) + (uint32_t)lane * 2u;
    const uint32_t a_cb = (uint32_t)__cvta_generic_to_shared(s_cb);
    const unsigned char *xl = reinterpret_cast<const unsigned char *>(x) + (size_t)lane * CB;

    int cur_h = -1;
    // rounds of round_units units (a few heads' worth), each split into
    // contiguous ranges over the CTAs: all CTAs work on the same few heads
    for (uint32_t r0 = 0; r0 < n_units; r0 += round_units) {
        const uint32_t nr = min(round_units, n_units - r0);
        const uint32_t u_begin = r0 + (uint32_t)((uint64_t)nr * blockIdx.x / gridDim.x);
        const uint32_t u_end = r0 + (uint32_t)((uint64_t)nr * (blockIdx.x + 1) / gridDim.x);
        for (uint32_t seg = u_begin; seg < u_end;) {
            // slabs are walked head by head (all batches of a head, then the
            // next head), so that few heads' search tables are in use at a time
            const uint32_t vs = seg / ups;                  // slab in head-major order
            const uint32_t seg_end = min(u_end, (vs + 1) * ups);
            const int h = (int)(vs / (uint32_t)B);
            const uint32_t slab = (vs % (uint32_t)B) * (uint32_t)H + (uint32_t)h;
            if (h != cur_h) {                                // (block-uniform)
                __syncthreads();
                const float4 *cbh = cb_all + (size_t)h * S;
                for (uint32_t i = threadIdx.x; i < (n_words + 1) * R; i += SPEC_THREADS) {
                    const uint32_t id = i / R;
                    s_tab[i] = id < n_words ? codeword((int)(id % 24u), __ldg(cbh + id / 24u))
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                __syncthreads();
                cur_h = h;
            }
            // this warp's share of the head's units: [ua, ub)
            const uint32_t nseg = seg_end - seg;
            const uint32_t ua = seg + (uint32_t)((uint64_t)nseg * warp / SPEC_WARPS);
            const uint32_t ub = seg + (uint32_t)((uint64_t)nseg * (warp + 1) / SPEC_WARPS);
            seg = seg_end;
            if (ua >= ub) continue;                          // (warp-uniform)
            WinState w{};
            if constexpr (SPEC) w = sa.win[h];
            const uint32_t span = w.hi_key - w.lo_key;
            const int top = SPEC ? median_top_shift(span) : 0;
            const uint4 *tb = tables + (size_t)h * LUT_ENTRIES;
            const float4 *cb = cb_all + (size_t)h * S;
            // packing groups of the call (fewer than 2^27: 32-bit indices)
            const uint32_t u_slab = vs * ups;               // (unit numbering of the walk)
            const uint32_t g_slab = slab * gps;
            const uint32_t Gb = g_slab + (ua - u_slab) * UNIT_G;
            const uint32_t Ge = g_slab + min((ub - u_slab) * UNIT_G, gps);
            // ring: group Gb + i sits in slot i mod NS (a unit's groups fill whole
            // rounds of the ring); prologue: groups Gb .. Gb + NS - 2
    #pragma unroll
            for (int i = 0; i < NS - 1; ++i) {
                if (Gb + i < Ge)
                    cp_async_chunk<CB>(a_ring + (uint32_t)i * 32u * CB, xl + (size_t)(Gb + i) * (32u * CB));
                cp_async_commit();
            }
            uint32_t n_stage = 0, n_below = 0, n_nf = 0, n_sat = 0;
            for (uint32_t u = ua; u < ub; ++u) {
                const uint32_t g0 = (u - u_slab) * UNIT_G;
                const uint32_t ng = min((uint32_t)UNIT_G, gps - g0);
                const uint32_t Gu = g_slab + g0;
                const uint32_t tile = slab * tps + g0 / TILE_GROUPS;
                uint32_t n_def = 0, fbm = 0, n_cv = 0;
                unsigned char *cv_u = sa.cvals + (size_t)(slab * ups + (u - u_slab)) * (CVAL_SLOTS * CB);
                auto step = [&](const uint32_t k) {
                    const uint32_t G = Gu + k;
                    // group G's copy was the (NS-1)-th latest commit: wait for it
                    cp_async_wait<NS - 2>();
                    RawChunk<DT> cur;
                    if constexpr (CB == 8) cur.v = lds_u2(a_ring + (k % NS) * 32u * CB);
                    else cur.v = lds_f4_ring(a_ring + (k % NS) * 32u * CB);
                    // refill the slot read in the previous step (this lane's bytes only)
                    if (G + (NS - 1) < Ge)
                        cp_async_chunk<CB>(a_ring + ((k + NS - 1) % NS) * 32u * CB,
                                           xl + (size_t)(G + (NS - 1)) * (32u * CB));
                    cp_async_commit();
                    const float x0 = cur.e(0), x1 = cur.e(1), x2 = cur.e(2), x3 = cur.e(3);
                    float r = chunk_norm(x0, x1, x2, x3);
                    // median window: key = r's bits (r >= 0; a NaN's bits exceed
                    // every finite key and +inf's, as in the median's order)
                    const uint32_t key = __float_as_uint(r);
                    bool cnd = false;
                    if constexpr (SPEC) {
                    n_below += key < w.lo_key ? 1u : 0u;
                    const bool in = key - w.lo_key < span;   // lo_key <= key < hi_key
                    const uint32_t mi = __ballot_sync(FULL, in);
                    if (mi) {
                        if (n_stage + 32 > SPEC_STAGE) {
                            flush_stage(stage, n_stage, lane, sa.cand_n + h,
                                        sa.cand + (uint64_t)h * sa.cand_cap, sa.cand_cap,
                                        sa.med_hist + (size_t)h * MED_BINS * 2, w.lo_key, top);
                            n_stage = 0;
                        }
                        if (in) stage[n_stage + __popc(mi & lt)] = key;
                        n_stage += __popc(mi);
                        __syncwarp();
                    }
                    // threshold band: above t_hi always an outlier, above t_lo possibly
                    const bool dfn = r > w.t_hi;             // (NaN: false)
                    cnd = r > w.t_lo;
                    n_def += dfn ? 1u : 0u;
                    const uint32_t mc = __ballot_sync(FULL, cnd);
                    if (lane == 0) sts_u32(a_cb + k * 4u, mc);
                    {   // the raw value of a possible outlier, for the fix-up pass
                        const uint32_t pos = n_cv + __popc(mc & lt);
                        if (cnd && pos < (uint32_t)CVAL_SLOTS)
                            *reinterpret_cast<decltype(cur.v) *>(cv_u + pos * CB) = cur.v;
                        n_cv += __popc(mc);
                    }
                    const uint32_t mu = __ballot_sync(FULL, cnd && !dfn);
                    if (mu) {
                        unsigned long long base = 0;
                        if (lane == 0) base = atomicAdd(sa.amb_n, (unsigned long long)__popc(mu));
                        base = __shfl_sync(FULL, base, 0);
                        if ((mu >> lane) & 1u) {
                            const unsigned long long pos = base + __popc(mu & lt);
                            if (pos < sa.amb_cap) sa.amb[pos] = make_uint2(tile, key);
                        }
                    }
                    if (dfn) r = 0.0f;                       // certain outlier: radius 0, index 0
                    }
                    // search every lane (branch-free); a lane whose chunk is zero,
                    // non-finite or a certain outlier reads some in-range record and
                    // keeps index 0.  r in (0, FLT_MAX] <=> its bits in [1, 0x7F7FFFFF].
                    const bool srch = __float_as_uint(r) - 1u < 0x7F7FFFFFu;
                    const float a0 = fabsf(x0), a1 = fabsf(x1), a2 = fabsf(x2), a3 = fabsf(x3);
                    const float m = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
                    const bool e0 = a0 == m, e01 = e0 || a1 == m, e012 = e01 || a2 == m;
                    const uint32_t a = e0 ? 0u : e01 ? 1u : e012 ? 2u : 3u;
                    const float xa = e0 ? x0 : e01 ? x1 : e012 ? x2 : x3;
                    const float c1 = e0 ? x1 : x0;
                    const float c2 = e01 ? x2 : x1;
                    const float c3 = e012 ? x3 : x2;
                    float inv;
                    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(m));   // cells are widened
                    const uint32_t cell = (uint32_t)((cell_coord(c1 * inv) * LUT_G + cell_coord(c2 * inv)) *
                                                         LUT_G + cell_coord(c3 * inv)) & (LUT_CELLS - 1u);
                    const uint32_t face = 2u * a + (xa < 0.0f ? 1u : 0u);
                    const uint4 rec = __ldg(tb + (face * LUT_CELLS + cell));
                    const uint32_t cnt = (rec.x >> 12) & 0xFu;          // 0: overflowing cell
                    const uint32_t kmax = __reduce_max_sync(FULL, cnt);
                    // the slots hold increasing ids (padded with the zero codeword
                    // 24 S); scored from the last to the first, a candidate that
                    // scores at least the best so far replaces it, so among equal
                    // scores the lowest index wins.  Only the warp's longest list
                    // is walked (straight-line code entered at slot kmax - 1).
                    float best = __int_as_float(0xFF800000);
                    uint32_t bid = 0;
    #define HQMQ_CAND(EXPR)                                                              \
        {                                                                                \
            const uint32_t id_ = (EXPR);                                                 \
            const float sc_ = score4(x0, x1, x2, x3, lds_cw(a_tab + id_ * (16u * R)));   \
            if (sc_ >= best) { best = sc_; bid = id_; }                                  \
        }
                    switch (kmax) {
                        default:
                        case 8: HQMQ_CAND(rec.w >> 16)
                        case 7: HQMQ_CAND(rec.w & 0xFFFFu)
                        case 6: HQMQ_CAND(rec.z >> 16)
                        case 5: HQMQ_CAND(rec.z & 0xFFFFu)
                        case 4: HQMQ_CAND(rec.y >> 16)
                        case 3: HQMQ_CAND(rec.y & 0xFFFFu)
                        case 2: HQMQ_CAND(rec.x >> 16)
                        case 1:
                        case 0: HQMQ_CAND(rec.x & LUT_ID_MASK)
                    }
    #undef HQMQ_CAND
                    const uint32_t idx = srch ? bid : 0u;
                    fbm |= (srch && cnt == 0u ? 1u : 0u) << k;   // overflowing cell: S-codeword loop later
                    // fp16 radius: RN-even, saturating at 65504 from 65520 up;
                    // NaN or inf -> 0x7E00 (counted)
                    const bool fin = r <= 3.40282347e38f;
                    const bool sat = fin && r >= 65520.0f;
                    uint16_t rh = __half_as_ushort(__float2half_rn(r));
                    rh = sat ? (uint16_t)0x7BFFu : rh;
                    rh = fin ? rh : (uint16_t)0x7E00u;
                    n_nf += fin ? 0u : 1u;
                    n_sat += (sat && !cnd) ? 1u : 0u;        // (the fix-up pass decides the others)
                    radius[G * 32u + (uint32_t)lane] = rh;
                    sts_u16(a_idx + k * 64u, idx);
                };
                if (ng == UNIT_G) {
    #pragma unroll kSpecUnroll
                    for (uint32_t k = 0; k < UNIT_G; ++k) step(k);
                } else {
                    for (uint32_t k = 0; k < ng; ++k) step(k);
                }
                if (__any_sync(FULL, fbm != 0u)) {          // (rare) overflowing cells
                    for (uint32_t k = 0; k < ng; ++k) {
                        if (!((fbm >> k) & 1u)) continue;
                        RawChunk<DT> v;
                        v.load(x, (size_t)(Gu + k) * 32u + (uint32_t)lane);
                        s_idx[k * 32 + lane] =
                            (uint16_t)sloop_index(v.e(0), v.e(1), v.e(2), v.e(3), cb, S);
                    }
                }
                __syncwarp();
                pack_tile<BB>(s_idx, ng, lane, words + (size_t)Gu * BB);
                if constexpr (SPEC) {
                    if ((uint32_t)lane < ng) sa.cbits[Gu + lane] = s_cb[lane];
                    n_def = __reduce_add_sync(FULL, n_def);
                    if (lane == 0 && n_def) atomicAdd(sa.tile_cnt + tile, n_def);
                }
                __syncwarp();                                // (s_idx, s_cb are refilled next unit)
            }
            if constexpr (SPEC) {
            n_below = __reduce_add_sync(FULL, n_below);
            if (lane == 0 && n_below) atomicAdd(sa.below + h, (unsigned long long)n_below);
            if (n_stage)
                flush_stage(stage, n_stage, lane, sa.cand_n + h, sa.cand + (uint64_t)h * sa.cand_cap,
                            sa.cand_cap, sa.med_hist + (size_t)h * MED_BINS * 2, w.lo_key, top);
            }
            const unsigned nf = __reduce_add_sync(FULL, n_nf);
            const unsigned ns = __reduce_add_sync(FULL, n_sat);
            if (lane == 0 && (nf | ns)) {
                if constexpr (SPEC) {
                    atomicAdd(sa.head_stat + 2 * h, (unsigned long long)nf);
                    atomicAdd(sa.head_stat + 2 * h + 1, (unsigned long long)ns);
                } else if (st) {
                    if (nf) status_add(st, HQMQ_FLAG_NONFINITE, &st->n_nonfinite, nf);
                    if (ns) status_add(st, HQMQ_FLAG_SATURATED, &st->n_saturated, ns);
                }
            }
        }
    }
}

template <int DT, int BB, int R, bool SPEC>
static int launch_spec(int B, int H, int T, int D, const void *x, const float *cb, uint32_t S,
                       const void *table, uint32_t *words, uint16_t *radius, const SpecArgs &sa,
                       DevStatus *st, int sm_count, cudaStream_t stream) {
    const uint32_t gps = (uint32_t)(((uint64_t)T * D / 4) / 32);
    const uint32_t ups = (gps + UNIT_G - 1) / UNIT_G;
    const uint32_t tps = (gps + TILE_GROUPS - 1) / TILE_GROUPS;
    const uint64_t n_units = (uint64_t)B * H * ups;
    const size_t smem = ((size_t)24 * S + 1) * R * sizeof(float4) + (size_t)SPEC_WARPS * WARP_SMEM;
    if (smem > SPEC_SMEM_MAX) return HQMQ_ERR_ARG;
    auto kern = k_encode_spec<DT, BB, R, SPEC>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return HQMQ_ERR_CUDA;
    uint64_t ctas = (uint64_t)sm_count;                  // one CTA per SM
    if (ctas > n_units) ctas = n_units;
    if (ctas < 1) ctas = 1;
    // a round covers at most SPEC_ROUND_HEADS heads (their tables, 4 MB each,
    // stay in L2 while x streams through) and at least a unit per warp
    uint64_t round_units = (uint64_t)SPEC_ROUND_HEADS * B * ups;
    if (round_units < ctas * SPEC_WARPS) round_units = ctas * SPEC_WARPS;
    if (round_units > n_units) round_units = n_units;
    kern<<<(unsigned)ctas, SPEC_THREADS, smem, stream>>>(
        x, B, H, gps, ups, tps, (uint32_t)n_units, (uint32_t)round_units,
        reinterpret_cast<const float4 *>(cb), S,
        reinterpret_cast<const uint4 *>(table), words, radius, sa, st);
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

template <int DT, int BB, bool SPEC>
static int launch_spec_r(int B, int H, int T, int D, const void *x, const float *cb, uint32_t S,
                         const void *table, uint32_t *words, uint16_t *radius, const SpecArgs &sa,
                         DevStatus *st, int sm_count, cudaStream_t stream) {
    // 8 table copies when they fit next to the warps' regions, else 4
    const size_t smem8 = ((size_t)24 * S + 1) * 8 * sizeof(float4) + (size_t)SPEC_WARPS * WARP_SMEM;
    if (smem8 <= SPEC_SMEM_MAX)
        return launch_spec<DT, BB, 8, SPEC>(B, H, T, D, x, cb, S, table, words, radius, sa, st,
                                            sm_count, stream);
    return launch_spec<DT, BB, 4, SPEC>(B, H, T, D, x, cb, S, table, words, radius, sa, st,
                                        sm_count, stream);
}

template <bool SPEC>
static int launch_spec_dt(int dtype, uint32_t b, int B, int H, int T, int D, const void *x,
                          const float *cb, uint32_t S, const void *table, uint32_t *words,
                          uint16_t *radius, const SpecArgs &sa, DevStatus *st, int sm_count,
                          cudaStream_t stream) {
    if (dtype == HQMQ_BF16) {
        if (b == 8)
            return launch_spec_r<HQMQ_BF16, 8, SPEC>(B, H, T, D, x, cb, S, table, words, radius,
                                                     sa, st, sm_count, stream);
        if (b == 10)
            return launch_spec_r<HQMQ_BF16, 10, SPEC>(B, H, T, D, x, cb, S, table, words, radius,
                                                      sa, st, sm_count, stream);
    } else {
        if (b == 8)
            return launch_spec_r<HQMQ_F32, 8, SPEC>(B, H, T, D, x, cb, S, table, words, radius,
                                                    sa, st, sm_count, stream);
        if (b == 10)
            return launch_spec_r<HQMQ_F32, 10, SPEC>(B, H, T, D, x, cb, S, table, words, radius,
                                                     sa, st, sm_count, stream);
    }
    return HQMQ_ERR_ARG;
}

}  // namespace hqmq

// True when the unit kernels of this file cover this index width (b = 8:
// S = 8..10; b = 10: S = 22..42).
extern "C" int hqmq_spec_encode_supported(uint32_t b) { return b == 8 || b == 10; }

// The one-read Med3x encode pass (speculative, chunk mode).
extern "C" int hqmq_launch_spec_encode_units(const void *x, int dtype, int B, int H, int T, int D,
                                             const float *cb, uint32_t S, uint32_t b,
                                             const void *table, uint32_t *words, uint16_t *radius,
                                             void *ws, int sm_count, cudaStream_t stream) {
    using namespace hqmq;
    const SpecArgs sa = spec_args(reinterpret_cast<char *>(ws),
                                  fused_layout(B, H, T, D, HQMQ_GRAN_CHUNK));
    return launch_spec_dt<true>(dtype, b, B, H, T, D, x, cb, S, table, words, radius, sa, nullptr,
                                sm_count, stream);
}

// The plain table encode (no Med3x threshold) with the same data flow.
extern "C" int hqmq_launch_table_encode_units(const void *x, int dtype, int B, int H, int T, int D,
                                              const float *cb, uint32_t S, uint32_t b,
                                              const void *table, uint32_t *words,
                                              uint16_t *radius, hqmq_status *st, int sm_count,
                                              cudaStream_t stream) {
    using namespace hqmq;
    return launch_spec_dt<false>(dtype, b, B, H, T, D, x, cb, S, table, words, radius, SpecArgs{},
                                 reinterpret_cast<DevStatus *>(st), sm_count, stream);
}
