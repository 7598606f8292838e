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
// streams its chunks through a private cp.async ring in shared memory (4
// packing groups, 3 ahead; 16-byte copies that bypass L1).  The head's
// codeword table sits in shared memory in R copies (lane l reads copy
// l mod R; R = 8 makes the 8 lanes of a 16-byte phase hit distinct bank
// groups), R chosen so that the CTA's shared memory stays within 144 KB and
// the SM keeps 92 KB of L1, through which the random table records go: at
// S = 32 that is R = 4, and the larger L1 is worth more than conflict-free
// codeword loads.
//
// A chunk step is software-pipelined: the next chunk's face, cell and record
// load are issued before the current chunk's candidates are scored.  The
// Med3x bookkeeping per chunk is only the count below the window and the
// candidate bit; chunks inside the window or above t_lo (a few per cent) are
// queued per warp and handled a queue at a time.  Indices of a unit are
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
constexpr int RING_SLOTS = 4;                      // input ring per warp: packing groups
constexpr int SPEC_STAGE = 128;                    // window keys staged per warp
constexpr int EVQ = 64;                            // event queue entries per warp
// per-warp shared bytes: input ring, window-key stage, index stage, candidate
// bits, event queue (keys, then raw chunks of CB bytes)
__host__ __device__ constexpr int warp_smem(int CB) {
    return RING_SLOTS * 32 * CB + SPEC_STAGE * 4 + UNIT_G * 32 * 2 + UNIT_G * 4 + EVQ * (4 + CB);
}
static_assert(warp_smem(8) % 16 == 0 && warp_smem(16) % 16 == 0,
              "per-warp shared regions stay 16-byte aligned");
static_assert(TILE_GROUPS % UNIT_G == 0, "a unit lies inside one list tile");
constexpr size_t SPEC_SMEM_MAX = 227 * 1024;
// Shared memory of a CTA up to which more table copies are taken: the rest of
// the SM's 256 KB is L1 (the carve-out rounds shared memory up: 144 KB -> 164
// KB, L1 92 KB), which the table records go through; measured on B200, the
// kernel runs faster with that L1 than with conflict-free codeword loads.
constexpr size_t SPEC_SMEM_L1 = 144 * 1024;
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

// Cell of the gnomonic point (t1, t2, t3) on the 32^3 grid, without
// float-to-int conversions: each coordinate's grid position v in [0, 32) is
// floored by adding 2^23 with rounding toward zero, which leaves floor(v) in
// the low bits of the sum; the three sums are combined with integer
// multiply-adds and the exponent bits subtracted once.  The map's constants
// are scaled by (1 - 2^-20) and offset by 2^-17 so that t = 1 stays below 32
// and t = -1 above 0; the shift of a boundary is below 3.2e-6 in t, inside
// the 1e-5 by which every cell of the table is widened.  A non-finite t gives
// some in-range cell (the mask).
__device__ __forceinline__ uint32_t cell_of(float c1, float c2, float c3, float inv) {
    constexpr float SC = 1.0f - 1.0f / 1048576.0f;
    constexpr float HG = 0.5f * LUT_G;
    constexpr float PA = MAP_A * HG * SC, PB = MAP_B * HG * SC, P0 = HG * SC + 1.0f / 131072.0f;
    constexpr float MAGIC = 8388608.0f;                    // 2^23
    constexpr uint32_t EXP = 0x4B000000u;                  // bits of 2^23
    // t1 and t2 as one pair through the packed f32x2 operations (each lane of
    // a pair is the IEEE operation on its own: the same values as scalar code)
    uint32_t b1, b2;
    asm("{.reg .b64 t, u, p, q;\n\t"
        "mov.b64 t, {%2, %3};\n\t"
        "mov.b64 u, {%4, %4};\n\t"
        "mul.rn.f32x2 t, t, u;\n\t"                       // (t1, t2)
        "mul.rn.f32x2 u, t, t;\n\t"                       // squares
        "mov.b64 p, {%5, %5};\n\t"
        "mov.b64 q, {%6, %6};\n\t"
        "fma.rn.f32x2 u, p, u, q;\n\t"                    // PB t^2 + PA
        "mov.b64 p, {%7, %7};\n\t"
        "fma.rn.f32x2 t, t, u, p;\n\t"                    // t (PB t^2 + PA) + P0
        "mov.b64 p, {%8, %8};\n\t"
        "add.rz.f32x2 t, t, p;\n\t"
        "mov.b64 {%0, %1}, t;}"
        : "=r"(b1), "=r"(b2)
        : "f"(c1), "f"(c2), "f"(inv), "f"(PB), "f"(PA), "f"(P0), "f"(MAGIC));
    const float t3 = c3 * inv;
    const uint32_t b3 = __float_as_uint(__fadd_rz(__fmaf_rn(t3, __fmaf_rn(PB, t3 * t3, PA), P0), MAGIC));
    const uint32_t c = (b1 * (uint32_t)LUT_G + b2) * (uint32_t)LUT_G + b3;
    return (c - EXP * (uint32_t)(LUT_G * LUT_G + LUT_G + 1)) & (uint32_t)(LUT_CELLS - 1);
}

// What a chunk step carries from its front half to its back half.
template <int DT> struct StepState {
    RawChunk<DT> v;         // the chunk as read
    float r;                // its norm (0 for a certain outlier)
    uint4 rec;              // its cell's record (in flight until used)
};

// SPEC = false: the plain table encode (no Med3x): no window bookkeeping, no
// candidate bits or values, status counts straight to st.
template <int DT, int BB, int R, bool SPEC>
__global__ void __launch_bounds__(SPEC_THREADS, 1)
k_encode_spec(const void *__restrict__ x, int B, int H, uint32_t gps, uint32_t ups, uint32_t tps,
              uint32_t n_units, uint32_t round_units, const float4 *__restrict__ cb_all, uint32_t S,
              const uint4 *__restrict__ tables, uint32_t *__restrict__ words,
              uint16_t *__restrict__ radius, SpecArgs sa, DevStatus *st) {
    constexpr int CB = DT == HQMQ_BF16 ? 8 : 16;       // bytes per chunk
    pdl_wait();                                        // (launched with launch_pdl)
    pdl_trigger();
    constexpr int NS = RING_SLOTS;                     // ring slots (packing groups)
    constexpr int RING_BYTES = NS * 32 * CB;
    static_assert(NS >= 2 && UNIT_G % NS == 0, "a unit's groups fill whole ring rounds");
    extern __shared__ __align__(16) unsigned char s_raw[];
    float4 *s_tab = reinterpret_cast<float4 *>(s_raw); // [24 S + 1][R]
    const uint32_t n_words = 24u * S;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    unsigned char *wsm = s_raw + (size_t)(n_words + 1) * R * sizeof(float4) +
                         (size_t)warp * warp_smem(CB);
    uint32_t *stage = reinterpret_cast<uint32_t *>(wsm + RING_BYTES);
    uint16_t *s_idx = reinterpret_cast<uint16_t *>(wsm + RING_BYTES + SPEC_STAGE * 4);
    uint32_t *s_cb = reinterpret_cast<uint32_t *>(wsm + RING_BYTES + SPEC_STAGE * 4 + UNIT_G * 64);
    // event queue: chunks of the current unit inside the median window or above
    // t_lo, in chunk order (their keys and raw values)
    uint32_t *q_key = s_cb + UNIT_G;
    using Raw = typename RingWord<CB>::T;
    Raw *q_raw = reinterpret_cast<Raw *>(q_key + EVQ);
    // 32-bit shared addresses of this lane's ring chunk (slot 0), table copy,
    // index stage entry (group 0) and the warp's candidate-bit words
    const uint32_t a_ring = (uint32_t)__cvta_generic_to_shared(wsm) + (uint32_t)lane * CB;
    const uint32_t a_tab = (uint32_t)__cvta_generic_to_shared(s_tab) + (uint32_t)(lane & (R - 1)) * 16u;
    const uint32_t a_idx = (uint32_t)__cvta_generic_to_shared(s_idx) + (uint32_t)lane * 2u;
    const uint32_t a_cb = (uint32_t)__cvta_generic_to_shared(s_cb);
    const unsigned char *xl = reinterpret_cast<const unsigned char *>(x) + (size_t)lane * CB;
    // Copies packing group G into ring slot `slot`: 16-byte copies that bypass
    // L1 (bf16: lanes 0..15 copy two chunks each), so that x does not take L1
    // space from the table records.
    const uint32_t a_ring0 = (uint32_t)__cvta_generic_to_shared(wsm);
    auto ring_copy = [&](uint32_t slot, uint32_t G) {
        if constexpr (CB == 8) {
            if (lane < 16)
                cp_async_chunk<16>(a_ring0 + slot * 256u + (uint32_t)lane * 16u,
                                   reinterpret_cast<const unsigned char *>(x) + (size_t)G * 256u + lane * 16u);
        } else {
            cp_async_chunk<16>(a_ring + slot * 32u * CB, xl + (size_t)G * (32u * CB));
        }
    };

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
                    ring_copy(i, Gb + i);
                cp_async_commit();
            }
            uint32_t n_stage = 0, n_below = 0, n_nf = 0, n_sat = 0;
            for (uint32_t u = ua; u < ub; ++u) {
                const uint32_t g0 = (u - u_slab) * UNIT_G;
                const uint32_t ng = min((uint32_t)UNIT_G, gps - g0);
                const uint32_t Gu = g_slab + g0;
                const uint32_t tile = slab * tps + g0 / TILE_GROUPS;
                uint32_t n_def = 0, fbm = 0, n_cv = 0, n_q = 0;
                unsigned char *cv_u = sa.cvals + (size_t)(slab * ups + (u - u_slab)) * (CVAL_SLOTS * CB);
                // The queued events of this unit, in chunk order: window keys to the
                // stage (flushed to the head's key list when full), the raw values
                // of the unit's first CVAL_SLOTS candidates (r > t_lo), the count of
                // certain outliers (r > t_hi) for the unit's list tile, and the
                // (tile, key) pairs of the band t_lo < r <= t_hi.  Warp-collective.
                auto events = [&]() {
                    __syncwarp();                            // (the lanes' queue writes)
                    for (uint32_t e0 = 0; e0 < n_q; e0 += 32) {
                        const uint32_t e = e0 + (uint32_t)lane;
                        const bool valid = e < n_q;
                        const uint32_t key = valid ? q_key[e] : 0u;
                        const float r = __uint_as_float(key);
                        const bool in = valid && key - w.lo_key < span;
                        const bool cnd = valid && r > w.t_lo;
                        const bool dfn = valid && r > w.t_hi;
                        const uint32_t mi = __ballot_sync(FULL, in);
                        if (mi) {
                            if (n_stage > (uint32_t)SPEC_STAGE - 32u) {
                                flush_stage(stage, n_stage, lane, sa.cand_n + h,
                                            sa.cand + (uint64_t)h * sa.cand_cap, sa.cand_cap,
                                            sa.med_hist + (size_t)h * MED_BINS * 2, w.lo_key, top);
                                n_stage = 0;
                            }
                            if (in) stage[n_stage + __popc(mi & lt)] = key;
                            n_stage += __popc(mi);
                        }
                        const uint32_t mc = __ballot_sync(FULL, cnd);
                        const uint32_t pos = n_cv + __popc(mc & lt);
                        if (cnd && pos < (uint32_t)CVAL_SLOTS)
                            *reinterpret_cast<Raw *>(cv_u + pos * CB) = q_raw[e];
                        n_cv += __popc(mc);
                        n_def += dfn ? 1u : 0u;
                        if (cnd && !dfn) {                   // (rare) inside the band
                            const unsigned long long p = atomicAdd(sa.amb_n, 1ull);
                            if (p < sa.amb_cap) sa.amb[p] = make_uint2(tile, key);
                        }
                    }
                    __syncwarp();                            // (the queue is refilled next)
                    n_q = 0;
                };
                // One chunk step is split in two: front(k) reads the chunk, does the
                // Med3x bookkeeping, finds its face and cell and issues the load of
                // the cell's record; back(k) scores the candidates and stores the
                // codes.  front(k + 1) runs before back(k), so that the record's L2
                // latency overlaps the scoring of the previous step.
                auto front = [&](const uint32_t k) -> StepState<DT> {
                    const uint32_t G = Gu + k;
                    // group G's copy was the (NS-1)-th latest commit: wait for it
                    cp_async_wait<NS - 2>();
                    if constexpr (CB == 8) __syncwarp();     // (lanes read chunks another lane copied)
                    RawChunk<DT> cur;
                    if constexpr (CB == 8) cur.v = lds_u2(a_ring + (k % NS) * 32u * CB);
                    else cur.v = lds_f4_ring(a_ring + (k % NS) * 32u * CB);
                    // refill the slot read in the previous step (this lane's bytes only)
                    if (G + (NS - 1) < Ge)
                        ring_copy((k + NS - 1) % NS, G + (NS - 1));
                    cp_async_commit();
                    const float x0 = cur.e(0), x1 = cur.e(1), x2 = cur.e(2), x3 = cur.e(3);
                    float r = chunk_norm(x0, x1, x2, x3);
                    // median window: key = r's bits (r >= 0; a NaN's bits exceed
                    // every finite key and +inf's, as in the median's order)
                    const uint32_t key = __float_as_uint(r);
                    if constexpr (SPEC) {
                    // Per chunk only what every chunk needs: the count below the
                    // window and the candidate bit.  Chunks inside the window or
                    // above t_lo (a few per cent) go to the event queue, handled
                    // a queue at a time by events().
                    n_below += key < w.lo_key ? 1u : 0u;
                    const bool in = key - w.lo_key < span;   // lo_key <= key < hi_key
                    const bool cnd = r > w.t_lo;             // (NaN: false)
                    const uint32_t mc = __ballot_sync(FULL, cnd);
                    if (lane == 0) sts_u32(a_cb + k * 4u, mc);
                    const uint32_t me = __ballot_sync(FULL, in || cnd);
                    if (n_q > (uint32_t)(EVQ - 32)) events();   // (warp-uniform) make room
                    if (in || cnd) {
                        const uint32_t q = n_q + __popc(me & lt);
                        q_key[q] = key;
                        q_raw[q] = cur.v;
                    }
                    n_q += __popc(me);
                    }
                    // search every lane (branch-free); a lane whose chunk is zero,
                    // non-finite or a certain outlier reads some in-range record and
                    // keeps index 0.  r in (0, FLT_MAX] <=> its bits in [1, 0x7F7FFFFF].
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
                    const uint32_t cell = cell_of(c1, c2, c3, inv);
                    const uint32_t face = 2u * a + (xa < 0.0f ? 1u : 0u);
                    StepState<DT> o;
                    o.v = cur;
                    o.r = r;
                    o.rec = __ldg(tb + (face * LUT_CELLS + cell));
                    return o;
                };
                auto back = [&](const uint32_t k, const StepState<DT> &c) {
                    const uint32_t G = Gu + k;
                    const float x0 = c.v.e(0), x1 = c.v.e(1), x2 = c.v.e(2), x3 = c.v.e(3);
                    // a certain outlier (r > t_hi) is encoded as index 0, radius 0
                    const bool cnd = SPEC && c.r > w.t_lo;
                    const float r = SPEC && c.r > w.t_hi ? 0.0f : c.r;
                    const uint4 rec = c.rec;
                    const bool srch = __float_as_uint(r) - 1u < 0x7F7FFFFFu;
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
                    StepState<DT> cs = front(0);
    #pragma unroll kSpecUnroll
                    for (uint32_t k = 0; k < UNIT_G - 1; ++k) {
                        const StepState<DT> ns = front(k + 1);
                        back(k, cs);
                        cs = ns;
                    }
                    back(UNIT_G - 1, cs);
                } else {
                    for (uint32_t k = 0; k < ng; ++k) back(k, front(k));
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
                    if (n_q) events();
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
    constexpr int CB = DT == HQMQ_BF16 ? 8 : 16;
    const size_t smem = ((size_t)24 * S + 1) * R * sizeof(float4) + (size_t)SPEC_WARPS * warp_smem(CB);
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
    if (launch_pdl(kern, dim3((unsigned)ctas), dim3(SPEC_THREADS), smem, stream, x, B, H, gps, ups,
                   tps, (uint32_t)n_units, (uint32_t)round_units,
                   reinterpret_cast<const float4 *>(cb), S, reinterpret_cast<const uint4 *>(table),
                   words, radius, sa, st) != cudaSuccess)
        return HQMQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

template <int DT, int BB, bool SPEC>
static int launch_spec_r(int B, int H, int T, int D, const void *x, const float *cb, uint32_t S,
                         const void *table, uint32_t *words, uint16_t *radius, const SpecArgs &sa,
                         DevStatus *st, int sm_count, cudaStream_t stream) {
    // 8 table copies when they fit next to the warps' regions, else 4
    // as many table copies (8, 4 or 2) as keep the CTA's shared memory within
    // SPEC_SMEM_L1, so that the SM keeps that much L1 for the table records
    constexpr int CB = DT == HQMQ_BF16 ? 8 : 16;
    const size_t warps = (size_t)SPEC_WARPS * warp_smem(CB);
    const size_t copy = ((size_t)24 * S + 1) * sizeof(float4);
    if (8 * copy + warps <= SPEC_SMEM_L1)
        return launch_spec<DT, BB, 8, SPEC>(B, H, T, D, x, cb, S, table, words, radius, sa, st,
                                            sm_count, stream);
    if (4 * copy + warps <= SPEC_SMEM_L1)
        return launch_spec<DT, BB, 4, SPEC>(B, H, T, D, x, cb, S, table, words, radius, sa, st,
                                            sm_count, stream);
    return launch_spec<DT, BB, 2, SPEC>(B, H, T, D, x, cb, S, table, words, radius, sa, st,
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
