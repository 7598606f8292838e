// search.cuh -- constants and device helpers of the table-driven HQMQ encode
// (search.cu: the per-face search table, the table encode and the Med3x
// list fix-up; encode_spec.cu: the one-read speculative encode).
//
// Faces and cells: a chunk x lies on the cube face of its first coordinate
// of largest magnitude (and that coordinate's sign); the other three
// coordinates in index order, divided by that magnitude, are its gnomonic
// coordinates t in [-1, 1]^3, cut into LUT_G^3 cells after the monotone map
// u(t) = t (A + B t^2).  Each cell's record lists the codewords that can be
// the argmax of <x, c> anywhere in the cell (gist.science/nl, Technische
// Samenvatting, section 1: the nearest of the 24 S products q_p q_s).
#pragma once

#include "med3_window.cuh"

namespace hqmq {

constexpr int LUT_G = 32;
constexpr int LUT_CELLS = LUT_G * LUT_G * LUT_G;   // 32768 cells per face
constexpr int LUT_FACES = 8;
constexpr int LUT_ENTRIES = LUT_FACES * LUT_CELLS;  // 4 MB per group
constexpr float MAP_A = 1.27323954f;               // 4 / pi (fp32)
constexpr float MAP_B = 1.0f - MAP_A;              // exact (Sterbenz)
constexpr int LUT_SLOTS = 8;
// Record: 8 slots of 16 bits; slot k holds candidate id k in its low 12 bits
// (24 S < 4096), in increasing order; the top 4 bits of slot 0 hold the count
// (1..8), 0 marks an overflowing cell; slots past the count hold the dummy id
// 24 S, whose shared-memory codeword is zero (score 0, below every real best
// score, and last in slot order).
constexpr uint32_t LUT_ID_MASK = 0x0FFFu;
constexpr uint32_t LUT_MAX_S = 48;                // 24 S codeword ids fit in 16 bits;
                                                  // shared memory fits 8 copies (144 KB)
constexpr double LUT_DELTA = 1e-5;                // cell growth in t (fp32 error ~1e-7)
constexpr int BUILD_THREADS = 128;
constexpr int BUILD_MAXC = 64;                     // candidates kept before pruning
constexpr int ENC_THREADS = 1024;

// ---------------------------------------------------------------------------
// encode with the table
// ---------------------------------------------------------------------------

// Cell index along one axis: floor((u(t) + 1) G / 2), as
// v = t (A G/2 + B G/2 t^2) + G/2 (the G/2 scalings are exact).  |t| <= 1 up
// to the rounding of t, so v >= -1e-6 truncates to 0; only the top needs a
// clamp.  (Points within the cells' widening of a boundary may land on either
// side: both cells list every codeword that can win there.)
__device__ __forceinline__ int cell_coord(float t) {
    constexpr float HG = 0.5f * LUT_G;
    const float v = __fmaf_rn(t, __fmaf_rn(MAP_B * HG, t * t, MAP_A * HG), HG);
    const int i = (int)v;
    return i > LUT_G - 1 ? LUT_G - 1 : i;
}

// S-codeword loop for one chunk (used for OVERFLOW cells); same result rules
// as encode.cu: ties to the lowest s, then the closed-form 2T choice.
__device__ __forceinline__ float dot_conj_score2(float x0, float x1, float x2, float x3, float4 q,
                                                 float &y0, float &y1, float &y2, float &y3) {
    y0 = __fmaf_rn(x3, q.w, __fmaf_rn(x2, q.z, __fmaf_rn(x1, q.y, __fmul_rn(x0, q.x))));
    y1 = __fmaf_rn(x3, q.z, __fmaf_rn(-x2, q.w, __fmaf_rn(x1, q.x, __fmul_rn(-x0, q.y))));
    y2 = __fmaf_rn(-x3, q.y, __fmaf_rn(x2, q.x, __fmaf_rn(x1, q.w, __fmul_rn(-x0, q.z))));
    y3 = __fmaf_rn(x3, q.x, __fmaf_rn(x2, q.y, __fmaf_rn(-x1, q.z, __fmul_rn(-x0, q.w))));
    const float a0 = fabsf(y0), a1 = fabsf(y1), a2 = fabsf(y2), a3 = fabsf(y3);
    const float m = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
    const float sum = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
    return fmaxf(__fadd_rn(m, m), sum);
}

__device__ __forceinline__ int closest_2t_of(float y0, float y1, float y2, float y3) {
    const float a0 = fabsf(y0), a1 = fabsf(y1), a2 = fabsf(y2), a3 = fabsf(y3);
    const float m = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
    const float sum = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
    if (__fadd_rn(m, m) >= sum) {
        const int ax = (a0 == m) ? 0 : (a1 == m) ? 1 : (a2 == m) ? 2 : 3;
        const float ya = ax == 0 ? y0 : ax == 1 ? y1 : ax == 2 ? y2 : y3;
        return 2 * ax + (ya < 0.0f ? 1 : 0);
    }
    return 8 + (y0 < 0.0f ? 1 : 0) + (y1 < 0.0f ? 2 : 0) + (y2 < 0.0f ? 4 : 0) +
           (y3 < 0.0f ? 8 : 0);
}

static __device__ uint32_t sloop_index(float x0, float x1, float x2, float x3,
                                const float4 *__restrict__ cb, uint32_t S) {
    float best = -1.0f;
    uint32_t bs = 0;
    float y0, y1, y2, y3;
    for (uint32_t s = 0; s < S; ++s) {
        const float sc = dot_conj_score2(x0, x1, x2, x3, __ldg(cb + s), y0, y1, y2, y3);
        if (sc > best) { best = sc; bs = s; }
    }
    dot_conj_score2(x0, x1, x2, x3, __ldg(cb + bs), y0, y1, y2, y3);
    return bs * 24u + (uint32_t)closest_2t_of(y0, y1, y2, y3);
}

__device__ __forceinline__ uint64_t shfl64(uint64_t v, int src) {
    const uint32_t lo = __shfl_sync(FULL, (uint32_t)v, src);
    const uint32_t hi = __shfl_sync(FULL, (uint32_t)(v >> 32), src);
    return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ uint64_t shfl64_down(uint64_t v, int d) {
    const uint32_t lo = __shfl_down_sync(FULL, (uint32_t)v, d);
    const uint32_t hi = __shfl_down_sync(FULL, (uint32_t)(v >> 32), d);
    return ((uint64_t)hi << 32) | lo;
}

// Packs the warp's 32 b-bit indices (lane k = chunk k) LSB-first into b words.
//
// Index width known at compile time (BB = 8 or 10): word w (lane w < BB) is
// the OR of PACK_TERMS consecutive indices, starting with chunk
// k0 = floor(32 w / BB) at bit offset o = 32 w - BB k0:
//   (idx[k0] >> o) | (idx[k0+1] << (BB - o)) | (idx[k0+2] << (2 BB - o)) | ...
// each fetched with one shuffle.  The checks below show that every shift is
// below 32 and every source lane exists.
//
// Width at run time (BB = 0, b in [5, 21]): each lane first gathers the 64-bit
// stream window starting at its own chunk (k, k+1, ..., by doubling), then
// lane w < b takes word w from the window of the chunk where that word starts.
template <int BB>
__host__ __device__ constexpr int pack_terms() {
    int n = 0;
    for (int w = 0; w < BB; ++w) {
        const int o = (32 * w) % BB;
        const int m = (31 + o) / BB + 1;
        n = m > n ? m : n;
    }
    return n;
}

template <int BB>
__host__ __device__ constexpr bool pack_plan_ok() {
    constexpr int nt = pack_terms<BB>();
    if (BB * (nt - 1) >= 32) return false;                  // a shift of 32 or more
    for (int w = 0; w < BB; ++w)
        if ((32 * w) / BB + nt - 1 > 31) return false;      // a source lane past 31
    return true;
}

struct PackConst {
    int k0, o;
};

__device__ __forceinline__ PackConst pack_const(uint32_t b, int lane) {
    PackConst c;
    c.k0 = (32 * lane) / (int)b;
    c.o = 32 * lane - c.k0 * (int)b;               // < b, and o + 32 <= 64
    c.k0 &= 31;
    return c;
}

template <int BB>
__device__ __forceinline__ void pack_group32(uint32_t idx, uint32_t b_rt, int lane, PackConst pc,
                                             uint32_t *__restrict__ dst) {
    if constexpr (BB != 0) {
        constexpr int NT = pack_terms<BB>();
        static_assert(pack_plan_ok<BB>(), "packing plan out of range");
        uint32_t wv = __shfl_sync(FULL, idx, pc.k0) >> pc.o;
#pragma unroll
        for (int m = 1; m < NT; ++m)
            wv |= __shfl_sync(FULL, idx, (pc.k0 + m) & 31) << (uint32_t)(BB * m - pc.o);
        if (lane < BB) dst[lane] = wv;
    } else {
        const uint32_t b = b_rt;
        uint64_t v = idx;
        const uint32_t n1 = __shfl_down_sync(FULL, idx, 1);
        if (lane + 1 < 32) v |= (uint64_t)n1 << b;
        const uint64_t v2 = shfl64_down(v, 2);
        if (lane + 2 < 32) v |= v2 << (2 * b);                 // 2b <= 42
        const uint64_t v4 = shfl64_down(v, 4);
        if (lane + 4 < 32 && 4 * b < 64) v |= v4 << (4 * b);
        const uint64_t vk = shfl64(v, pc.k0);
        if (lane < (int)b) dst[lane] = (uint32_t)(vk >> pc.o);
    }
}

// LIST: 0 = no list; HQMQ_GRAN_CHUNK + 1 / HQMQ_GRAN_ELEMENT + 1 = write the
// ordered outlier list of that granularity (thr exact, tile_off from the
// Med3x window pipeline).  ENC: encode (else write the list only).
// LIST_SPEC (chunk mode, the one-read path, before the exact threshold is
// known): also does pass B's work for the Med3x window (keys below and inside
// the window, certain outliers per tile, uncertain keys) and encodes
// speculatively: a chunk with r > t_hi (above every possible threshold) as an
// outlier (index 0, radius 0), every other chunk as a bulk chunk; records per
// packing group the chunks with r > t_lo.
// (k_list_fix, after the exact threshold, then writes the list.)
// Work: warp tiles of TILE_GROUPS consecutive packing groups; a CTA owns a
// contiguous range of tiles and walks it slab by slab (one head at a time).
// Packs a warp tile's indices, staged in shared memory (s_idx[k], k = the
// chunk's position in the tile), into the tile's ng * BB words: lane l
// writes words l, l + 32, ... (coalesced), word w being the OR of the
// pack_terms<BB>() indices that overlap it (see pack_group32).
template <int BB>
__device__ __forceinline__ void pack_tile(const uint16_t *s_idx, uint32_t ng, int lane,
                                          uint32_t *__restrict__ dst) {
    constexpr int NT = pack_terms<BB>();
    static_assert(pack_plan_ok<BB>(), "packing plan out of range");
    const uint32_t nw = ng * BB;
    for (uint32_t w = (uint32_t)lane; w < nw; w += 32) {
        const uint32_t k0 = (32u * w) / BB;
        const uint32_t o = 32u * w - BB * k0;
        uint32_t v = (uint32_t)s_idx[k0] >> o;
#pragma unroll
        for (int m = 1; m < NT; ++m) v |= (uint32_t)s_idx[k0 + m] << (uint32_t)(BB * m - o);
        dst[w] = v;
    }
}

constexpr int LIST_SPEC = 3;

// Clears the b-bit index of lane `lane` in its packing group's words.
__device__ __forceinline__ void clear_index(uint32_t *gw, uint32_t b, int lane) {
    const uint32_t bit = b * (uint32_t)lane, w0 = bit >> 5, o = bit & 31u;
    const uint32_t mask = (1u << b) - 1u;                // (b <= 21)
    atomicAnd(gw + w0, ~(mask << o));
    if (o + b > 32u) atomicAnd(gw + w0 + 1, ~(mask >> (32u - o)));
}

// Shared memory of the table encode: the 24 S codewords and a zero word, in
// 8 copies.
inline size_t enc_smem_bytes(uint32_t S) { return ((size_t)24 * S + 1) * 8 * sizeof(float4); }

}  // namespace hqmq
