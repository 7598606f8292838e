// med3_window.cuh -- shared layout of the windowed Med3x pipeline
// (med3_window.cu: sample, window, full pass, selection, tile offsets;
// search.cu: the encode pass that also writes the ordered outlier list).
#pragma once

#include <math.h>

#include "hqmq_device.cuh"

namespace hqmq {

constexpr int TILE_GROUPS = 32;                  // packing groups per warp tile
constexpr int TILE_CHUNKS = TILE_GROUPS * 32;    // 1024 chunks
constexpr int SAMPLE_PERIOD = 128;               // one sampled quad (4 chunks) per 128 chunks
constexpr int KEY_BINS = 65536;                  // sample histogram
constexpr int WINDOW_SIGMAS = 8;                 // half-width of the rank window

// Per-head state of the rank window.
struct WinState {
    uint32_t lo_key, hi_key;   // candidate keys: lo_key <= key < hi_key
    uint32_t miss;             // 1: exact fallback decides this head
    float t_lo, t_hi;          // thr is known to lie in [t_lo, t_hi]
    uint32_t pad[3];
};

// Counters, cleared with the histograms at the start of every call.
struct Counters {
    unsigned long long amb_n;  // uncertain (tile, key) pairs appended
    uint32_t fin_done;         // CTAs of the finalize step that are done
    uint32_t pad;
    // followed by uint32_t sample_done[H]: sample CTAs of head h that are done,
    // then uint32_t median_done[H]: finalize CTAs of head h that are done
};

constexpr int MED_BINS = 4096;                   // radix digit of the median select (12 bits)
constexpr int CVAL_SLOTS = 32;                   // possible outliers kept per 256-chunk unit
constexpr int MED_SLICES = 16;                   // finalize CTAs per head

struct FusedLayout {
    uint64_t sample_hist, counters, med_hist, win, below, cand_n, cand, amb, tile_cnt, tile_off,
        cbits, head_stat, cvals, total;
    uint64_t zero_bytes;       // [0, zero_bytes) is cleared per call
    uint64_t cand_cap;         // keys per head
    uint64_t amb_cap;          // (tile, key) pairs per call
    uint64_t n_per_head;       // keys per head (chunks or elements)
    uint32_t tiles_per_slab;
    uint64_t n_tiles;
};

inline uint64_t align256_(uint64_t v) { return (v + 255) & ~(uint64_t)255; }

inline FusedLayout fused_layout(int B, int H, int T, int D, int gran) {
    FusedLayout L;
    const uint64_t cps = (uint64_t)T * D / 4;
    const uint64_t gps = cps / 32;
    L.tiles_per_slab = (uint32_t)((gps + TILE_GROUPS - 1) / TILE_GROUPS);
    L.n_tiles = (uint64_t)B * H * L.tiles_per_slab;
    L.n_per_head = (uint64_t)B * cps * (gran == HQMQ_GRAN_CHUNK ? 1 : 4);
    // expected window: +-WINDOW_SIGMAS sample standard deviations of the median
    // rank, plus the two 2^15-key edge bins; the buffer holds twice that
    const double ns = (double)L.n_per_head / 32.0 + 1.0;
    const double frac = (2.0 * WINDOW_SIGMAS * 0.5 * sqrt(ns) + 8.0) / ns + 0.02;
    uint64_t cap = (uint64_t)(2.0 * frac * (double)L.n_per_head) + 4096;
    L.cand_cap = cap < L.n_per_head ? cap : L.n_per_head;
    L.cand_cap = (L.cand_cap + 3) & ~(uint64_t)3;   // each head's keys start 16-byte aligned
    const uint64_t n_keys = L.n_per_head * H;
    L.amb_cap = n_keys / 25 + 4096;              // 4% of the keys may sit in thr's band
    uint64_t off = 0;
    L.sample_hist = off; off = align256_(off + (uint64_t)H * KEY_BINS * 4);
    L.counters = off;    off = align256_(off + sizeof(Counters) + (uint64_t)H * 8);
    L.med_hist = off;    off = align256_(off + (uint64_t)H * MED_BINS * 4 * 2);   // top digit, then next
    L.head_stat = off;   off = align256_(off + (uint64_t)H * 16);   // per head: non-finite, saturated
    L.tile_cnt = off;    off = align256_(off + L.n_tiles * 4);      // (a tile may be counted by several warps)
    L.zero_bytes = off;
    L.win = off;         off = align256_(off + (uint64_t)H * sizeof(WinState));
    L.below = off;       off = align256_(off + (uint64_t)H * 8);
    L.cand_n = off;      off = align256_(off + (uint64_t)H * 8);
    L.cand = off;        off = align256_(off + (uint64_t)H * L.cand_cap * 4);
    L.amb = off;         off = align256_(off + L.amb_cap * 8);
    L.tile_off = off;    off = align256_(off + (L.n_tiles + 1) * 4);
    L.cbits = off;       off = align256_(off + (uint64_t)B * H * gps * 4);
    // raw values of the possible outliers (r > t_lo), CVAL_SLOTS per 8-group
    // unit (chunk mode; 16 bytes per chunk covers fp32 input)
    L.cvals = off;       off = align256_(off + (uint64_t)B * H * ((gps + 7) / 8) * CVAL_SLOTS * 16);
    L.total = off;
    return L;
}

constexpr int STAGE = 256;          // window keys staged per warp before one global append

// Shift of the top radix digit of the median select: keys are taken as
// d = key - lo_key < span, cut into 12-bit digits from the top of the span.
__host__ __device__ __forceinline__ int median_top_shift(uint32_t span) {
    int bits = 0;
    for (uint32_t v = span - 1u; v; v >>= 1) ++bits;
    return ((bits + 11) / 12 - 1) * 12;
}

// Appends the warp's staged window keys to the head's buffer (one atomic) and
// counts each appended key's top digit (median_top_shift) into the head's
// digit histogram, so that the select starts from a complete histogram.
__device__ __forceinline__ void flush_stage(uint32_t *stage, uint32_t n, int lane,
                                            unsigned long long *cand_n_h, uint32_t *cand_h,
                                            uint64_t cand_cap, uint32_t *hist_h, uint32_t lo_key,
                                            int top) {
    __syncwarp();                                  // the lanes' stage writes
    unsigned long long base = 0;
    if (lane == 0) base = atomicAdd(cand_n_h, (unsigned long long)n);
    base = __shfl_sync(FULL, base, 0);
    for (uint32_t i = lane; i < n; i += 32)
        if (base + i < cand_cap) {
            const uint32_t key = stage[i];
            cand_h[base + i] = key;
            atomicAdd(hist_h + (((key - lo_key) >> top) & (MED_BINS - 1)), 1u);
        }
    __syncwarp();
}

// Workspace pointers of the one-read chunk-mode path: the encode pass also
// does pass B's work and encodes speculatively (a chunk above the largest
// possible threshold t_hi as an outlier, every other chunk as a bulk chunk);
// the fix-up pass after the exact threshold writes the list.
struct SpecArgs {
    const WinState *win;
    unsigned long long *below, *cand_n, *amb_n;
    uint32_t *cand, *tile_cnt;
    uint2 *amb;
    uint64_t cand_cap, amb_cap;
    uint32_t *cbits;                 // per packing group: chunks with r > t_lo
    unsigned long long *head_stat;   // per head: [non-finite, saturated] of the encode pass
    uint32_t *med_hist;              // per head: top-digit counts of the staged keys
    unsigned char *cvals;            // per unit: raw values of its first CVAL_SLOTS possible outliers
};

inline SpecArgs spec_args(char *ws, const FusedLayout &L) {
    SpecArgs a;
    a.win = reinterpret_cast<const WinState *>(ws + L.win);
    a.below = reinterpret_cast<unsigned long long *>(ws + L.below);
    a.cand_n = reinterpret_cast<unsigned long long *>(ws + L.cand_n);
    a.amb_n = reinterpret_cast<unsigned long long *>(ws + L.counters);   // Counters::amb_n
    a.cand = reinterpret_cast<uint32_t *>(ws + L.cand);
    a.tile_cnt = reinterpret_cast<uint32_t *>(ws + L.tile_cnt);
    a.amb = reinterpret_cast<uint2 *>(ws + L.amb);
    a.cand_cap = L.cand_cap;
    a.amb_cap = L.amb_cap;
    a.cbits = reinterpret_cast<uint32_t *>(ws + L.cbits);
    a.head_stat = reinterpret_cast<unsigned long long *>(ws + L.head_stat);
    a.med_hist = reinterpret_cast<uint32_t *>(ws + L.med_hist);
    a.cvals = reinterpret_cast<unsigned char *>(ws + L.cvals);
    return a;
}

}  // namespace hqmq
