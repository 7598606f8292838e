// med3_window.cu -- Med3x in two reads of x.
//
// The rule (gist.science/nl, Technische Samenvatting, section 3; gist.science/
// pt, Resumo Tecnico, section 3): r_med = the median chunk norm over the current
// batch (here: per head over one call, lower median at rank N/2 - 1), outlier
// iff r > fl32(C r_med).  The results are exactly those of the three-pass radix
// select of med3.cu; only the data flow differs:
//
//  A+W k_sample_window reads a 1/32 sample (the first 128 chunks of every
//                      4096, read by a warp as one contiguous block) into a
//                      per-head histogram of the top 16 key bits; the last
//                      CTA of each head then picks a key window [lo, hi) that
//                      holds the sample ranks within +-8 standard deviations of
//                      the median rank; the exact threshold then lies in
//                      [t_lo, t_hi].
//  B   k_pass_b        one full read: per head the count of keys below the
//                      window and the keys inside it (staged per warp, appended
//                      to the head's list);
//                      per 1024-chunk tile the count of certain outliers
//                      (r > t_hi) and a list of uncertain ones (t_lo < r <= t_hi).
//  F   k_finalize      per head: the exact median from the window keys (radix
//                      select, 12-bit digits), or,
//                      if the window missed the median (or a buffer
//                      overflowed), the exact three-pass select over x and
//                      exact tile counts (never taken on the bench workloads;
//                      it keeps the result exact for any input); then the
//                      uncertain keys above the exact threshold; the last CTA
//                      scans the tile counts into tile and slab offsets.
//  C   (search.cu)     the second read writes the ordered list (and encodes).
//                      In chunk mode with search tables the encode pass does
//                      B's work in the same, single read of x, and a fix-up
//                      pass after F writes the list (search.cu, LIST_SPEC and
//                      LIST_FIX).
//
// A memset clears the histograms and counters first.  No CTA waits for
// another: where a step needs the results of all CTAs of the previous one,
// the last CTA to finish (an atomic ticket after a fence) does it.
#include "med3_window.cuh"

namespace hqmq {

constexpr int WIN_THREADS = 1024;
constexpr int PB_THREADS = 256;


__device__ __forceinline__ float key_to_float(uint32_t k) {
    return k >= 0x7F800001u ? __int_as_float(0x7FC00000) : __uint_as_float(k);
}

// fl32(C * value of key); a key at or above +inf's maps to +inf
__device__ __forceinline__ float thr_of_key(float C, uint32_t k) {
    if (k >= 0x7F800000u) return __int_as_float(0x7F800000);
    return __fmul_rn(C, __uint_as_float(k));
}

template <int GRAN>
__device__ __forceinline__ void chunk_keys(float x0, float x1, float x2, float x3, uint32_t *k) {
    if (GRAN == HQMQ_GRAN_CHUNK) {
        k[0] = mag_key(chunk_norm(x0, x1, x2, x3));
    } else {
        k[0] = mag_key(fabsf(x0));
        k[1] = mag_key(fabsf(x1));
        k[2] = mag_key(fabsf(x2));
        k[3] = mag_key(fabsf(x3));
    }
}

// ---------------------------------------------------------------------------
// Histogram search helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(FULL, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// Block-wide (1024 threads) select of two ranks in a histogram of NB bins.
// Warp w owns the contiguous bins [w NB/32, (w+1) NB/32), read as 128-bin
// pieces (lane l: bins 4l..4l+3 of each piece, one 16-byte load; all pieces
// in flight).  One block scan of the 32 warp totals finds the warp holding
// each rank; that warp finds the piece from its piece totals, re-reads that
// piece and scans it.  Returns in s_out[k] the bin whose cumulative count
// first exceeds rank k (k = 0, 1) and in s_out[k + 2] the rank inside that bin
// (NB - 1 and 0 if the rank is not below the total).
template <bool GLOBAL>
__device__ __forceinline__ uint4 hist_ld4(const uint32_t *p) {
    // GLOBAL: bins written by other CTAs of this kernel (read through L2)
    if constexpr (GLOBAL) return __ldcg(reinterpret_cast<const uint4 *>(p));
    else return *reinterpret_cast<const uint4 *>(p);
}

template <int NB, bool GLOBAL>
__device__ void block_select2(const uint32_t *hist, uint64_t r0, uint64_t r1, uint32_t *s_warp,
                              uint32_t *s_out) {
    constexpr int PW = NB / 32;                         // bins per warp
    constexpr int NP = PW / 128;                        // 128-bin pieces per warp
    static_assert(PW % 128 == 0 && NP <= 16, "histogram size");
    const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
    if (t == 0) {
        s_out[0] = s_out[1] = NB - 1;
        s_out[2] = s_out[3] = 0;
    }
    const uint32_t *wh = hist + wid * PW;
    uint32_t ps[NP];
#pragma unroll
    for (int c = 0; c < NP; ++c) {
        const uint4 u = hist_ld4<GLOBAL>(wh + c * 128 + 4 * lane);
        ps[c] = u.x + u.y + u.z + u.w;
    }
    uint32_t wtot = 0;
#pragma unroll
    for (int c = 0; c < NP; ++c) {
        ps[c] = __reduce_add_sync(FULL, ps[c]);
        wtot += ps[c];
    }
    if (lane == 0) s_warp[wid] = wtot;
    __syncthreads();
    if (wid == 0) {
        const uint32_t wv = s_warp[lane];
        s_warp[lane] = warp_incl_scan(wv, lane) - wv;
    }
    __syncthreads();
    const uint64_t wex = s_warp[wid];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint64_t r = k ? r1 : r0;
        if (r < wex || r >= wex + wtot) continue;       // (warp-uniform)
        uint64_t c0 = wex;
        int pc = NP - 1;
#pragma unroll
        for (int c = 0; c < NP; ++c) {
            if (r < c0 + ps[c]) { pc = c; break; }
            c0 += ps[c];
        }
        const uint4 u = hist_ld4<GLOBAL>(wh + pc * 128 + 4 * lane);
        const uint32_t ls = u.x + u.y + u.z + u.w;
        const uint32_t inc = warp_incl_scan(ls, lane);
        const uint64_t before = c0 + inc - ls;
        if (r >= before && r < before + ls) {
            const uint32_t rr = (uint32_t)(r - before);
            const uint32_t e = rr < u.x ? 0 : rr < u.x + u.y ? 1 : rr < u.x + u.y + u.z ? 2 : 3;
            const uint32_t eb = e == 0 ? 0 : e == 1 ? u.x : e == 2 ? u.x + u.y : u.x + u.y + u.z;
            s_out[k] = (uint32_t)(wid * PW + pc * 128 + 4 * lane) + e;
            s_out[k + 2] = rr - eb;
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// A + W: sample histogram; the last sample CTA of each head picks its window
// ---------------------------------------------------------------------------
constexpr int SAMPLE_THREADS = 1024;

// Window of head h from its complete sample histogram (one CTA).  n_samples:
// the head's sample count (every sampled quad adds 4 chunks' keys).
__device__ void select_window(int h, uint64_t n_per_head, uint64_t n_samples, float C,
                              const uint32_t *hist, WinState *win, unsigned long long *below,
                              unsigned long long *cand_n, uint32_t *s_warp, uint32_t *s_out) {
    const double ns = (double)n_samples;
    const double q = ((double)(n_per_head / 2 - 1) + 0.5) / (double)n_per_head;
    const double half = WINDOW_SIGMAS * 0.5 * sqrt(ns) + 4.0;
    double rlo = floor(q * ns - half), rhi = ceil(q * ns + half);
    if (rlo < 0) rlo = 0;
    if (rhi > ns - 1) rhi = ns - 1;
    block_select2<KEY_BINS, true>(hist, (uint64_t)rlo, (uint64_t)rhi, s_warp, s_out);
    if (threadIdx.x == 0) {
        WinState w;
        const uint64_t lo = (uint64_t)s_out[0] << 15;
        uint64_t hi = ((uint64_t)s_out[1] + 1) << 15;
        if (hi > 0x80000000ull) hi = 0x80000000ull;
        w.lo_key = (uint32_t)lo;
        w.hi_key = (uint32_t)(hi - 1) + 1u;          // (hi <= 2^31)
        w.miss = 0;
        w.t_lo = thr_of_key(C, (uint32_t)lo);
        w.t_hi = thr_of_key(C, (uint32_t)(hi - 1));
        w.pad[0] = w.pad[1] = w.pad[2] = 0;
        win[h] = w;
        below[h] = 0;
        cand_n[h] = 0;
    }
}

template <int DT, int GRAN>
__global__ void __launch_bounds__(SAMPLE_THREADS, 1)
k_sample_window(const void *__restrict__ x, int H, uint32_t cps, uint32_t ctas_per_head,
                uint64_t n_per_head, uint64_t n_samples, float C, uint32_t *__restrict__ hist,
                uint32_t *__restrict__ sample_done, WinState *__restrict__ win,
                unsigned long long *__restrict__ below, unsigned long long *__restrict__ cand_n) {
    // per-CTA histogram in shared memory: 65536 16-bit counters packed in
    // pairs (a CTA sees far fewer than 65536 samples), then one global add
    // per non-empty bin
    extern __shared__ uint32_t s_pair[];                       // [KEY_BINS / 2]
    __shared__ uint32_t s_warp[32], s_out[4], s_last;
    pdl_trigger();                                 // (the encode pass may be scheduled)
    for (int i = threadIdx.x; i < KEY_BINS / 2; i += blockDim.x) s_pair[i] = 0;
    __syncthreads();
    const int slab = blockIdx.y;
    const int h = slab % H;
    uint32_t *hh = hist + (size_t)h * KEY_BINS;
    const uint64_t base = (uint64_t)slab * cps;
    const uint32_t n_quads = (cps + SAMPLE_PERIOD - 1) / SAMPLE_PERIOD;
    for (uint32_t q = blockIdx.x * blockDim.x + threadIdx.x; q < n_quads;
         q += gridDim.x * blockDim.x) {
        // quads 32 m .. 32 m + 31 read the first 128 chunks (1 KB of bf16) of
        // the m-th run of 32 x 128 chunks: a warp reads one contiguous block
        // (the same sample size as one quad per 128 chunks, without the DRAM
        // fetch granularity reading 4 x the sampled bytes), and the block
        // holds whole head vectors, every position inside them; a quad past
        // the slab's last full run reads the start of its own 128 chunks
        uint64_t j0 = base + (uint64_t)(q >> 5) * (32u * SAMPLE_PERIOD) + 4u * (q & 31u);
        if (j0 + 4 > base + cps) j0 = base + (uint64_t)q * SAMPLE_PERIOD;
        RawChunk<DT> v[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c].load(x, j0 + c);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            constexpr int NK = GRAN == HQMQ_GRAN_CHUNK ? 1 : 4;
            uint32_t k[4];
            chunk_keys<GRAN>(v[c].e(0), v[c].e(1), v[c].e(2), v[c].e(3), k);
#pragma unroll
            for (int i = 0; i < NK; ++i) {
                const uint32_t bin = k[i] >> 15;
                atomicAdd(&s_pair[bin >> 1], 1u << ((bin & 1) * 16));
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < KEY_BINS / 2; i += blockDim.x) {
        const uint32_t v = s_pair[i];
        if (v & 0xFFFFu) atomicAdd(hh + 2 * i, v & 0xFFFFu);
        if (v >> 16) atomicAdd(hh + 2 * i + 1, v >> 16);
    }
    // the last of the head's CTAs (no CTA waits for another) reads the
    // complete histogram: every CTA's adds are ordered before its ticket
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(sample_done + h, 1u) == ctas_per_head - 1 ? 1u : 0u;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    select_window(h, n_per_head, n_samples, C, hh, win, below, cand_n, s_warp, s_out);
}

// ---------------------------------------------------------------------------
// B: one full read
// ---------------------------------------------------------------------------
template <int DT, int GRAN>
__global__ void __launch_bounds__(PB_THREADS)
k_pass_b(const void *__restrict__ x, int H, uint32_t cps, uint32_t tiles_per_slab, uint64_t n_tiles,
         const WinState *__restrict__ win, unsigned long long *__restrict__ below,
         unsigned long long *__restrict__ cand_n, uint32_t *__restrict__ cand, uint64_t cand_cap,
         unsigned long long *__restrict__ amb_n,
         uint2 *__restrict__ amb, uint64_t amb_cap, uint32_t *__restrict__ tile_cnt,
         uint32_t *__restrict__ med_hist) {
    constexpr int NK = GRAN == HQMQ_GRAN_CHUNK ? 1 : 4;
    constexpr int U = 8;                              // groups in flight per lane
    const int lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    const uint32_t gps = cps / 32;
    const uint64_t warp_g = (uint64_t)blockIdx.x * (PB_THREADS / 32) + (threadIdx.x >> 5);
    const uint64_t n_warps = (uint64_t)gridDim.x * (PB_THREADS / 32);
    __shared__ uint32_t s_stage[PB_THREADS / 32][STAGE];
    uint32_t *stage = s_stage[threadIdx.x >> 5];
    uint32_t n_stage = 0;
    int stage_h = -1;
    for (uint64_t t = warp_g; t < n_tiles; t += n_warps) {
        const uint64_t slab = t / tiles_per_slab;
        const uint32_t ti = (uint32_t)(t % tiles_per_slab);
        const int h = (int)(slab % (uint64_t)H);
        const WinState w = win[h];
        if (h != stage_h) {                                   // warp-uniform
            if (n_stage) {
                const WinState ws = win[stage_h];
                flush_stage(stage, n_stage, lane, cand_n + stage_h,
                            cand + (uint64_t)stage_h * cand_cap, cand_cap,
                            med_hist + (size_t)stage_h * MED_BINS * 2, ws.lo_key,
                            median_top_shift(ws.hi_key - ws.lo_key));
            }
            n_stage = 0;
            stage_h = h;
        }
        const uint32_t g0 = ti * TILE_GROUPS;
        const uint32_t g1 = min(g0 + TILE_GROUPS, gps);
        unsigned long long n_below = 0;
        uint32_t n_def = 0;
        for (uint32_t g = g0; g < g1; g += U) {
            RawChunk<DT> v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                v[u].zero();
                if (g + u < g1) v[u].load(x, (slab * gps + g + u) * 32 + lane);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (g + u >= g1) break;                       // warp-uniform
                uint32_t k[4];
                chunk_keys<GRAN>(v[u].e(0), v[u].e(1), v[u].e(2), v[u].e(3), k);
#pragma unroll
                for (int i = 0; i < NK; ++i) {
                    const uint32_t key = k[i];
                    n_below += key < w.lo_key ? 1u : 0u;
                    const bool in = key >= w.lo_key && key < w.hi_key;
                    const uint32_t m = __ballot_sync(FULL, in);
                    if (m) {
                        if (n_stage + 32 > STAGE) {
                            flush_stage(stage, n_stage, lane, cand_n + h,
                                        cand + (uint64_t)h * cand_cap, cand_cap,
                                        med_hist + (size_t)h * MED_BINS * 2, w.lo_key,
                                        median_top_shift(w.hi_key - w.lo_key));
                            n_stage = 0;
                        }
                        if (in) {
                            stage[n_stage + __popc(m & lt)] = key;
                        }
                        n_stage += __popc(m);
                        __syncwarp();
                    }
                    const float val = __uint_as_float(key);     // NaN keys compare false
                    n_def += val > w.t_hi ? 1u : 0u;
                    const bool amb_in = val > w.t_lo && val <= w.t_hi;
                    const uint32_t ma = __ballot_sync(FULL, amb_in);
                    if (ma) {
                        unsigned long long base = 0;
                        if (lane == 0) base = atomicAdd(amb_n, (unsigned long long)__popc(ma));
                        base = __shfl_sync(FULL, base, 0);
                        if (amb_in) {
                            const unsigned long long pos = base + __popc(ma & lt);
                            if (pos < amb_cap) amb[pos] = make_uint2((uint32_t)t, key);
                        }
                    }
                }
            }
        }
        n_below = __reduce_add_sync(FULL, (unsigned)n_below);
        n_def = __reduce_add_sync(FULL, n_def);
        if (lane == 0) {
            tile_cnt[t] = n_def;
            if (n_below) atomicAdd(below + h, n_below);
        }
    }
    if (n_stage) {
        const WinState ws = win[stage_h];
        flush_stage(stage, n_stage, lane, cand_n + stage_h, cand + (uint64_t)stage_h * cand_cap,
                    cand_cap, med_hist + (size_t)stage_h * MED_BINS * 2, ws.lo_key,
                    median_top_shift(ws.hi_key - ws.lo_key));
    }
}

// ---------------------------------------------------------------------------
// F + X + U + S: per head the exact median (or the exact fallback), the
// uncertain keys above it; the last CTA then scans the tile counts
// ---------------------------------------------------------------------------
struct __align__(16) FinalSmem {
    uint32_t buf[MED_BINS];            // digit counts (median) or 2048 bins (fallback)
    uint32_t wtot[32];
    uint32_t out[4];
    uint32_t last;
};

// Exact median of head h from its staged window keys: the key of rank
// k = N/2 - 1 - below among them, by a radix select on d = key - lo_key in
// 12-bit digits from the top of the window's span.  The top digit's counts
// come from all MED_SLICES finalize CTAs of the head (each counts a slice of
// the keys into the head's global histogram); the head's last CTA selects it
// and runs the remaining digits alone (only keys inside the chosen bin
// count).
struct MedianPlan {
    bool ok;                 // false: the window missed (the exact fallback decides)
    uint32_t k;              // rank among the staged keys
    uint64_t nc;             // staged keys
    uint32_t span;           // hi_key - lo_key
    int top;                 // shift of the top digit
};

__device__ MedianPlan median_plan(int h, uint64_t n_per_head, const WinState &w,
                                  const unsigned long long *below,
                                  const unsigned long long *cand_n, uint64_t cand_cap,
                                  bool amb_overflow) {
    MedianPlan p;
    const long long k = (long long)(n_per_head / 2 - 1) - (long long)below[h];
    p.nc = cand_n[h];
    p.ok = !(amb_overflow || k < 0 || (unsigned long long)k >= p.nc || p.nc > cand_cap);
    p.k = p.ok ? (uint32_t)k : 0u;
    p.span = w.hi_key - w.lo_key;                      // >= 2^15
    p.top = median_top_shift(p.span);
    return p;
}

// Adds the digit at shift sh of every staged key d in [i_begin, i_end) whose
// bits above the digit equal those of `prefix` to hist (shared, MED_BINS).
__device__ void median_count(const uint32_t *ch, uint64_t i_begin, uint64_t i_end,
                             const WinState &w, uint32_t span, int sh, uint32_t prefix,
                             uint32_t *hist) {
    const int hs = sh + 12;                            // bits above this digit
    const uint32_t want = hs >= 32 ? 0u : prefix >> hs;
    auto add = [&](uint32_t key) {
        const uint32_t d = key - w.lo_key;
        if (d < span && (hs >= 32 || (d >> hs) == want))
            atomicAdd(&hist[(d >> sh) & (MED_BINS - 1)], 1u);
    };
    // 16-byte loads from the first multiple of 4 at or after i_begin
    uint64_t a = (i_begin + 3) & ~(uint64_t)3;
    if (a > i_end) a = i_end;
    for (uint64_t i = i_begin + threadIdx.x; i < a; i += WIN_THREADS) add(ch[i]);
    const uint64_t n4 = (i_end - a) / 4;
    const uint4 *ch4 = reinterpret_cast<const uint4 *>(ch + a);
    constexpr int U = 4;
    for (uint64_t i0 = threadIdx.x; i0 < n4; i0 += (uint64_t)U * WIN_THREADS) {
        uint4 q[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint64_t i = i0 + (uint64_t)u * WIN_THREADS;
            q[u] = i < n4 ? ch4[i] : make_uint4(w.hi_key, w.hi_key, w.hi_key, w.hi_key);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) { add(q[u].x); add(q[u].y); add(q[u].z); add(q[u].w); }
    }
    for (uint64_t i = a + 4 * n4 + threadIdx.x; i < i_end; i += WIN_THREADS) add(ch[i]);
}

// Exact three-pass radix select over x for head h, then its exact tile
// counts (the path when the sample window missed the median).
template <int DT, int GRAN>
__device__ void exact_fallback(const void *x, int B, int H, int h, uint32_t cps,
                               uint32_t tiles_per_slab, uint64_t n_per_head, float C, float *rmed,
                               float *thr, uint32_t *tile_cnt, DevStatus *st, FinalSmem &sm) {
    constexpr int NK = GRAN == HQMQ_GRAN_CHUNK ? 1 : 4;
    uint32_t *s_hist = sm.buf;                         // 2048 bins
    uint32_t *s_warp = sm.wtot;
    if (threadIdx.x == 0 && st) atomicOr(&st->flags, HQMQ_FLAG_MED3_FALLBACK);
    uint32_t prefix = 0;
    uint64_t krem = n_per_head / 2 - 1;
    const int shifts[3] = {20, 9, 0};
    const int widths[3] = {11, 11, 9};
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int P = 0; P < 3; ++P) {
        for (int i = threadIdx.x; i < 2048; i += WIN_THREADS) s_hist[i] = 0;
        __syncthreads();
        const int sh = shifts[P], hs = sh + widths[P];
        const uint32_t mask = (1u << widths[P]) - 1u;
        for (int b = 0; b < B; ++b) {
            const uint64_t base = ((uint64_t)b * H + h) * cps;
            for (uint32_t c = threadIdx.x; c < cps; c += WIN_THREADS) {
                RawChunk<DT> v;
                v.load(x, base + c);
                uint32_t k[4];
                chunk_keys<GRAN>(v.e(0), v.e(1), v.e(2), v.e(3), k);
#pragma unroll
                for (int i = 0; i < NK; ++i)
                    if (P == 0 || (k[i] >> hs) == (prefix >> hs))
                        atomicAdd(&s_hist[(k[i] >> sh) & mask], 1u);
            }
        }
        __syncthreads();
        // 2048 bins: thread t owns bins 2t and 2t+1
        const uint32_t b0 = s_hist[2 * threadIdx.x], b1 = s_hist[2 * threadIdx.x + 1];
        const uint32_t local = b0 + b1;
        const uint32_t inc = warp_incl_scan(local, lane);
        if (lane == 31) s_warp[wid] = inc;
        __syncthreads();
        if (wid == 0) {
            const uint32_t wv = s_warp[lane];
            s_warp[lane] = warp_incl_scan(wv, lane) - wv;
        }
        __syncthreads();
        const uint64_t excl = (uint64_t)s_warp[wid] + inc - local;
        if (krem >= excl && krem < excl + local) {
            const uint32_t digit = krem < excl + b0 ? 2 * threadIdx.x : 2 * threadIdx.x + 1;
            sm.out[0] = digit;
            sm.out[1] = (uint32_t)(krem - (krem < excl + b0 ? excl : excl + b0));
        }
        __syncthreads();
        prefix |= sm.out[0] << sh;
        krem = sm.out[1];
        __syncthreads();
    }
    const float m = key_to_float(prefix);
    const float th = __fmul_rn(C, m);
    if (threadIdx.x == 0) { rmed[h] = m; thr[h] = th; }
    // exact tile counts of this head's slabs
    const uint32_t gps = cps / 32;
    for (int b = 0; b < B; ++b) {
        const uint64_t slab = (uint64_t)b * H + h;
        for (uint32_t ti = wid; ti < tiles_per_slab; ti += WIN_THREADS / 32) {
            uint32_t n = 0;
            const uint32_t g1 = min((ti + 1) * TILE_GROUPS, gps);
            for (uint32_t g = ti * TILE_GROUPS; g < g1; ++g) {
                RawChunk<DT> v;
                v.load(x, (slab * gps + g) * 32 + lane);
                uint32_t k[4];
                chunk_keys<GRAN>(v.e(0), v.e(1), v.e(2), v.e(3), k);
#pragma unroll
                for (int i = 0; i < NK; ++i) n += __uint_as_float(k[i]) > th ? 1u : 0u;
            }
            n = __reduce_add_sync(FULL, n);
            if (lane == 0) tile_cnt[slab * tiles_per_slab + ti] = n;
        }
    }
}

// Exclusive scan of the tile counts into tile offsets (n_tiles + 1 entries,
// the last one the total) and slab offsets (one CTA).  Per step, warp w owns SCAN_WARP consecutive tiles, read and written as
// 128-tile pieces (lane l: tiles 4l..4l+3 of each piece, one 16-byte access;
// all pieces in flight); each piece is scanned by the warp, the block scans
// the 32 warp totals.
constexpr int SCAN_PIECES = 8;
constexpr int SCAN_WARP = SCAN_PIECES * 128;
__device__ void scan_tiles(const uint32_t *tile_cnt, uint64_t n_tiles, uint32_t tiles_per_slab,
                           uint32_t n_slabs, uint64_t cap, uint32_t *tile_off, uint32_t *slab_off,
                           DevStatus *st, FinalSmem &sm) {
    const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
    uint32_t *s_warp = sm.wtot;
    unsigned long long carry = 0;                      // (the same in every thread)
    for (uint64_t b0 = 0; b0 < n_tiles; b0 += (uint64_t)SCAN_WARP * 32) {
        const uint64_t wb = b0 + (uint64_t)wid * SCAN_WARP;
        uint4 v[SCAN_PIECES];
#pragma unroll
        for (int c = 0; c < SCAN_PIECES; ++c) {
            const uint64_t i0 = wb + c * 128 + 4 * lane;
            if (i0 + 4 <= n_tiles) {
                v[c] = __ldcg(reinterpret_cast<const uint4 *>(tile_cnt + i0));
            } else {
                v[c].x = i0 < n_tiles ? __ldcg(tile_cnt + i0) : 0u;
                v[c].y = i0 + 1 < n_tiles ? __ldcg(tile_cnt + i0 + 1) : 0u;
                v[c].z = i0 + 2 < n_tiles ? __ldcg(tile_cnt + i0 + 2) : 0u;
                v[c].w = 0u;                           // (i0 + 3 >= n_tiles here)
            }
        }
        // (a tile holds at most 4096 keys: every partial sum below fits 32 bits)
        uint32_t inc[SCAN_PIECES], ls[SCAN_PIECES], wtot = 0;
#pragma unroll
        for (int c = 0; c < SCAN_PIECES; ++c) {
            ls[c] = v[c].x + v[c].y + v[c].z + v[c].w;
            inc[c] = warp_incl_scan(ls[c], lane);
            wtot += __shfl_sync(FULL, inc[c], 31);
        }
        if (lane == 0) s_warp[wid] = wtot;
        __syncthreads();
        if (wid == 0) {
            const uint32_t wv = s_warp[lane];
            const uint32_t wi = warp_incl_scan(wv, lane);
            s_warp[lane] = wi - wv;
            if (lane == 31) sm.out[0] = wi;                // this step's total
        }
        __syncthreads();
        uint32_t base = (uint32_t)(carry + s_warp[wid]);
#pragma unroll
        for (int c = 0; c < SCAN_PIECES; ++c) {
            const uint64_t i0 = wb + c * 128 + 4 * lane;
            uint4 o;
            o.x = base + inc[c] - ls[c];
            o.y = o.x + v[c].x;
            o.z = o.y + v[c].y;
            o.w = o.z + v[c].z;
            if (i0 + 4 <= n_tiles) {
                *reinterpret_cast<uint4 *>(tile_off + i0) = o;
            } else {
                if (i0 < n_tiles) tile_off[i0] = o.x;
                if (i0 + 1 < n_tiles) tile_off[i0 + 1] = o.y;
                if (i0 + 2 < n_tiles) tile_off[i0 + 2] = o.z;
            }
            base += __shfl_sync(FULL, inc[c], 31);
        }
        carry += sm.out[0];
        __syncthreads();                               // (s_warp and out reused)
    }
    // tile_off was written by this CTA: visible to it after the barrier
    for (uint32_t sl = t; sl < n_slabs; sl += WIN_THREADS)
        slab_off[sl] = tile_off[(uint64_t)sl * tiles_per_slab];
    if (t == 0) {
        tile_off[n_tiles] = (uint32_t)carry;
        slab_off[n_slabs] = (uint32_t)carry;
        if (st) {
            atomicAdd(&st->n_outliers, carry);
            if (carry > cap) atomicOr(&st->flags, HQMQ_FLAG_OUTLIER_OVERFLOW);
        }
    }
}

template <int DT, int GRAN>
__global__ void __launch_bounds__(WIN_THREADS)
k_finalize(const void *__restrict__ x, int B, int H, uint32_t cps, uint32_t tiles_per_slab,
           uint64_t n_tiles, uint64_t n_per_head, float C, WinState *__restrict__ win,
           const unsigned long long *__restrict__ below,
           const unsigned long long *__restrict__ cand_n, const uint32_t *__restrict__ cand,
           uint64_t cand_cap, const unsigned long long *__restrict__ amb_n,
           const uint2 *__restrict__ amb, uint64_t amb_cap, float *__restrict__ rmed,
           float *__restrict__ thr, uint32_t *__restrict__ tile_cnt,
           uint32_t *__restrict__ tile_off, uint32_t *__restrict__ slab_off, uint32_t n_slabs,
           uint64_t cap, uint32_t *__restrict__ med_hist, uint32_t *__restrict__ median_done,
           uint32_t *__restrict__ fin_done, DevStatus *st) {
    __shared__ FinalSmem sm;
    pdl_wait();                                    // (launched with launch_pdl)
    pdl_trigger();
    const int h = blockIdx.y;
    const WinState w = win[h];
    const unsigned long long n_amb = *amb_n;
    const MedianPlan mp = median_plan(h, n_per_head, w, below, cand_n, cand_cap,
                                      n_amb > amb_cap);
    const uint32_t *ch = cand + (uint64_t)h * cand_cap;
    // per head two digit histograms: the top digit's counts of the staged keys
    // were added when they were staged (flush_stage), so the top digit is
    // known here; the MED_SLICES CTAs of the head count the next digit of
    // the keys inside that top bin, each over a slice of the keys
    uint32_t *gh = med_hist + (size_t)h * MED_BINS * 2;
    uint32_t *gh2 = gh + MED_BINS;
    uint32_t prefix = 0, rem = 0;
    if (mp.ok) {                                       // (block-uniform)
        block_select2<MED_BINS, true>(gh, mp.k, mp.k, sm.wtot, sm.out);
        prefix = sm.out[0] << mp.top;
        rem = sm.out[2];
        __syncthreads();                               // (everyone has read out[])
        if (mp.top > 0) {
            for (uint32_t i = threadIdx.x; i < MED_BINS; i += WIN_THREADS) sm.buf[i] = 0;
            __syncthreads();
            const uint64_t i0 = mp.nc * blockIdx.x / gridDim.x;
            const uint64_t i1 = mp.nc * (blockIdx.x + 1) / gridDim.x;
            median_count(ch, i0, i1, w, mp.span, mp.top - 12, prefix, sm.buf);
            __syncthreads();
            for (uint32_t i = threadIdx.x; i < MED_BINS; i += WIN_THREADS)
                if (sm.buf[i]) atomicAdd(gh2 + i, sm.buf[i]);
        }
    }
    // the head's last CTA (no CTA waits for another) finishes the head
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
        sm.last = atomicAdd(median_done + h, 1u) == gridDim.x - 1 ? 1u : 0u;
    __syncthreads();
    if (!sm.last) return;
    __threadfence();
    if (!mp.ok) {
        if (threadIdx.x == 0) win[h].miss = 1;
        exact_fallback<DT, GRAN>(x, B, H, h, cps, tiles_per_slab, n_per_head, C, rmed, thr,
                                 tile_cnt, st, sm);
    } else {
        if (mp.top > 0) {
            block_select2<MED_BINS, true>(gh2, rem, rem, sm.wtot, sm.out);
            prefix |= sm.out[0] << (mp.top - 12);
            rem = sm.out[2];
            __syncthreads();
        }
        // further digits (spans above 2^24 only): this CTA over all keys
        for (int sh = mp.top - 24; sh >= 0; sh -= 12) {
            for (uint32_t i = threadIdx.x; i < MED_BINS; i += WIN_THREADS) sm.buf[i] = 0;
            __syncthreads();
            median_count(ch, 0, mp.nc, w, mp.span, sh, prefix, sm.buf);
            __syncthreads();
            block_select2<MED_BINS, false>(sm.buf, rem, rem, sm.wtot, sm.out);
            prefix |= sm.out[0] << sh;
            rem = sm.out[2];
            __syncthreads();
        }
        const float m = key_to_float(w.lo_key + prefix);
        const float th = __fmul_rn(C, m);
        if (threadIdx.x == 0) { rmed[h] = m; thr[h] = th; }
        // uncertain keys of this head above its exact threshold
        for (uint64_t i = threadIdx.x; i < n_amb; i += WIN_THREADS) {
            const uint2 e = amb[i];
            if ((int)((e.x / tiles_per_slab) % (uint32_t)H) != h) continue;
            if (__uint_as_float(e.y) > th) atomicAdd(tile_cnt + e.x, 1u);
        }
    }
    // the last head to finish scans the tiles
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) sm.last = atomicAdd(fin_done, 1u) == gridDim.y - 1 ? 1u : 0u;
    __syncthreads();
    if (!sm.last) return;
    __threadfence();
    scan_tiles(tile_cnt, n_tiles, tiles_per_slab, n_slabs, cap, tile_off, slab_off, st, sm);
}

// ---------------------------------------------------------------------------
// host: steps A..S (the caller then launches pass C)
// ---------------------------------------------------------------------------
// Memset, A + W and (unless the caller's encode pass does its work) B.
template <int DT, int GRAN>
static int run_front(const void *x, int B, int H, int T, int D, float C, char *ws, bool pass_b,
                     int sm_count, cudaStream_t stream) {
    const FusedLayout L = fused_layout(B, H, T, D, GRAN);
    const SpecArgs a = spec_args(ws, L);
    uint32_t *sample_hist = reinterpret_cast<uint32_t *>(ws + L.sample_hist);
    uint32_t *sample_done = reinterpret_cast<uint32_t *>(ws + L.counters + sizeof(Counters));
    WinState *win = reinterpret_cast<WinState *>(ws + L.win);
    const uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    const int n_slabs = B * H;

    // histograms, counters and per-head status counts
    if (cudaMemsetAsync(ws, 0, L.zero_bytes, stream) != cudaSuccess) return HQMQ_ERR_CUDA;
    // A + W: one wave of CTAs (one per SM: 128 KB of shared counters each)
    const uint32_t n_quads = (cps + SAMPLE_PERIOD - 1) / SAMPLE_PERIOD;
    uint64_t ax = (n_quads + SAMPLE_THREADS - 1) / SAMPLE_THREADS;
    const uint64_t afill = (uint64_t)sm_count / (uint64_t)n_slabs;
    if (ax > afill) ax = afill;
    // 16-bit shared counters: at most 60000 samples per CTA
    const uint64_t keys_per_quad = 4 * (GRAN == HQMQ_GRAN_CHUNK ? 1 : 4);
    const uint64_t ax_min = ((uint64_t)n_quads * keys_per_quad + 59999) / 60000;
    if (ax < ax_min) ax = ax_min;
    if (ax < 1) ax = 1;
    const size_t sample_smem = (size_t)KEY_BINS / 2 * sizeof(uint32_t);
    if (cudaFuncSetAttribute(k_sample_window<DT, GRAN>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sample_smem) != cudaSuccess)
        return HQMQ_ERR_CUDA;
    k_sample_window<DT, GRAN><<<dim3((unsigned)ax, (unsigned)n_slabs), SAMPLE_THREADS,
                                sample_smem, stream>>>(x, H, cps, (uint32_t)(ax * B), L.n_per_head,
                                                       (uint64_t)B * n_quads * keys_per_quad, C,
                                                       sample_hist, sample_done, win, a.below,
                                                       a.cand_n);
    if (pass_b) {
        uint64_t bx = (L.n_tiles + PB_THREADS / 32 - 1) / (PB_THREADS / 32);
        const uint64_t bmax = (uint64_t)sm_count * 8;
        if (bx > bmax) bx = bmax;
        k_pass_b<DT, GRAN><<<(unsigned)bx, PB_THREADS, 0, stream>>>(
            x, H, cps, L.tiles_per_slab, L.n_tiles, win, a.below, a.cand_n, a.cand, a.cand_cap,
            a.amb_n, a.amb, a.amb_cap, a.tile_cnt, a.med_hist);
    }
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

// F + X + U + S; the tile offsets go to tile_off.
template <int DT, int GRAN>
static int run_finish(const void *x, int B, int H, int T, int D, float C, float *rmed, float *thr,
                      uint32_t *slab_off, uint32_t *tile_off, uint64_t cap, char *ws,
                      hqmq_status *st_, int sm_count, cudaStream_t stream) {
    DevStatus *st = reinterpret_cast<DevStatus *>(st_);
    const FusedLayout L = fused_layout(B, H, T, D, GRAN);
    const SpecArgs a = spec_args(ws, L);
    Counters *ctr = reinterpret_cast<Counters *>(ws + L.counters);
    WinState *win = reinterpret_cast<WinState *>(ws + L.win);
    const uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    uint32_t *median_done = reinterpret_cast<uint32_t *>(ws + L.counters + sizeof(Counters)) + H;
    uint32_t *med_hist = reinterpret_cast<uint32_t *>(ws + L.med_hist);
    // slices per head: one per 2^18 keys of the head (the window holds a few
    // percent of them), at most MED_SLICES and about one wave of CTAs in all
    uint64_t slices = L.n_per_head >> 18;
    const uint64_t wave = (uint64_t)sm_count / (uint64_t)(H > 0 ? H : 1);
    if (slices > wave) slices = wave;
    if (slices > (uint64_t)MED_SLICES) slices = MED_SLICES;
    if (slices < 1) slices = 1;
    if (launch_pdl(k_finalize<DT, GRAN>, dim3((unsigned)slices, H), dim3(WIN_THREADS), 0, stream,
                   x, B, H, cps, L.tiles_per_slab, L.n_tiles, L.n_per_head, C, win, a.below,
                   a.cand_n, a.cand, a.cand_cap, a.amb_n, a.amb, a.amb_cap, rmed, thr,
                   a.tile_cnt, tile_off, slab_off, (uint32_t)(B * H), cap, med_hist, median_done,
                   &ctr->fin_done, st) != cudaSuccess)
        return HQMQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

}  // namespace hqmq

extern "C" uint64_t hqmq_window_workspace_bytes(int B, int H, int T, int D, int gran) {
    return hqmq::fused_layout(B, H, T, D, gran).total;
}

// Steps memset, A + W and (if pass_b) B.
extern "C" int hqmq_launch_med3_front(const void *x, int dtype, int B, int H, int T, int D,
                                      float C, int gran, void *ws, int pass_b, int sm_count,
                                      cudaStream_t stream) {
    using namespace hqmq;
    char *w = reinterpret_cast<char *>(ws);
    const bool pb = pass_b != 0;
    if (dtype == HQMQ_BF16)
        return gran == HQMQ_GRAN_CHUNK
                   ? run_front<HQMQ_BF16, HQMQ_GRAN_CHUNK>(x, B, H, T, D, C, w, pb, sm_count, stream)
                   : run_front<HQMQ_BF16, HQMQ_GRAN_ELEMENT>(x, B, H, T, D, C, w, pb, sm_count,
                                                             stream);
    return gran == HQMQ_GRAN_CHUNK
               ? run_front<HQMQ_F32, HQMQ_GRAN_CHUNK>(x, B, H, T, D, C, w, pb, sm_count, stream)
               : run_front<HQMQ_F32, HQMQ_GRAN_ELEMENT>(x, B, H, T, D, C, w, pb, sm_count, stream);
}

// Steps F + X + U + S.  The tile offsets go to tile_off_out (n_tiles + 1
// entries) if given, else into ws; *tile_off returns where they are.
extern "C" int hqmq_launch_med3_finish(const void *x, int dtype, int B, int H, int T, int D,
                                       float C, int gran, float *rmed, float *thr,
                                       uint32_t *slab_off, uint32_t *tile_off_out, uint64_t cap,
                                       void *ws, hqmq_status *st, int sm_count, cudaStream_t stream,
                                       const uint32_t **tile_off, uint32_t *tiles_per_slab) {
    using namespace hqmq;
    const FusedLayout L = fused_layout(B, H, T, D, gran);
    char *w = reinterpret_cast<char *>(ws);
    uint32_t *to = tile_off_out ? tile_off_out : reinterpret_cast<uint32_t *>(w + L.tile_off);
    *tile_off = to;
    *tiles_per_slab = L.tiles_per_slab;
    if (dtype == HQMQ_BF16)
        return gran == HQMQ_GRAN_CHUNK
                   ? run_finish<HQMQ_BF16, HQMQ_GRAN_CHUNK>(x, B, H, T, D, C, rmed, thr, slab_off,
                                                            to, cap, w, st, sm_count, stream)
                   : run_finish<HQMQ_BF16, HQMQ_GRAN_ELEMENT>(x, B, H, T, D, C, rmed, thr,
                                                              slab_off, to, cap, w, st, sm_count, stream);
    return gran == HQMQ_GRAN_CHUNK
               ? run_finish<HQMQ_F32, HQMQ_GRAN_CHUNK>(x, B, H, T, D, C, rmed, thr, slab_off, to,
                                                       cap, w, st, sm_count, stream)
               : run_finish<HQMQ_F32, HQMQ_GRAN_ELEMENT>(x, B, H, T, D, C, rmed, thr, slab_off, to,
                                                         cap, w, st, sm_count, stream);
}

// All steps A..S (two-read path); returns the tile offsets for pass C.
extern "C" int hqmq_launch_med3_window(const void *x, int dtype, int B, int H, int T, int D,
                                       float C, int gran, float *rmed, float *thr,
                                       uint32_t *slab_off, uint32_t *tile_off_out, uint64_t cap,
                                       void *ws, hqmq_status *st, int sm_count,
                                       cudaStream_t stream, const uint32_t **tile_off,
                                       uint32_t *tiles_per_slab) {
    const int rc = hqmq_launch_med3_front(x, dtype, B, H, T, D, C, gran, ws, 1, sm_count, stream);
    if (rc != HQMQ_OK) return rc;
    return hqmq_launch_med3_finish(x, dtype, B, H, T, D, C, gran, rmed, thr, slab_off,
                                   tile_off_out, cap, ws, st, sm_count, stream, tile_off,
                                   tiles_per_slab);
}

extern "C" uint64_t hqmq_list_tile_count(int B, int H, int T, int D) {
    return hqmq::fused_layout(B, H, T, D, HQMQ_GRAN_CHUNK).n_tiles;
}
