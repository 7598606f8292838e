// med3_window.cu -- Med3x in two reads of x.
//
// The rule (gist.science/nl, Technische Samenvatting, section 3; gist.science/
// pt, Resumo Tecnico, section 3): r_med = the median chunk norm over the current
// batch (here: per head over one call, lower median at rank N/2 - 1), outlier
// iff r > fl32(C r_med).  The results are exactly those of the three-pass radix
// select of med3.cu; only the data flow differs:
//
//  A  k_sample_hist    reads a 1/32 sample (4 consecutive chunks of every 128,
//                      the quad's slot rotating through all 32 slots) into a
//                      per-head histogram of the top 16 key bits.
//  W  k_window_select  picks per head a key window [lo, hi) that holds the
//                      sample ranks within +-8 standard deviations of the median
//                      rank; the exact threshold then lies in [t_lo, t_hi].
//  B  k_pass_b         one full read: per head the count of keys below the
//                      window and the keys inside it (list + fine histogram);
//                      per 1024-chunk tile the count of certain outliers
//                      (r > t_hi) and a list of uncertain ones (t_lo < r <= t_hi).
//  F  k_med_final      per head: the exact median from the window keys.
//  X  k_fallback_exact per head whose window missed the median (or whose buffers
//                      overflowed): exact three-pass select over x and exact
//                      tile counts.  Never taken on the bench workloads; it keeps
//                      the result exact for any input.
//  U  k_amb_fixup      adds the uncertain keys that exceed the exact threshold.
//  S  k_tile_scan      tile offsets, per-slab offsets, total, overflow status.
//  C  (search.cu)      the second read writes the ordered list (and encodes).
//
// No kernel waits on another CTA; every step is a separate launch on the
// caller's stream.
#include "med3_window.cuh"

namespace hqmq {

constexpr int WIN_THREADS = 1024;
constexpr int PB_THREADS = 256;
constexpr int FINAL_KEYS = 8192;   // per-key counters of one fine bin (bin width <= 2^13)

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
// A: sample histogram
// ---------------------------------------------------------------------------
constexpr int SAMPLE_THREADS = 1024;

template <int DT, int GRAN>
__global__ void __launch_bounds__(SAMPLE_THREADS)
k_sample_hist(const void *__restrict__ x, int H, uint32_t cps, uint32_t *__restrict__ hist) {
    // per-CTA histogram in shared memory: 65536 16-bit counters packed in
    // pairs (a CTA sees far fewer than 65536 samples), then one global add
    // per non-empty bin
    extern __shared__ uint32_t s_pair[];                       // [KEY_BINS / 2]
    for (int i = threadIdx.x; i < KEY_BINS / 2; i += blockDim.x) s_pair[i] = 0;
    __syncthreads();
    const int slab = blockIdx.y;
    uint32_t *hh = hist + (size_t)(slab % H) * KEY_BINS;
    const uint64_t base = (uint64_t)slab * cps;
    const uint32_t n_quads = (cps + SAMPLE_PERIOD - 1) / SAMPLE_PERIOD;
    for (uint32_t q = blockIdx.x * blockDim.x + threadIdx.x; q < n_quads;
         q += gridDim.x * blockDim.x) {
        // quad slot (37 q) mod 32 of the q-th 128-chunk period: over 32
        // periods every slot is sampled once, whatever the chunks' position
        // inside a head vector
        const uint32_t slot = (37u * q) & 31u;
        uint64_t j0 = base + (uint64_t)q * SAMPLE_PERIOD + 4u * slot;
        if (j0 + 4 > base + cps) j0 = base + (uint64_t)q * SAMPLE_PERIOD;   // short last period
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
}

// Block-wide (1024 threads = 32 warps) search of a histogram of NB bins, warp
// w owning the contiguous bins [w NB/32, (w+1) NB/32), read coalesced:
// rank_bin_totals() stores the warp totals and the totals of every block of
// 32 bins; rank_bin_find() then locates the warp, the block (from the block
// totals) and the bin (one 32-bin read), and returns in s_out[which] the bin
// whose cumulative count first exceeds `rank` and in s_out[which + 2] the
// rank inside that bin.
template <int NB>
__device__ void rank_bin_totals(const uint32_t *hist, uint32_t *s_wtot, uint32_t *s_blk) {
    constexpr int PER = NB / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t acc = 0;
    for (int i = 0; i < PER; i += 32) {
        const uint32_t bt = __reduce_add_sync(FULL, hist[w * PER + i + lane]);
        if (lane == 0) s_blk[(w * PER + i) / 32] = bt;
        acc += bt;
    }
    if (lane == 0) s_wtot[w] = acc;
    __syncthreads();
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(FULL, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

template <int NB>
__device__ void rank_bin_find(const uint32_t *hist, const uint32_t *s_wtot,
                              const uint32_t *s_blk, uint64_t rank, uint32_t *s_out, int which) {
    constexpr int PER = NB / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint64_t cum = 0;
    int ww = 31;
    for (int k = 0; k < 32; ++k) {
        const uint32_t t = s_wtot[k];
        if (rank < cum + t) { ww = k; break; }
        cum += t;
    }
    if (w == ww) {
        uint64_t c = cum;
        int blk = -1;
        for (int i = 0; i < PER / 32; i += 32) {             // block totals of this warp
            const uint32_t v = (i + lane < PER / 32) ? s_blk[ww * (PER / 32) + i + lane] : 0u;
            const uint32_t inc = warp_incl_scan(v, lane);
            const uint32_t tot = __shfl_sync(FULL, inc, 31);
            if (rank < c + tot) {
                const uint32_t bal = __ballot_sync(FULL, rank < c + inc);
                const int src = __ffs(bal) - 1;
                blk = i + src;
                c += __shfl_sync(FULL, inc - v, src);
                break;
            }
            c += tot;
        }
        if (blk >= 0) {                   // (rank below the total, as the callers ensure)
            const uint32_t v = hist[ww * PER + blk * 32 + lane];
            const uint32_t inc = warp_incl_scan(v, lane);
            const bool mine = rank >= c + inc - v && rank < c + inc;
            const uint32_t bal = __ballot_sync(FULL, mine);
            if (lane == __ffs(bal) - 1) {
                s_out[which] = (uint32_t)(ww * PER + blk * 32 + lane);
                s_out[which + 2] = (uint32_t)(rank - (c + inc - v));
            }
        } else if (lane == 0) {
            s_out[which] = NB - 1;
            s_out[which + 2] = 0;
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// W: window per head
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(WIN_THREADS)
k_window_select(uint64_t n_per_head, float C, const uint32_t *__restrict__ sample_hist,
                uint32_t *__restrict__ fine_hist, WinState *__restrict__ win,
                unsigned long long *__restrict__ below, unsigned long long *__restrict__ cand_n) {
    __shared__ uint32_t s_wtot[32];
    __shared__ uint32_t s_blk[KEY_BINS / 32];
    __shared__ uint32_t s_out[4];
    const int h = blockIdx.x;
    const uint32_t *hist = sample_hist + (size_t)h * KEY_BINS;
    uint32_t *fh = fine_hist + (size_t)h * KEY_BINS;
    for (int i = threadIdx.x; i < KEY_BINS; i += WIN_THREADS) fh[i] = 0;
    rank_bin_totals<KEY_BINS>(hist, s_wtot, s_blk);
    uint64_t tot = 0;
    for (int k = 0; k < 32; ++k) tot += s_wtot[k];
    const double ns = (double)tot;
    const double q = ((double)(n_per_head / 2 - 1) + 0.5) / (double)n_per_head;
    const double half = WINDOW_SIGMAS * 0.5 * sqrt(ns) + 4.0;
    double rlo = floor(q * ns - half), rhi = ceil(q * ns + half);
    if (rlo < 0) rlo = 0;
    if (rhi > ns - 1) rhi = ns - 1;
    rank_bin_find<KEY_BINS>(hist, s_wtot, s_blk, (uint64_t)rlo, s_out, 0);
    rank_bin_find<KEY_BINS>(hist, s_wtot, s_blk, (uint64_t)rhi, s_out, 1);
    if (threadIdx.x == 0) {
        WinState w;
        const uint64_t lo = (uint64_t)s_out[0] << 15;
        uint64_t hi = ((uint64_t)s_out[1] + 1) << 15;
        if (hi > 0x80000000ull) hi = 0x80000000ull;
        const uint64_t span = hi - lo;
        uint32_t sh = 0;
        while (((span - 1) >> sh) >= (uint64_t)KEY_BINS) ++sh;
        w.lo_key = (uint32_t)lo;
        w.hi_key = (uint32_t)(hi - 1) + 1u;          // (hi <= 2^31)
        w.shift = sh;
        w.miss = 0;
        w.t_lo = thr_of_key(C, (uint32_t)lo);
        w.t_hi = thr_of_key(C, (uint32_t)(hi - 1));
        w.pad[0] = w.pad[1] = 0;
        win[h] = w;
        below[h] = 0;
        cand_n[h] = 0;
    }
}

// ---------------------------------------------------------------------------
// B: one full read
// ---------------------------------------------------------------------------
constexpr int STAGE = 256;          // window keys staged per warp before one global append

// Appends the warp's staged window keys to the head's buffer (one atomic).
__device__ __forceinline__ void flush_stage(uint32_t *stage, uint32_t n, int lane,
                                            unsigned long long *cand_n_h, uint32_t *cand_h,
                                            uint64_t cand_cap) {
    unsigned long long base = 0;
    if (lane == 0) base = atomicAdd(cand_n_h, (unsigned long long)n);
    base = __shfl_sync(FULL, base, 0);
    for (uint32_t i = lane; i < n; i += 32)
        if (base + i < cand_cap) cand_h[base + i] = stage[i];
    __syncwarp();
}

template <int DT, int GRAN>
__global__ void __launch_bounds__(PB_THREADS)
k_pass_b(const void *__restrict__ x, int H, uint32_t cps, uint32_t tiles_per_slab, uint64_t n_tiles,
         const WinState *__restrict__ win, unsigned long long *__restrict__ below,
         unsigned long long *__restrict__ cand_n, uint32_t *__restrict__ cand, uint64_t cand_cap,
         uint32_t *__restrict__ fine_hist, unsigned long long *__restrict__ amb_n,
         uint2 *__restrict__ amb, uint64_t amb_cap, uint32_t *__restrict__ tile_cnt) {
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
            if (n_stage)
                flush_stage(stage, n_stage, lane, cand_n + stage_h,
                            cand + (uint64_t)stage_h * cand_cap, cand_cap);
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
                                        cand + (uint64_t)h * cand_cap, cand_cap);
                            n_stage = 0;
                        }
                        if (in) {
                            stage[n_stage + __popc(m & lt)] = key;
                            atomicAdd(fine_hist + (size_t)h * KEY_BINS + ((key - w.lo_key) >> w.shift),
                                      1u);
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
    if (n_stage)
        flush_stage(stage, n_stage, lane, cand_n + stage_h, cand + (uint64_t)stage_h * cand_cap,
                    cand_cap);
}

// ---------------------------------------------------------------------------
// F: exact median from the window keys
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(WIN_THREADS)
k_med_final(uint64_t n_per_head, float C, WinState *__restrict__ win,
            const unsigned long long *__restrict__ below,
            const unsigned long long *__restrict__ cand_n, const uint32_t *__restrict__ cand,
            uint64_t cand_cap, const uint32_t *__restrict__ fine_hist,
            const unsigned long long *__restrict__ amb_n, uint64_t amb_cap,
            float *__restrict__ rmed, float *__restrict__ thr) {
    __shared__ uint32_t s_wtot[32];
    __shared__ uint32_t s_blk[KEY_BINS / 32];
    __shared__ uint32_t s_out[4];
    __shared__ uint32_t s_cnt[FINAL_KEYS];             // one counter per key of the bin
    const int h = blockIdx.x;
    const WinState w = win[h];
    const long long k = (long long)(n_per_head / 2 - 1) - (long long)below[h];
    const unsigned long long nc = cand_n[h];
    const bool miss = (*amb_n > amb_cap) || k < 0 || (unsigned long long)k >= nc ||
                      nc > cand_cap || (1u << w.shift) > (uint32_t)FINAL_KEYS;
    if (miss) {                                        // block-uniform
        if (threadIdx.x == 0) win[h].miss = 1;
        return;
    }
    const uint32_t *fh = fine_hist + (size_t)h * KEY_BINS;
    rank_bin_totals<KEY_BINS>(fh, s_wtot, s_blk);
    rank_bin_find<KEY_BINS>(fh, s_wtot, s_blk, (uint64_t)k, s_out, 0);
    const uint32_t bin_lo = w.lo_key + (s_out[0] << w.shift);
    const uint32_t kk = s_out[2];                      // rank inside the fine bin
    const uint32_t width = 1u << w.shift;
    for (uint32_t i = threadIdx.x; i < (uint32_t)FINAL_KEYS; i += WIN_THREADS) s_cnt[i] = 0;
    __syncthreads();
    // count every candidate key of the bin by its exact value (bf16 inputs
    // repeat values, so a bin may hold many equal keys)
    const uint32_t *ch = cand + (uint64_t)h * cand_cap;
    for (uint64_t i = threadIdx.x; i < nc; i += WIN_THREADS) {
        const uint32_t d = ch[i] - bin_lo;
        if (d < width) atomicAdd(&s_cnt[d], 1u);
    }
    __syncthreads();
    rank_bin_totals<FINAL_KEYS>(s_cnt, s_wtot, s_blk);
    rank_bin_find<FINAL_KEYS>(s_cnt, s_wtot, s_blk, kk, s_out, 1);
    if (threadIdx.x == 0) {
        const float m = key_to_float(bin_lo + s_out[1]);
        rmed[h] = m;
        thr[h] = __fmul_rn(C, m);
    }
}

// ---------------------------------------------------------------------------
// X: exact fallback for heads whose window missed (one CTA per head)
// ---------------------------------------------------------------------------
template <int DT, int GRAN>
__global__ void __launch_bounds__(WIN_THREADS)
k_fallback_exact(const void *__restrict__ x, int B, int H, uint32_t cps, uint32_t tiles_per_slab,
                 uint64_t n_per_head, float C, const WinState *__restrict__ win,
                 float *__restrict__ rmed, float *__restrict__ thr, uint32_t *__restrict__ tile_cnt,
                 DevStatus *st) {
    constexpr int NK = GRAN == HQMQ_GRAN_CHUNK ? 1 : 4;
    __shared__ uint32_t s_hist[2048];
    __shared__ uint32_t s_warp[32];
    __shared__ uint32_t s_out[4];
    const int h = blockIdx.x;
    if (!win[h].miss) return;                              // the common case
    if (threadIdx.x == 0 && st) atomicOr(&st->flags, HQMQ_FLAG_MED3_FALLBACK);
    uint32_t prefix = 0;
    uint64_t krem = n_per_head / 2 - 1;
    const int shifts[3] = {20, 9, 0};
    const int widths[3] = {11, 11, 9};
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
        // 2048 bins: threads 0..1023 own 2 bins each; reuse the 64-bin finder
        // through a padded copy is unnecessary: scan directly
        uint32_t b0 = s_hist[2 * threadIdx.x], b1 = s_hist[2 * threadIdx.x + 1];
        uint32_t local = b0 + b1, inc = local;
        const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t v = __shfl_up_sync(FULL, inc, o);
            if (lane >= o) inc += v;
        }
        if (lane == 31) s_warp[wid] = inc;
        __syncthreads();
        if (wid == 0) {
            uint32_t wv = s_warp[lane], wi = wv;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint32_t v = __shfl_up_sync(FULL, wi, o);
                if (lane >= o) wi += v;
            }
            s_warp[lane] = wi - wv;
        }
        __syncthreads();
        const uint64_t excl = (uint64_t)s_warp[wid] + inc - local;
        if (krem >= excl && krem < excl + local) {
            const uint32_t digit = krem < excl + b0 ? 2 * threadIdx.x : 2 * threadIdx.x + 1;
            s_out[0] = digit;
            s_out[1] = (uint32_t)(krem - (krem < excl + b0 ? excl : excl + b0));
        }
        __syncthreads();
        prefix |= s_out[0] << sh;
        krem = s_out[1];
        __syncthreads();
    }
    const float m = key_to_float(prefix);
    const float th = __fmul_rn(C, m);
    if (threadIdx.x == 0) { rmed[h] = m; thr[h] = th; }
    // exact tile counts of this head's slabs
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
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

// ---------------------------------------------------------------------------
// U: uncertain keys above the exact threshold
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
k_amb_fixup(int H, uint32_t tiles_per_slab, const WinState *__restrict__ win,
            const float *__restrict__ thr, const unsigned long long *__restrict__ amb_n,
            const uint2 *__restrict__ amb, uint64_t amb_cap, uint32_t *__restrict__ tile_cnt) {
    uint64_t n = *amb_n;
    if (n > amb_cap) return;                 // every head then took the fallback
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (uint64_t)gridDim.x * blockDim.x) {
        const uint2 e = amb[i];
        const int h = (int)((e.x / tiles_per_slab) % (uint32_t)H);
        if (win[h].miss) continue;           // recounted exactly by the fallback
        if (__uint_as_float(e.y) > thr[h]) atomicAdd(tile_cnt + e.x, 1u);
    }
}

// ---------------------------------------------------------------------------
// S: tile offsets (one CTA; each thread scans a contiguous run of tiles)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
k_tile_scan(const uint32_t *__restrict__ tile_cnt, uint64_t n_tiles, uint32_t tiles_per_slab,
            uint32_t n_slabs, uint64_t cap, uint32_t *__restrict__ tile_off,
            uint32_t *__restrict__ slab_off, DevStatus *st) {
    __shared__ unsigned long long s_warp[32];
    __shared__ unsigned long long s_carry;
    const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
    if (t == 0) s_carry = 0;
    __syncthreads();
    // blocks of 16384 tiles: thread t scans tiles 16t .. 16t+15 of the block
    constexpr int PT = 16;
    for (uint64_t b0 = 0; b0 < n_tiles; b0 += 1024 * PT) {
        uint32_t v[PT];
        const uint64_t first = b0 + (uint64_t)PT * t;
        if (first + PT <= n_tiles) {
            const uint4 *p4 = reinterpret_cast<const uint4 *>(tile_cnt + first);
#pragma unroll
            for (int q = 0; q < PT / 4; ++q) {
                const uint4 u = p4[q];
                v[4 * q] = u.x; v[4 * q + 1] = u.y; v[4 * q + 2] = u.z; v[4 * q + 3] = u.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < PT; ++k) v[k] = first + k < n_tiles ? tile_cnt[first + k] : 0u;
        }
        unsigned long long local = 0;
#pragma unroll
        for (int k = 0; k < PT; ++k) local += v[k];
        unsigned long long inc = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long u = __shfl_up_sync(FULL, inc, o);
            if (lane >= o) inc += u;
        }
        if (lane == 31) s_warp[wid] = inc;
        __syncthreads();
        if (wid == 0) {
            const unsigned long long wv = s_warp[lane];
            unsigned long long wi = wv;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long u = __shfl_up_sync(FULL, wi, o);
                if (lane >= o) wi += u;
            }
            s_warp[lane] = wi - wv;
        }
        __syncthreads();
        unsigned long long run = s_carry + s_warp[wid] + inc - local;
#pragma unroll
        for (int k = 0; k < PT; ++k) {
            const uint64_t i = first + k;
            if (i < n_tiles) {
                tile_off[i] = (uint32_t)run;
                if (i % tiles_per_slab == 0) slab_off[i / tiles_per_slab] = (uint32_t)run;
            }
            run += v[k];
        }
        __syncthreads();
        if (t == 1023) s_carry = run;
        __syncthreads();
    }
    if (t == 0) {
        const unsigned long long total = s_carry;
        slab_off[n_slabs] = (uint32_t)total;
        if (st) {
            atomicAdd(&st->n_outliers, total);
            if (total > cap) atomicOr(&st->flags, HQMQ_FLAG_OUTLIER_OVERFLOW);
        }
    }
}

// ---------------------------------------------------------------------------
// host: steps A..S (the caller then launches pass C)
// ---------------------------------------------------------------------------
template <int DT, int GRAN>
static int run_window(const void *x, int B, int H, int T, int D, float C, float *rmed, float *thr,
                      uint32_t *slab_off, uint64_t cap, char *ws, hqmq_status *st_,
                      int sm_count, cudaStream_t stream) {
    DevStatus *st = reinterpret_cast<DevStatus *>(st_);
    const FusedLayout L = fused_layout(B, H, T, D, GRAN);
    uint32_t *sample_hist = reinterpret_cast<uint32_t *>(ws + L.sample_hist);
    uint32_t *fine_hist = reinterpret_cast<uint32_t *>(ws + L.fine_hist);
    WinState *win = reinterpret_cast<WinState *>(ws + L.win);
    unsigned long long *below = reinterpret_cast<unsigned long long *>(ws + L.below);
    unsigned long long *cand_n = reinterpret_cast<unsigned long long *>(ws + L.cand_n);
    unsigned long long *amb_n = reinterpret_cast<unsigned long long *>(ws + L.amb_n);
    uint32_t *cand = reinterpret_cast<uint32_t *>(ws + L.cand);
    uint2 *amb = reinterpret_cast<uint2 *>(ws + L.amb);
    uint32_t *tile_cnt = reinterpret_cast<uint32_t *>(ws + L.tile_cnt);
    uint32_t *tile_off = reinterpret_cast<uint32_t *>(ws + L.tile_off);
    const uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    const int n_slabs = B * H;

    if (cudaMemsetAsync(sample_hist, 0, (size_t)H * KEY_BINS * 4, stream) != cudaSuccess ||
        cudaMemsetAsync(amb_n, 0, 8, stream) != cudaSuccess)
        return HQMQ_ERR_CUDA;
    const uint32_t n_quads = (cps + SAMPLE_PERIOD - 1) / SAMPLE_PERIOD;
    uint64_t ax = (n_quads + SAMPLE_THREADS - 1) / SAMPLE_THREADS;
    const uint64_t afill = ((uint64_t)sm_count + n_slabs - 1) / n_slabs;
    if (ax > afill) ax = afill;
    // 16-bit shared counters: at most 60000 samples per CTA
    const uint64_t keys_per_quad = 4 * (GRAN == HQMQ_GRAN_CHUNK ? 1 : 4);
    const uint64_t ax_min = ((uint64_t)n_quads * keys_per_quad + 59999) / 60000;
    if (ax < ax_min) ax = ax_min;
    if (ax < 1) ax = 1;
    const size_t sample_smem = (size_t)KEY_BINS / 2 * sizeof(uint32_t);
    if (cudaFuncSetAttribute(k_sample_hist<DT, GRAN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sample_smem) != cudaSuccess)
        return HQMQ_ERR_CUDA;
    k_sample_hist<DT, GRAN><<<dim3((unsigned)ax, (unsigned)n_slabs), SAMPLE_THREADS, sample_smem,
                              stream>>>(
        x, H, cps, sample_hist);
    k_window_select<<<H, WIN_THREADS, 0, stream>>>(L.n_per_head, C, sample_hist, fine_hist, win,
                                                   below, cand_n);
    uint64_t bx = (L.n_tiles + PB_THREADS / 32 - 1) / (PB_THREADS / 32);
    const uint64_t bmax = (uint64_t)sm_count * 8;
    if (bx > bmax) bx = bmax;
    k_pass_b<DT, GRAN><<<(unsigned)bx, PB_THREADS, 0, stream>>>(
        x, H, cps, L.tiles_per_slab, L.n_tiles, win, below, cand_n, cand, L.cand_cap, fine_hist,
        amb_n, amb, L.amb_cap, tile_cnt);
    k_med_final<<<H, WIN_THREADS, 0, stream>>>(L.n_per_head, C, win, below, cand_n, cand,
                                               L.cand_cap, fine_hist, amb_n, L.amb_cap, rmed, thr);
    k_fallback_exact<DT, GRAN><<<H, WIN_THREADS, 0, stream>>>(
        x, B, H, cps, L.tiles_per_slab, L.n_per_head, C, win, rmed, thr, tile_cnt, st);
    const uint64_t ux = (uint64_t)sm_count * 2;
    k_amb_fixup<<<(unsigned)ux, 256, 0, stream>>>(H, L.tiles_per_slab, win, thr, amb_n, amb,
                                                  L.amb_cap, tile_cnt);
    k_tile_scan<<<1, 1024, 0, stream>>>(tile_cnt, L.n_tiles, L.tiles_per_slab, (uint32_t)n_slabs,
                                        cap, tile_off, slab_off, st);
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

}  // namespace hqmq

extern "C" uint64_t hqmq_window_workspace_bytes(int B, int H, int T, int D, int gran) {
    return hqmq::fused_layout(B, H, T, D, gran).total;
}

// Steps A..S; returns the tile offsets (inside ws) for pass C.
extern "C" int hqmq_launch_med3_window(const void *x, int dtype, int B, int H, int T, int D,
                                       float C, int gran, float *rmed, float *thr,
                                       uint32_t *slab_off, uint64_t cap, void *ws,
                                       hqmq_status *st, int sm_count, cudaStream_t stream,
                                       const uint32_t **tile_off, uint32_t *tiles_per_slab) {
    using namespace hqmq;
    const FusedLayout L = fused_layout(B, H, T, D, gran);
    char *w = reinterpret_cast<char *>(ws);
    *tile_off = reinterpret_cast<const uint32_t *>(w + L.tile_off);
    *tiles_per_slab = L.tiles_per_slab;
    if (dtype == HQMQ_BF16) {
        if (gran == HQMQ_GRAN_CHUNK)
            return run_window<HQMQ_BF16, HQMQ_GRAN_CHUNK>(x, B, H, T, D, C, rmed, thr, slab_off,
                                                          cap, w, st, sm_count, stream);
        return run_window<HQMQ_BF16, HQMQ_GRAN_ELEMENT>(x, B, H, T, D, C, rmed, thr, slab_off, cap,
                                                        w, st, sm_count, stream);
    }
    if (gran == HQMQ_GRAN_CHUNK)
        return run_window<HQMQ_F32, HQMQ_GRAN_CHUNK>(x, B, H, T, D, C, rmed, thr, slab_off, cap, w,
                                                     st, sm_count, stream);
    return run_window<HQMQ_F32, HQMQ_GRAN_ELEMENT>(x, B, H, T, D, C, rmed, thr, slab_off, cap, w,
                                                   st, sm_count, stream);
}
