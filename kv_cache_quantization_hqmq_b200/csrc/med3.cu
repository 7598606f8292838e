// med3.cu -- Med3x: per-head median chunk norm, threshold, ordered outlier list.
//
// gist.science/nl, Technische Samenvatting, section 3 (and gist.science/pt,
// Resumo Tecnico, section 3): take the median chunk norm r_med of the current
// batch; chunks with r > C r_med (C = 3) are stored in full fp16 with a flag
// and the remaining bulk is quantised.  Here the batch is one call (one
// (layer, role) tensor) and the median is taken per head over all its batches
// and tokens; the lower median (rank N/2 - 1) is used for even N.
//
// Exact selection by radix select on the order-preserving bit pattern of the
// non-negative fp32 magnitudes (31 significant bits; NaN -> 0x7FFFFFFF):
// three histogram passes over the input with digits of 11, 11 and 9 bits,
// each followed by a one-CTA-per-head select that narrows the prefix and the
// remaining rank.  No kernel waits on another CTA: passes are separate
// launches on the caller's stream.
//
// The ordered list is written by a count pass (outliers per tile), a scan of
// the tile counts (tile and slab offsets, total, overflow) and a write pass
// that ranks the outliers inside each tile with a block-wide scan.
#include "hqmq_device.cuh"

namespace hqmq {

constexpr int HIST_BINS = 2048;
constexpr int MED_THREADS = 256;
constexpr int MED_UNROLL = 4;        // chunks in flight per thread
constexpr int TILE = 4096;           // chunks per extraction tile
constexpr int LIST_TILE = 1024;      // chunks per list tile (the tile offsets callers get)
constexpr int EXT_THREADS = 256;
constexpr int EXT_ROWS = 8;          // rows of EXT_THREADS chunks loaded at once (count)
constexpr int WR_ROWS = 4;           // the same for the ordered write

struct SelState {
    uint32_t prefix;   // key bits fixed so far
    uint32_t krem;     // rank still to find among keys with that prefix
};

// Digit of pass P: bits [shift, shift + width) of the 31-bit key.
__host__ __device__ constexpr int pass_shift(int P) { return P == 0 ? 20 : (P == 1 ? 9 : 0); }
__host__ __device__ constexpr int pass_width(int P) { return P == 2 ? 9 : 11; }

template <int DT, int GRAN, int P>
__global__ void __launch_bounds__(MED_THREADS)
k_med_hist(const void *__restrict__ x, int H, uint32_t chunks_per_slab,
           const SelState *__restrict__ state, uint32_t *__restrict__ hist) {
    __shared__ uint32_t s_hist[HIST_BINS];
    for (int i = threadIdx.x; i < HIST_BINS; i += MED_THREADS) s_hist[i] = 0;
    __syncthreads();
    const int slab = blockIdx.y;
    const int h = slab % H;
    constexpr int shift = pass_shift(P);
    constexpr uint32_t mask = (1u << pass_width(P)) - 1u;
    constexpr int hi_shift = shift + pass_width(P);      // bits above the digit
    const uint32_t want = P == 0 ? 0u : (state[h].prefix >> hi_shift);
    const uint64_t base = (uint64_t)slab * chunks_per_slab;
    const uint32_t stride = gridDim.x * MED_THREADS;
    for (uint32_t c0 = blockIdx.x * MED_THREADS + threadIdx.x; c0 < chunks_per_slab;
         c0 += MED_UNROLL * stride) {
        RawChunk<DT> raw[MED_UNROLL];
#pragma unroll
        for (int u = 0; u < MED_UNROLL; ++u) {       // all loads first
            const uint32_t c = c0 + u * stride;
            raw[u].zero();
            if (c < chunks_per_slab) raw[u].load(x, base + c);
        }
        float v[MED_UNROLL][4];
#pragma unroll
        for (int u = 0; u < MED_UNROLL; ++u)
#pragma unroll
            for (int i = 0; i < 4; ++i) v[u][i] = raw[u].e(i);
#pragma unroll
        for (int u = 0; u < MED_UNROLL; ++u) {
            if (c0 + u * stride >= chunks_per_slab) break;
            if (GRAN == HQMQ_GRAN_CHUNK) {
                uint32_t key = mag_key(chunk_norm(v[u][0], v[u][1], v[u][2], v[u][3]));
                if (P == 0 || (key >> hi_shift) == want)
                    atomicAdd(&s_hist[(key >> shift) & mask], 1u);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t key = mag_key(fabsf(v[u][i]));
                    if (P == 0 || (key >> hi_shift) == want)
                        atomicAdd(&s_hist[(key >> shift) & mask], 1u);
                }
            }
        }
    }
    __syncthreads();
    uint32_t *gh = hist + (size_t)h * HIST_BINS;
    for (int i = threadIdx.x; i < HIST_BINS; i += MED_THREADS)
        if (s_hist[i]) atomicAdd(gh + i, s_hist[i]);
}

// One CTA (1024 threads, 2 bins each) per head: find the digit holding rank
// krem, fix it into the prefix, reduce the rank, clear the histogram.  The
// last pass turns the prefix into r_med and thr = fl32(C * r_med).
template <int P>
__global__ void __launch_bounds__(1024)
k_med_select(uint64_t n_per_head, float C, SelState *__restrict__ state,
             uint32_t *__restrict__ hist, float *__restrict__ rmed, float *__restrict__ thr) {
    __shared__ uint32_t s_warp[32];
    const int h = blockIdx.x;
    uint32_t *gh = hist + (size_t)h * HIST_BINS;
    SelState stt;
    if (P == 0) { stt.prefix = 0; stt.krem = (uint32_t)(n_per_head / 2 - 1); }
    else stt = state[h];
    const int t = threadIdx.x;
    const uint32_t b0 = gh[2 * t], b1 = gh[2 * t + 1];
    const uint32_t local = b0 + b1;
    // block exclusive scan of `local`
    const int lane = t & 31, wid = t >> 5;
    uint32_t inc = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t v = __shfl_up_sync(FULL, inc, o);
        if (lane >= o) inc += v;
    }
    if (lane == 31) s_warp[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        uint32_t w = s_warp[lane];
        uint32_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t v = __shfl_up_sync(FULL, wi, o);
            if (lane >= o) wi += v;
        }
        s_warp[lane] = wi - w;   // exclusive warp offsets
    }
    __syncthreads();
    const uint32_t excl = s_warp[wid] + inc - local;
    gh[2 * t] = 0;
    gh[2 * t + 1] = 0;
    const uint32_t k = stt.krem;
    if (k >= excl && k < excl + local) {
        uint32_t digit, below;
        if (k < excl + b0) { digit = 2 * t; below = excl; }
        else { digit = 2 * t + 1; below = excl + b0; }
        SelState ns;
        ns.prefix = stt.prefix | (digit << pass_shift(P));
        ns.krem = k - below;
        state[h] = ns;
        if (P == 2) {
            float m = ns.prefix == 0x7FFFFFFFu ? __int_as_float(0x7FC00000) : __uint_as_float(ns.prefix);
            rmed[h] = m;
            thr[h] = __fmul_rn(C, m);
        }
    }
}

// Outliers of one chunk: chunk mode 0/1, element mode a 4-bit mask.
template <int GRAN>
__device__ __forceinline__ uint32_t outlier_mask(float x0, float x1, float x2, float x3, float th) {
    if (GRAN == HQMQ_GRAN_CHUNK) return chunk_norm(x0, x1, x2, x3) > th ? 1u : 0u;
    return (fabsf(x0) > th ? 1u : 0u) | (fabsf(x1) > th ? 2u : 0u) | (fabsf(x2) > th ? 4u : 0u) |
           (fabsf(x3) > th ? 8u : 0u);
}

template <int DT, int GRAN, int TL = TILE>
__global__ void __launch_bounds__(EXT_THREADS)
k_extract_count(const void *__restrict__ x, int H, uint32_t chunks_per_slab,
                uint32_t tiles_per_slab, const float *__restrict__ thr,
                uint32_t *__restrict__ tile_count) {
    __shared__ uint32_t s_red[EXT_THREADS / 32];
    const int slab = blockIdx.y;
    const float th = thr[slab % H];
    const uint32_t c0 = blockIdx.x * TL;
    const uint32_t c1 = min(c0 + TL, chunks_per_slab);
    const uint64_t base = (uint64_t)slab * chunks_per_slab;
    uint32_t cnt = 0;
    for (uint32_t cb = c0 + threadIdx.x; cb < c1; cb += EXT_ROWS * EXT_THREADS) {
        RawChunk<DT> v[EXT_ROWS];
#pragma unroll
        for (int u = 0; u < EXT_ROWS; ++u) {
            const uint32_t c = cb + u * EXT_THREADS;
            v[u].zero();
            if (c < c1) v[u].load(x, base + c);
        }
#pragma unroll
        for (int u = 0; u < EXT_ROWS; ++u)
            if (cb + u * EXT_THREADS < c1)
                cnt += __popc(outlier_mask<GRAN>(v[u].e(0), v[u].e(1), v[u].e(2), v[u].e(3), th));
    }
    cnt = __reduce_add_sync(FULL, cnt);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t s = 0;
        for (int i = 0; i < EXT_THREADS / 32; ++i) s += s_red[i];
        tile_count[(uint64_t)slab * tiles_per_slab + blockIdx.x] = s;
    }
}

// Exclusive scan of all tile counts (one CTA of 1024 threads, sequential
// blocks of 1024 with a running carry in 64 bits).
__global__ void __launch_bounds__(1024)
k_extract_scan(const uint32_t *__restrict__ tile_count, uint64_t n_tiles,
               uint32_t tiles_per_slab, uint32_t n_slabs, uint64_t cap,
               uint32_t *__restrict__ tile_off, uint32_t *__restrict__ slab_off, DevStatus *st,
               bool write_total = false) {
    __shared__ uint32_t s_warp[32];
    __shared__ unsigned long long s_carry;
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (uint64_t b0 = 0; b0 < n_tiles; b0 += 1024) {
        uint64_t i = b0 + threadIdx.x;
        uint32_t v = i < n_tiles ? tile_count[i] : 0u;
        uint32_t inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t u = __shfl_up_sync(FULL, inc, o);
            if (lane >= o) inc += u;
        }
        if (lane == 31) s_warp[wid] = inc;
        __syncthreads();
        if (wid == 0) {
            uint32_t w = s_warp[lane], wi = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint32_t u = __shfl_up_sync(FULL, wi, o);
                if (lane >= o) wi += u;
            }
            s_warp[lane] = wi - w;
        }
        __syncthreads();
        unsigned long long carry = s_carry;
        unsigned long long excl = carry + s_warp[wid] + inc - v;
        if (i < n_tiles) {
            tile_off[i] = (uint32_t)excl;
            if (i % tiles_per_slab == 0) slab_off[i / tiles_per_slab] = (uint32_t)excl;
        }
        __syncthreads();
        if (threadIdx.x == 1023) s_carry = excl + v;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        unsigned long long total = s_carry;
        slab_off[n_slabs] = (uint32_t)total;
        if (write_total) tile_off[n_tiles] = (uint32_t)total;
        if (st) {
            atomicAdd(&st->n_outliers, total);
            if (total > cap) atomicOr(&st->flags, HQMQ_FLAG_OUTLIER_OVERFLOW);
        }
    }
}

template <int DT, int GRAN, int TL = TILE>
__global__ void __launch_bounds__(EXT_THREADS)
k_extract_write(const void *__restrict__ x, int H, uint32_t chunks_per_slab,
                uint32_t tiles_per_slab, const float *__restrict__ thr,
                const uint32_t *__restrict__ tile_off, uint64_t cap,
                uint32_t *__restrict__ out_idx, uint16_t *__restrict__ out_val, DevStatus *st) {
    constexpr int NW = EXT_THREADS / 32;
    __shared__ uint32_t s_tot[WR_ROWS][NW];
    const int slab = blockIdx.y;
    const float th = thr[slab % H];
    const uint32_t c0 = blockIdx.x * TL;
    const uint32_t c1 = min(c0 + TL, chunks_per_slab);
    const uint64_t base = (uint64_t)slab * chunks_per_slab;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint64_t pos = tile_off[(uint64_t)slab * tiles_per_slab + blockIdx.x];
    unsigned n_sat = 0;
    // WR_ROWS rows of EXT_THREADS chunks per batch: row u, thread t holds
    // chunk cb + u*EXT_THREADS + t, so list order = (row, warp, lane) order
    for (uint32_t cb = c0; cb < c1; cb += WR_ROWS * EXT_THREADS) {
        RawChunk<DT> v[WR_ROWS];
        uint32_t m[WR_ROWS], incl[WR_ROWS];
#pragma unroll
        for (int u = 0; u < WR_ROWS; ++u) {
            const uint32_t c = cb + u * EXT_THREADS + threadIdx.x;
            v[u].zero();
            if (c < c1) v[u].load(x, base + c);
        }
#pragma unroll
        for (int u = 0; u < WR_ROWS; ++u) {
            const uint32_t c = cb + u * EXT_THREADS + threadIdx.x;
            m[u] = c < c1 ? outlier_mask<GRAN>(v[u].e(0), v[u].e(1), v[u].e(2), v[u].e(3), th)
                          : 0u;
            uint32_t inc = __popc(m[u]);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint32_t t = __shfl_up_sync(FULL, inc, o);
                if (lane >= o) inc += t;
            }
            incl[u] = inc;
            if (lane == 31) s_tot[u][wid] = inc;
        }
        __syncthreads();
        uint32_t run = 0;          // outliers of this batch before (row u, warp wid)
        uint32_t batch_total = 0;
#pragma unroll
        for (int u = 0; u < WR_ROWS; ++u)
#pragma unroll
            for (int w = 0; w < NW; ++w) batch_total += s_tot[u][w];
#pragma unroll
        for (int u = 0; u < WR_ROWS; ++u) {
            uint32_t before = run;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                uint32_t t = s_tot[u][w];
                before += w < wid ? t : 0u;
                run += t;
            }
            if (m[u]) {
                uint64_t p = pos + before + incl[u] - __popc(m[u]);
                const uint64_t j = base + cb + u * EXT_THREADS + threadIdx.x;
                if (GRAN == HQMQ_GRAN_CHUNK) {
                    if (p < cap) {
                        int s0 = 0, s1 = 0, s2 = 0, s3 = 0;
                        uint32_t h0 = f32_to_f16_sat(v[u].e(0), s0), h1 = f32_to_f16_sat(v[u].e(1), s1);
                        uint32_t h2 = f32_to_f16_sat(v[u].e(2), s2), h3 = f32_to_f16_sat(v[u].e(3), s3);
                        n_sat += s0 + s1 + s2 + s3;
                        out_idx[p] = (uint32_t)j;
                        uint32_t *vv = reinterpret_cast<uint32_t *>(out_val + p * 4);
                        vv[0] = h0 | (h1 << 16);
                        vv[1] = h2 | (h3 << 16);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (m[u] & (1u << i)) {
                            if (p < cap) {
                                int sv = 0;
                                out_val[p] = f32_to_f16_sat(v[u].e(i), sv);
                                n_sat += sv;
                                out_idx[p] = (uint32_t)(j * 4 + i);
                            }
                            ++p;
                        }
                    }
                }
            }
        }
        pos += batch_total;
        __syncthreads();   // s_tot reuse
    }
    unsigned ns = __reduce_add_sync(FULL, n_sat);
    if (lane == 0 && ns && st) status_add(st, HQMQ_FLAG_SATURATED, &st->n_saturated, ns);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static inline uint64_t align256(uint64_t v) { return (v + 255) & ~(uint64_t)255; }

struct WsLayout {
    uint64_t hist, state, tile_count, tile_off, total;
    uint32_t tiles_per_slab;
    uint64_t n_tiles;
};

static WsLayout ws_layout(int B, int H, int T, int D) {
    WsLayout L;
    uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    L.tiles_per_slab = (cps + TILE - 1) / TILE;
    L.n_tiles = (uint64_t)B * H * L.tiles_per_slab;
    uint64_t off = 0;
    L.hist = off; off = align256(off + (uint64_t)H * HIST_BINS * 4);
    L.state = off; off = align256(off + (uint64_t)H * sizeof(SelState));
    L.tile_count = off; off = align256(off + L.n_tiles * 4);
    L.tile_off = off; off = align256(off + L.n_tiles * 4);
    L.total = off;
    return L;
}

template <int DT, int GRAN>
static int run(const void *x, int B, int H, int T, int D, float C, float *rmed, float *thr,
               uint32_t *out_idx, uint16_t *out_val, uint32_t *slab_off, uint64_t cap, char *ws,
               hqmq_status *st_, int sm_count, cudaStream_t stream) {
    DevStatus *st = reinterpret_cast<DevStatus *>(st_);
    WsLayout L = ws_layout(B, H, T, D);
    uint32_t *hist = reinterpret_cast<uint32_t *>(ws + L.hist);
    SelState *state = reinterpret_cast<SelState *>(ws + L.state);
    uint32_t *tile_count = reinterpret_cast<uint32_t *>(ws + L.tile_count);
    uint32_t *tile_off = reinterpret_cast<uint32_t *>(ws + L.tile_off);
    const uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    const int n_slabs = B * H;
    const uint64_t n_per_head = (uint64_t)B * cps * (GRAN == HQMQ_GRAN_CHUNK ? 1 : 4);

    if (cudaMemsetAsync(hist, 0, (size_t)H * HIST_BINS * 4, stream) != cudaSuccess)
        return HQMQ_ERR_CUDA;
    // histogram grid: about 8 CTAs per SM in total, split over the slabs
    uint64_t per_slab_ctas = ((uint64_t)cps + MED_THREADS * 8 - 1) / (MED_THREADS * 8);
    uint64_t fill = ((uint64_t)sm_count * 8 + n_slabs - 1) / n_slabs;
    uint64_t gx = per_slab_ctas < fill ? per_slab_ctas : fill;
    if (gx < 1) gx = 1;
    dim3 hgrid((unsigned)gx, (unsigned)n_slabs);
    k_med_hist<DT, GRAN, 0><<<hgrid, MED_THREADS, 0, stream>>>(x, H, cps, state, hist);
    k_med_select<0><<<H, 1024, 0, stream>>>(n_per_head, C, state, hist, rmed, thr);
    k_med_hist<DT, GRAN, 1><<<hgrid, MED_THREADS, 0, stream>>>(x, H, cps, state, hist);
    k_med_select<1><<<H, 1024, 0, stream>>>(n_per_head, C, state, hist, rmed, thr);
    k_med_hist<DT, GRAN, 2><<<hgrid, MED_THREADS, 0, stream>>>(x, H, cps, state, hist);
    k_med_select<2><<<H, 1024, 0, stream>>>(n_per_head, C, state, hist, rmed, thr);
    dim3 tgrid(L.tiles_per_slab, (unsigned)n_slabs);
    k_extract_count<DT, GRAN><<<tgrid, EXT_THREADS, 0, stream>>>(x, H, cps, L.tiles_per_slab, thr,
                                                                 tile_count);
    k_extract_scan<<<1, 1024, 0, stream>>>(tile_count, L.n_tiles, L.tiles_per_slab,
                                           (uint32_t)n_slabs, cap, tile_off, slab_off, st);
    k_extract_write<DT, GRAN><<<tgrid, EXT_THREADS, 0, stream>>>(x, H, cps, L.tiles_per_slab, thr,
                                                                 tile_off, cap, out_idx, out_val,
                                                                 st);
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

// The list of a call under a given per-head threshold (no median): count
// per 1024-chunk list tile, scan, ordered write.  tile_off_out (NULL: kept
// in the workspace) receives the list tile offsets and the total.
inline uint64_t thr_ws_bytes(int B, int H, int T, int D, uint64_t *n_tiles_out) {
    const uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    const uint64_t n_tiles = (uint64_t)B * H * ((cps + LIST_TILE - 1) / LIST_TILE);
    if (n_tiles_out) *n_tiles_out = n_tiles;
    return align256(n_tiles * 4) + align256((n_tiles + 1) * 4);
}

template <int DT, int GRAN>
static int run_thr(const void *x, int B, int H, int T, int D, const float *thr, uint32_t *out_idx,
                   uint16_t *out_val, uint32_t *slab_off, uint32_t *tile_off_out, uint64_t cap,
                   char *ws, hqmq_status *st_, cudaStream_t stream) {
    DevStatus *st = reinterpret_cast<DevStatus *>(st_);
    uint64_t n_tiles = 0;
    thr_ws_bytes(B, H, T, D, &n_tiles);
    const uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    const uint32_t tps = (cps + LIST_TILE - 1) / LIST_TILE;
    uint32_t *tile_count = reinterpret_cast<uint32_t *>(ws);
    uint32_t *tile_off = tile_off_out ? tile_off_out
                                      : reinterpret_cast<uint32_t *>(ws + align256(n_tiles * 4));
    const int n_slabs = B * H;
    dim3 tgrid(tps, (unsigned)n_slabs);
    k_extract_count<DT, GRAN, LIST_TILE><<<tgrid, EXT_THREADS, 0, stream>>>(x, H, cps, tps, thr,
                                                                              tile_count);
    k_extract_scan<<<1, 1024, 0, stream>>>(tile_count, n_tiles, tps, (uint32_t)n_slabs, cap,
                                           tile_off, slab_off, st, true);
    k_extract_write<DT, GRAN, LIST_TILE><<<tgrid, EXT_THREADS, 0, stream>>>(
        x, H, cps, tps, thr, tile_off, cap, out_idx, out_val, st);
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

}  // namespace hqmq

extern "C" uint64_t hqmq_thr_extract_workspace_bytes(int B, int H, int T, int D) {
    return hqmq::thr_ws_bytes(B, H, T, D, nullptr);
}

extern "C" int hqmq_launch_outlier_extract_thr(const void *x, int dtype, int B, int H, int T, int D,
                                               const float *thr, int gran, uint32_t *out_idx,
                                               uint16_t *out_val, uint32_t *slab_off,
                                               uint32_t *tile_off, uint64_t cap, void *ws,
                                               hqmq_status *st, cudaStream_t stream) {
    using namespace hqmq;
    char *w = reinterpret_cast<char *>(ws);
    if (dtype == HQMQ_BF16) {
        if (gran == HQMQ_GRAN_CHUNK)
            return run_thr<HQMQ_BF16, HQMQ_GRAN_CHUNK>(x, B, H, T, D, thr, out_idx, out_val,
                                                       slab_off, tile_off, cap, w, st, stream);
        return run_thr<HQMQ_BF16, HQMQ_GRAN_ELEMENT>(x, B, H, T, D, thr, out_idx, out_val, slab_off,
                                                     tile_off, cap, w, st, stream);
    }
    if (gran == HQMQ_GRAN_CHUNK)
        return run_thr<HQMQ_F32, HQMQ_GRAN_CHUNK>(x, B, H, T, D, thr, out_idx, out_val, slab_off,
                                                  tile_off, cap, w, st, stream);
    return run_thr<HQMQ_F32, HQMQ_GRAN_ELEMENT>(x, B, H, T, D, thr, out_idx, out_val, slab_off,
                                                tile_off, cap, w, st, stream);
}

extern "C" uint64_t hqmq_med3_workspace_bytes(int B, int H, int T, int D) {
    return hqmq::ws_layout(B, H, T, D).total;
}

extern "C" int hqmq_launch_outlier_extract(const void *x, int dtype, int B, int H, int T, int D,
                                           float C, int gran, float *rmed, float *thr,
                                           uint32_t *out_idx, uint16_t *out_val,
                                           uint32_t *slab_off, uint64_t cap, void *ws,
                                           hqmq_status *st, int sm_count, cudaStream_t stream) {
    using namespace hqmq;
    char *w = reinterpret_cast<char *>(ws);
    if (dtype == HQMQ_BF16) {
        if (gran == HQMQ_GRAN_CHUNK)
            return run<HQMQ_BF16, HQMQ_GRAN_CHUNK>(x, B, H, T, D, C, rmed, thr, out_idx, out_val,
                                                   slab_off, cap, w, st, sm_count, stream);
        return run<HQMQ_BF16, HQMQ_GRAN_ELEMENT>(x, B, H, T, D, C, rmed, thr, out_idx, out_val,
                                                 slab_off, cap, w, st, sm_count, stream);
    }
    if (gran == HQMQ_GRAN_CHUNK)
        return run<HQMQ_F32, HQMQ_GRAN_CHUNK>(x, B, H, T, D, C, rmed, thr, out_idx, out_val,
                                              slab_off, cap, w, st, sm_count, stream);
    return run<HQMQ_F32, HQMQ_GRAN_ELEMENT>(x, B, H, T, D, C, rmed, thr, out_idx, out_val, slab_off,
                                            cap, w, st, sm_count, stream);
}
