// search.cu -- exact local search for the HQMQ encode (table-driven).
//
// The encode snaps a chunk x to the codeword c = q_p q_s of the 24 S-word
// effective codebook with the largest <x, c>, ties to the lowest index
// s 24 + p (gist.science/nl, Technische Samenvatting, section 1).  The
// S-codeword loop of encode.cu costs one quaternion product per secondary
// codeword.  This file replaces it by a lookup of the few codewords that can
// win in the neighbourhood of x:
//
// 1. Faces.  Let a be the first coordinate of largest |x_a| and sg = (x_a < 0).
//    x lies on face f = 2 a + sg of the cube: the directions with
//    |x_a| >= |x_k| and that sign of x_a.  Its gnomonic coordinates are the
//    other three coordinates, in index order, divided by |x_a|:
//    t in [-1, 1]^3.
// 2. Cells.  t is mapped by the monotone u(t) = t (A + B t^2) (A = 4/pi,
//    B = 1 - A, so u(+-1) = +-1), which roughly equalises the angular size of
//    the cells, and u is cut into G^3 cells per face.
// 3. Candidates.  For each cell (grown by DELTA on every side to absorb fp32
//    rounding of t), a codeword c is kept unless (i) its angle from the cell
//    centre exceeds the best angle there by more than twice the cell's angular
//    radius, or (ii) another codeword c* beats it at all 8 corners of the cell:
//    <x, c* - c> is linear in x, and the cell's directions are positive
//    multiples of the points of a box with those corners, so c* beats c on the
//    whole cell iff it does at the corners.  Both tests only drop codewords
//    that cannot be the argmax anywhere in the cell, so the list is a superset
//    of the possible winners.  Up to SLOTS survivors are stored in increasing
//    index order; a cell with more is marked OVERFLOW and its chunks use the
//    S-codeword loop.
// 4. Encode.  Score the cell's candidates in slot order with fp32 <x, c> and
//    keep a candidate only if it scores strictly higher: among equal scores
//    the lowest index wins, as the rule asks.  The tables stay in global memory
//    (L2-resident: 4 MB per head, 8 faces x 32^3 cells x 16 B); candidate
//    codewords come from a shared-memory copy of the 24 S codewords replicated
//    8 times so that the 8 lanes of each quarter-warp read 8 different bank
//    groups (no conflicts).
#include "search.cuh"

namespace hqmq {


// Inverse of u(t) = t (A + B t^2) on [-1, 1] (monotone: u' >= A + 3B > 0), by
// bisection in fp64.
__device__ double t_of_u(double u) {
    if (u <= -1.0) return -1.0;
    if (u >= 1.0) return 1.0;
    double lo = -1.0, hi = 1.0;
    const double a = (double)MAP_A, b = (double)MAP_B;
    for (int it = 0; it < 64; ++it) {
        const double m = 0.5 * (lo + hi);
        if (m * (a + b * m * m) < u) lo = m; else hi = m;
    }
    return 0.5 * (lo + hi);
}

// ---------------------------------------------------------------------------
// table build: one thread per (cell, group)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(BUILD_THREADS)
k_build_search_table(const float4 *__restrict__ cb_all, uint32_t S, uint4 *__restrict__ tables) {
    extern __shared__ double4 s_cw[];                 // [24 S] codewords in fp64 (exact copies)
    const uint32_t g = blockIdx.y;
    const uint32_t n_words = 24u * S;
    for (uint32_t i = threadIdx.x; i < n_words; i += BUILD_THREADS) {
        float4 c = codeword((int)(i % 24u), cb_all[(size_t)g * S + i / 24u]);
        s_cw[i] = make_double4(c.x, c.y, c.z, c.w);
    }
    __syncthreads();
    const uint32_t entry = blockIdx.x * BUILD_THREADS + threadIdx.x;   // face * cells + cell
    if (entry >= (uint32_t)LUT_ENTRIES) return;
    const int face = (int)(entry / LUT_CELLS), cell = (int)(entry % LUT_CELLS);
    const int ax = face >> 1;                          // coordinate of largest |x|
    const double sgn = (face & 1) ? -1.0 : 1.0;        // its sign
    int other[3];                                      // the other coordinates, in order
    for (int k = 0, n = 0; k < 4; ++k)
        if (k != ax) other[n++] = k;
    const int ic[3] = {cell / (LUT_G * LUT_G), (cell / LUT_G) % LUT_G, cell % LUT_G};
    double lo[3], hi[3], mid[3];
    for (int k = 0; k < 3; ++k) {
        lo[k] = t_of_u(-1.0 + 2.0 * ic[k] / LUT_G) - LUT_DELTA;
        hi[k] = t_of_u(-1.0 + 2.0 * (ic[k] + 1) / LUT_G) + LUT_DELTA;
        mid[k] = 0.5 * (lo[k] + hi[k]);
    }
    // corners (x_a = +-1, the others = t) and the centre direction
    double cor[8][4];
    for (int q = 0; q < 8; ++q) {
        cor[q][ax] = sgn;
        for (int k = 0; k < 3; ++k) cor[q][other[k]] = ((q >> k) & 1) ? hi[k] : lo[k];
    }
    double uc[4];
    {
        const double cn = sqrt(1.0 + mid[0] * mid[0] + mid[1] * mid[1] + mid[2] * mid[2]);
        uc[ax] = sgn / cn;
        for (int k = 0; k < 3; ++k) uc[other[k]] = mid[k] / cn;
    }
    double cos_rho = 1.0;                              // angular radius of the cell
    for (int q = 0; q < 8; ++q) {
        double n = sqrt(cor[q][0] * cor[q][0] + cor[q][1] * cor[q][1] + cor[q][2] * cor[q][2] +
                        cor[q][3] * cor[q][3]);
        double d = (uc[0] * cor[q][0] + uc[1] * cor[q][1] + uc[2] * cor[q][2] +
                    uc[3] * cor[q][3]) / n;
        cos_rho = fmin(cos_rho, d);
    }
    double best = -2.0;
    for (uint32_t i = 0; i < n_words; ++i) {
        double4 c = s_cw[i];
        best = fmax(best, uc[0] * c.x + uc[1] * c.y + uc[2] * c.z + uc[3] * c.w);
    }
    const double rho = acos(fmin(1.0, cos_rho));
    const double lim = acos(fmax(-1.0, fmin(1.0, best))) + 2.0 * rho + 1e-9;
    const double cos_lim = lim >= 3.141592653589793 ? -2.0 : cos(lim) - 1e-12;
    // (i) angle prefilter
    uint32_t cand[BUILD_MAXC];
    int nc = 0;
    bool overflow = false;
    for (uint32_t i = 0; i < n_words; ++i) {
        double4 c = s_cw[i];
        double d = uc[0] * c.x + uc[1] * c.y + uc[2] * c.z + uc[3] * c.w;
        if (d >= cos_lim) {
            if (nc == BUILD_MAXC) { overflow = true; break; }
            cand[nc++] = i;
        }
    }
    uint32_t keep[LUT_SLOTS];
    int nk = 0;
    if (!overflow) {
        // (ii) dominance on the corners
        for (int j = 0; j < nc && !overflow; ++j) {
            const double4 cj = s_cw[cand[j]];
            bool dominated = false;
            for (int k = 0; k < nc && !dominated; ++k) {
                if (k == j) continue;
                const double4 ck = s_cw[cand[k]];
                const double d0 = ck.x - cj.x, d1 = ck.y - cj.y, d2 = ck.z - cj.z,
                             d3 = ck.w - cj.w;
                bool all = true;
                for (int q = 0; q < 8 && all; ++q) {
                    double v = cor[q][0] * d0 + cor[q][1] * d1 + cor[q][2] * d2 + cor[q][3] * d3;
                    all = v > 1e-12;
                }
                dominated = all;
            }
            if (!dominated) {
                if (nk == LUT_SLOTS) { overflow = true; break; }
                keep[nk++] = cand[j];                  // (cand is in increasing id order)
            }
        }
    }
    uint32_t slot[LUT_SLOTS];
    if (overflow) nk = 0;
    for (int q = 0; q < LUT_SLOTS; ++q) slot[q] = nk > 0 ? (q < nk ? keep[q] : n_words) : 0u;
    slot[0] |= (uint32_t)nk << 12;
    tables[(size_t)g * LUT_ENTRIES + entry] =
        make_uint4(slot[0] | (slot[1] << 16), slot[2] | (slot[3] << 16),
                   slot[4] | (slot[5] << 16), slot[6] | (slot[7] << 16));
}


template <int DT, int LIST, bool ENC, int BB>
__global__ void __launch_bounds__(ENC_THREADS, 1)
k_encode_lut(const void *__restrict__ x, int H, uint32_t groups_per_slab, uint32_t tiles_per_slab,
             uint32_t n_tiles, const float4 *__restrict__ cb_all, uint32_t S, uint32_t b_rt,
             const uint4 *__restrict__ tables, const float *__restrict__ thr, int gran,
             uint32_t *__restrict__ words, uint16_t *__restrict__ radius,
             const uint32_t *__restrict__ tile_off, uint64_t cap, uint32_t *__restrict__ out_idx,
             uint16_t *__restrict__ out_val, DevStatus *st, SpecArgs sa) {
    extern __shared__ float4 s_tab[];                    // [24 S + 1][8]: codewords, then zero
                                                         // (LIST_SPEC: then the key stages)
    const uint32_t b = BB ? (uint32_t)BB : b_rt;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const int n_warps = ENC_THREADS / 32;
    const uint32_t n_words = 24u * S;
    const uint32_t lane7 = (uint32_t)(lane & 7);
    const PackConst pc = pack_const(b, lane);

    // (chunk and list indices fit 32 bits: a call has fewer than 2^32 elements)
    const uint32_t t_begin = (uint32_t)((uint64_t)n_tiles * blockIdx.x / gridDim.x);
    const uint32_t t_end = (uint32_t)((uint64_t)n_tiles * (blockIdx.x + 1) / gridDim.x);
    const uint32_t cap32 = cap < 0xFFFFFFFFull ? (uint32_t)cap : 0xFFFFFFFFu;
    int cur_head = -1;
    unsigned n_nf = 0, n_sat = 0;
    // LIST_SPEC: this warp's stage of window keys (of head stage_h)
    uint32_t *stage = reinterpret_cast<uint32_t *>(s_tab + (size_t)(n_words + 1) * 8) + warp * STAGE;
    // BB != 0: this warp's tile of indices, packed at the end of the tile
    constexpr bool PACK_TILE = BB != 0;
    uint16_t *s_idx = reinterpret_cast<uint16_t *>(
                          reinterpret_cast<uint32_t *>(s_tab + (size_t)(n_words + 1) * 8) +
                          (LIST == LIST_SPEC ? (ENC_THREADS / 32) * STAGE : 0)) +
                      warp * TILE_CHUNKS;
    uint32_t n_stage = 0;
    int stage_h = -1;
    for (uint32_t seg = t_begin; seg < t_end;) {
        const uint32_t slab = seg / tiles_per_slab;
        const uint32_t seg_end = min(t_end, (slab + 1) * tiles_per_slab);
        const int h = (int)(slab % (uint32_t)H);
        const float4 *cb = cb_all + (size_t)h * S;
        const uint4 *tb = tables + (size_t)h * LUT_ENTRIES;
        WinState w{};
        if (LIST == LIST_SPEC) w = sa.win[h];
        if (LIST == LIST_SPEC && h != stage_h) {
            if (n_stage) {
                const WinState ws = sa.win[stage_h];
                flush_stage(stage, n_stage, lane, sa.cand_n + stage_h,
                            sa.cand + (uint64_t)stage_h * sa.cand_cap, sa.cand_cap,
                            sa.med_hist + (size_t)stage_h * MED_BINS * 2, ws.lo_key,
                            median_top_shift(ws.hi_key - ws.lo_key));
            }
            n_stage = 0;
            stage_h = h;
        }
        if (ENC && h != cur_head) {                      // (block-uniform)
            __syncthreads();
            for (uint32_t i = threadIdx.x; i < (n_words + 1) * 8; i += ENC_THREADS) {
                const uint32_t id = i >> 3;
                s_tab[i] = id < n_words ? codeword((int)(id % 24u), __ldg(cb + id / 24u))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            __syncthreads();
            cur_head = h;
        }
        const bool med3 = thr != nullptr;
        const float th = med3 ? __ldg(thr + h) : 0.0f;
        for (uint32_t t = seg + warp; t < seg_end; t += n_warps) {
            const uint32_t g0 = (t % tiles_per_slab) * TILE_GROUPS;
            const uint32_t g1 = min(g0 + TILE_GROUPS, groups_per_slab);
            const uint32_t gbase = slab * groups_per_slab;
            uint32_t lpos = (LIST && LIST != LIST_SPEC) ? __ldg(tile_off + t) : 0u;   // list position
            uint32_t t_def = 0, t_below = 0, t_cbits = 0;     // LIST_SPEC
            RawChunk<DT> nxt;
            nxt.load(x, (size_t)(gbase + g0) * 32 + lane);
            for (uint32_t g = g0; g < g1; ++g) {
                const uint32_t G = gbase + g;
                const uint32_t j = G * 32 + (uint32_t)lane;   // chunk index
                const RawChunk<DT> cur = nxt;
                if (g + 1 < g1) nxt.load(x, (size_t)j + 32);
                float x0 = cur.e(0), x1 = cur.e(1), x2 = cur.e(2), x3 = cur.e(3);
                float r = chunk_norm(x0, x1, x2, x3);
                if (LIST == HQMQ_GRAN_CHUNK + 1) {           // ordered chunk list
                    const bool o = r > th;
                    const uint32_t m = __ballot_sync(FULL, o);
                    if (o) {
                        const uint32_t p = lpos + __popc(m & lt);
                        if (p < cap32) {
                            int sv = 0;
                            const uint32_t h01 = f32x2_to_f16x2_sat(x0, x1, sv);
                            const uint32_t h23 = f32x2_to_f16x2_sat(x2, x3, sv);
                            n_sat += sv;
                            out_idx[p] = j;
                            reinterpret_cast<uint2 *>(out_val)[p] = make_uint2(h01, h23);
                        }
                    }
                    lpos += __popc(m);
                } else if (LIST == HQMQ_GRAN_ELEMENT + 1) {  // ordered element list
                    const float xs[4] = {x0, x1, x2, x3};
                    uint32_t mk = 0;
#pragma unroll
                    for (int i = 0; i < 4; ++i) mk |= (fabsf(xs[i]) > th ? 1u : 0u) << i;
                    const uint32_t n = __popc(mk);
                    uint32_t inc = n;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const uint32_t v = __shfl_up_sync(FULL, inc, o);
                        if (lane >= o) inc += v;
                    }
                    uint32_t p = lpos + inc - n;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (mk & (1u << i)) {
                            if (p < cap32) {
                                int sv = 0;
                                out_val[p] = f32_to_f16_sat(xs[i], sv);
                                n_sat += sv;
                                out_idx[p] = j * 4 + i;
                            }
                            ++p;
                        }
                    }
                    lpos += __shfl_sync(FULL, inc, 31);
                }
                bool spec_cand = false;                      // LIST_SPEC: r > t_lo
                if (LIST == LIST_SPEC) {
                    // key: r's bits (r >= 0; a NaN's bits exceed every finite
                    // key and +inf's, as in the median's order)
                    const uint32_t key = __float_as_uint(r);
                    t_below += key < w.lo_key ? 1u : 0u;
                    const bool in = key >= w.lo_key && key < w.hi_key;
                    const uint32_t mi = __ballot_sync(FULL, in);
                    if (mi) {
                        if (n_stage + 32 > STAGE) {
                            flush_stage(stage, n_stage, lane, sa.cand_n + h,
                                        sa.cand + (uint64_t)h * sa.cand_cap, sa.cand_cap,
                                        sa.med_hist + (size_t)h * MED_BINS * 2, w.lo_key,
                                        median_top_shift(w.hi_key - w.lo_key));
                            n_stage = 0;
                        }
                        if (in) stage[n_stage + __popc(mi & lt)] = key;
                        n_stage += __popc(mi);
                        __syncwarp();
                    }
                    const bool dfn = r > w.t_hi;             // (NaN: false)
                    spec_cand = r > w.t_lo;
                    t_def += dfn ? 1u : 0u;
                    const uint32_t mc = __ballot_sync(FULL, spec_cand);
                    if (lane == (int)(g - g0)) t_cbits = mc;       // stored per tile
                    const bool unc = spec_cand && !dfn;
                    const uint32_t mu = __ballot_sync(FULL, unc);
                    if (mu) {
                        unsigned long long base = 0;
                        if (lane == 0) base = atomicAdd(sa.amb_n, (unsigned long long)__popc(mu));
                        base = __shfl_sync(FULL, base, 0);
                        if (unc) {
                            const unsigned long long pos = base + __popc(mu & lt);
                            if (pos < sa.amb_cap) sa.amb[pos] = make_uint2(t, key);
                        }
                    }
                    if (dfn) r = 0.0f;                       // certain outlier: radius 0, index 0
                }
                if (!ENC) continue;
                if (med3 && LIST != LIST_SPEC) {
                    if (gran == HQMQ_GRAN_CHUNK) {
                        if (r > th) r = 0.0f;        // outlier chunk: no search, radius 0
                    } else {
                        if (fabsf(x0) > th) x0 = 0.0f;
                        if (fabsf(x1) > th) x1 = 0.0f;
                        if (fabsf(x2) > th) x2 = 0.0f;
                        if (fabsf(x3) > th) x3 = 0.0f;
                        r = chunk_norm(x0, x1, x2, x3);
                    }
                }
                const bool finite = r == r && r != __int_as_float(0x7F800000);
                const bool search = finite && r > 0.0f;
                // every lane runs the candidate loop up to the warp's longest
                // list (lanes without a search score candidate 0 of cell 0)
                uint4 rec = make_uint4(1u << 12, 0u, 0u, 0u);
                if (search) {
                    const float a0 = fabsf(x0), a1 = fabsf(x1), a2 = fabsf(x2), a3 = fabsf(x3);
                    const float m = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
                    const bool e0 = a0 == m, e01 = e0 || a1 == m, e012 = e01 || a2 == m;
                    // face: first coordinate a of largest |x_a| and the sign of
                    // x_a; cell: the other three coordinates in index order / m
                    const int a = e0 ? 0 : e01 ? 1 : e012 ? 2 : 3;
                    const float xa = e0 ? x0 : e01 ? x1 : e012 ? x2 : x3;
                    const float c1 = e0 ? x1 : x0;
                    const float c2 = e01 ? x2 : x1;
                    const float c3 = e012 ? x3 : x2;
                    float inv;
                    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(m));   // cells are widened
                    const int cell = (cell_coord(c1 * inv) * LUT_G + cell_coord(c2 * inv)) * LUT_G +
                                     cell_coord(c3 * inv);
                    const int face = 2 * a + (xa < 0.0f ? 1 : 0);
                    rec = __ldg(tb + face * LUT_CELLS + cell);
                }
                const uint32_t cnt = (rec.x >> 12) & 0xFu;
                const bool fallback = cnt == 0;                    // overflowing cell
                const uint32_t sl[4] = {rec.x, rec.y, rec.z, rec.w};
                const uint32_t kmax = __reduce_max_sync(FULL, cnt);
                // slots hold increasing ids: a strictly higher score replaces
                // the best, so equal scores keep the lowest index
                float best = __int_as_float(0xFF800000);           // -inf
                uint32_t bid = 0;
#pragma unroll
                for (int k = 0; k < LUT_SLOTS; ++k) {
                    if ((uint32_t)k >= kmax) break;                // warp-uniform
                    const uint32_t id = (sl[k >> 1] >> ((k & 1) * 16)) & LUT_ID_MASK;
                    const float4 c = s_tab[(id << 3) | lane7];
                    const float sc = __fmaf_rn(x3, c.w, __fmaf_rn(x2, c.z,
                                     __fmaf_rn(x1, c.y, __fmul_rn(x0, c.x))));
                    if (sc > best) { best = sc; bid = id; }
                }
                uint32_t idx = 0;
                if (search && !fallback) idx = bid;
                if (search && fallback) idx = sloop_index(x0, x1, x2, x3, cb, S);
                uint16_t rh;
                if (!finite) {
                    rh = 0x7E00u;
                    ++n_nf;
                } else {
                    int sat = 0;
                    rh = radius_to_f16(r, sat);
                    if (!spec_cand) n_sat += sat;            // (LIST_FIX decides the others)
                }
                radius[j] = rh;
                if (PACK_TILE)
                    s_idx[(g - g0) * 32 + lane] = (uint16_t)idx;
                else
                    pack_group32<BB>(idx, b, lane, pc, words + (size_t)G * b);
            }
            if (PACK_TILE && ENC) {
                __syncwarp();
                pack_tile<BB ? BB : 8>(s_idx, g1 - g0, lane, words + (size_t)(gbase + g0) * b);
                __syncwarp();                                  // (s_idx is refilled next tile)
            }
            if (LIST == LIST_SPEC) {
                t_def = __reduce_add_sync(FULL, t_def);
                t_below = __reduce_add_sync(FULL, t_below);
                if (lane == 0) {
                    sa.tile_cnt[t] = t_def;
                    if (t_below) atomicAdd(sa.below + h, (unsigned long long)t_below);
                }
                if (lane < (int)(g1 - g0)) sa.cbits[gbase + g0 + lane] = t_cbits;
            }
        }
        if (LIST == LIST_SPEC) {                             // status counts per head
            const unsigned nf = __reduce_add_sync(FULL, n_nf);
            const unsigned ns = __reduce_add_sync(FULL, n_sat);
            if (lane == 0 && (nf | ns)) {
                atomicAdd(sa.head_stat + 2 * h, (unsigned long long)nf);
                atomicAdd(sa.head_stat + 2 * h + 1, (unsigned long long)ns);
            }
            n_nf = n_sat = 0;
        }
        seg = seg_end;
    }
    if (LIST == LIST_SPEC) {
        if (n_stage) {
            const WinState ws = sa.win[stage_h];
            flush_stage(stage, n_stage, lane, sa.cand_n + stage_h,
                        sa.cand + (uint64_t)stage_h * sa.cand_cap, sa.cand_cap,
                        sa.med_hist + (size_t)stage_h * MED_BINS * 2, ws.lo_key,
                        median_top_shift(ws.hi_key - ws.lo_key));
        }
        return;
    }
    const unsigned nf = __reduce_add_sync(FULL, n_nf);
    const unsigned ns = __reduce_add_sync(FULL, n_sat);
    if (lane == 0 && st) {
        if (nf) status_add(st, HQMQ_FLAG_NONFINITE, &st->n_nonfinite, nf);
        if (ns) status_add(st, HQMQ_FLAG_SATURATED, &st->n_saturated, ns);
    }
}

// The list pass of the one-read chunk-mode path (after the exact threshold):
// per tile of a head whose window held, the chunks recorded by the encode
// pass (r > t_lo) are read again, decided (r > thr) and written to the
// ordered list; those with r <= t_hi were encoded as bulk chunks and get
// index 0 and radius 0.  A head whose window missed is encoded again exactly
// (S-codeword loop, list, radius, index), as hqmq_encode does.  Also adds the
// encode pass's status counts of the heads whose result stands.
constexpr int FIX_THREADS = 256;

template <int DT>
__global__ void __launch_bounds__(FIX_THREADS)
k_list_fix(const void *__restrict__ x, int H, uint32_t groups_per_slab, uint32_t tiles_per_slab,
           uint32_t n_tiles, const float4 *__restrict__ cb_all, uint32_t S, uint32_t b,
           const float *__restrict__ thr, uint32_t *__restrict__ words,
           uint16_t *__restrict__ radius, const uint32_t *__restrict__ tile_off, uint64_t cap,
           uint32_t *__restrict__ out_idx, uint16_t *__restrict__ out_val, DevStatus *st,
           SpecArgs sa, int use_cvals) {
    // use_cvals: the encode pass kept the raw values of the first CVAL_SLOTS
    // possible outliers of each 8-group unit, in chunk order (sa.cvals);
    // chunks of a unit with more of them are read from x
    constexpr int CB = DT == HQMQ_BF16 ? 8 : 16;
    pdl_wait();                                    // (launched with launch_pdl)
    pdl_trigger();
    const uint32_t units_per_slab = (groups_per_slab + 7) / 8;
    const int lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    const uint32_t cap32 = cap < 0xFFFFFFFFull ? (uint32_t)cap : 0xFFFFFFFFu;
    const PackConst pc = pack_const(b, lane);
    const uint32_t warp_g = blockIdx.x * (FIX_THREADS / 32) + (threadIdx.x >> 5);
    const uint32_t n_warps = gridDim.x * (FIX_THREADS / 32);
    unsigned n_nf = 0, n_sat = 0;
    for (uint32_t t = warp_g; t < n_tiles; t += n_warps) {
        const uint32_t slab = t / tiles_per_slab;
        const int h = (int)(slab % (uint32_t)H);
        const WinState w = sa.win[h];
        const bool miss = w.miss != 0;
        const float th = __ldg(thr + h);
        const uint32_t g0 = (t % tiles_per_slab) * TILE_GROUPS;
        const uint32_t g1 = min(g0 + TILE_GROUPS, groups_per_slab);
        const uint32_t gbase = slab * groups_per_slab;
        uint32_t lpos = __ldg(tile_off + t);
        if (!miss) {
            // the recorded chunks (r > t_lo) of this tile, in order: lane i
            // reads group i's bits; candidate k (in tile order) goes to lane
            // k mod 32, which finds its group by a search over the
            // inclusive counts and its chunk as the group's n-th set bit
            const uint32_t ng = g1 - g0;
            const uint32_t gw = (uint32_t)lane < ng ? __ldg(sa.cbits + gbase + g0 + lane) : 0u;
            const uint32_t pcount = __popc(gw);
            uint32_t incl = pcount;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(FULL, incl, o);
                if (lane >= o) incl += v;
            }
            const uint32_t total = __shfl_sync(FULL, incl, 31);
            for (uint32_t k0 = 0; k0 < total; k0 += 32) {        // (warp-uniform)
                const uint32_t k = k0 + (uint32_t)lane;
                const bool c = k < total;
                uint32_t gl = 0;                                // first group with incl > k
#pragma unroll
                for (int step = 16; step >= 1; step >>= 1) {
                    const uint32_t v = __shfl_sync(FULL, incl, (int)(gl + step - 1));
                    if (v <= k) gl += step;
                }
                gl &= 31u;
                const uint32_t ex = __shfl_sync(FULL, incl - pcount, (int)gl);
                const uint32_t word = __shfl_sync(FULL, gw, (int)gl);
                // the candidate's unit (8 groups) and its rank there
                const uint32_t ug = gl & ~7u;
                const uint32_t u_before = __shfl_sync(FULL, incl - pcount, (int)ug);
                const uint32_t u_total = __shfl_sync(FULL, incl, (int)(ug + 7)) - u_before;
                const uint32_t bit = c ? __fns(word, 0u, (int)(k - ex + 1)) : 0u;
                const uint32_t G = gbase + g0 + gl;
                const uint32_t j = G * 32 + bit;
                float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f, r = 0.f;
                if (c) {
                    RawChunk<DT> v;
                    if (use_cvals && u_total <= (uint32_t)CVAL_SLOTS) {
                        const uint32_t u = slab * units_per_slab + (g0 + gl) / 8;
                        v.v = *reinterpret_cast<const decltype(v.v) *>(
                            sa.cvals + ((size_t)u * CVAL_SLOTS + (k - u_before)) * CB);
                    } else {
                        v.load(x, j);
                    }
                    x0 = v.e(0); x1 = v.e(1); x2 = v.e(2); x3 = v.e(3);
                    r = chunk_norm(x0, x1, x2, x3);
                }
                const bool o = c && r > th;
                const uint32_t mo = __ballot_sync(FULL, o);
                if (o) {
                    const uint32_t p = lpos + __popc(mo & lt);
                    if (p < cap32) {
                        int sv = 0;
                        const uint32_t h01 = f32x2_to_f16x2_sat(x0, x1, sv);
                        const uint32_t h23 = f32x2_to_f16x2_sat(x2, x3, sv);
                        n_sat += sv;
                        out_idx[p] = j;
                        reinterpret_cast<uint2 *>(out_val)[p] = make_uint2(h01, h23);
                    }
                    if (!(r > w.t_hi)) {                // encoded as a bulk chunk: zero it
                        radius[j] = 0;
                        clear_index(words + (size_t)G * b, b, (int)bit);
                    }
                } else if (c && !(r > w.t_hi) && r >= 65520.0f) {
                    ++n_sat;                             // bulk radius saturated (uncounted)
                }
                lpos += __popc(mo);
            }
            continue;
        }
        // a head whose window missed: exact list and encode of the tile
        const float4 *cb = cb_all + (size_t)h * S;
        for (uint32_t g = g0; g < g1; ++g) {
            const uint32_t G = gbase + g;
            const uint32_t j = G * 32 + (uint32_t)lane;
            RawChunk<DT> v;
            v.load(x, j);
            const float x0 = v.e(0), x1 = v.e(1), x2 = v.e(2), x3 = v.e(3);
            float r = chunk_norm(x0, x1, x2, x3);
            const bool o = r > th;
            const uint32_t m = __ballot_sync(FULL, o);
            if (o) {
                const uint32_t p = lpos + __popc(m & lt);
                if (p < cap32) {
                    int sv = 0;
                    const uint32_t h01 = f32x2_to_f16x2_sat(x0, x1, sv);
                    const uint32_t h23 = f32x2_to_f16x2_sat(x2, x3, sv);
                    n_sat += sv;
                    out_idx[p] = j;
                    reinterpret_cast<uint2 *>(out_val)[p] = make_uint2(h01, h23);
                }
                r = 0.0f;                                  // outlier chunk: radius 0, index 0
            }
            lpos += __popc(m);
            const bool finite = r == r && r != __int_as_float(0x7F800000);
            const uint32_t idx = (finite && r > 0.0f) ? sloop_index(x0, x1, x2, x3, cb, S) : 0u;
            uint16_t rh;
            if (!finite) {
                rh = 0x7E00u;
                ++n_nf;
            } else {
                int sat = 0;
                rh = radius_to_f16(r, sat);
                n_sat += sat;
            }
            radius[j] = rh;
            pack_group32<0>(idx, b, lane, pc, words + (size_t)G * b);
        }
    }
    const unsigned nf = __reduce_add_sync(FULL, n_nf);
    const unsigned ns = __reduce_add_sync(FULL, n_sat);
    if (lane == 0 && st) {
        if (nf) status_add(st, HQMQ_FLAG_NONFINITE, &st->n_nonfinite, nf);
        if (ns) status_add(st, HQMQ_FLAG_SATURATED, &st->n_saturated, ns);
    }
    if (blockIdx.x == 0 && st) {
        // the encode pass's status counts of the heads whose result stands
        for (int hh = threadIdx.x; hh < H; hh += FIX_THREADS)
            if (!sa.win[hh].miss) {
                status_add(st, HQMQ_FLAG_NONFINITE, &st->n_nonfinite, sa.head_stat[2 * hh]);
                status_add(st, HQMQ_FLAG_SATURATED, &st->n_saturated, sa.head_stat[2 * hh + 1]);
            }
    }
}


}  // namespace hqmq

extern "C" uint64_t hqmq_lut_bytes_per_group(uint32_t S) {
    if (S < 1 || S > hqmq::LUT_MAX_S) return 0;
    return (uint64_t)hqmq::LUT_ENTRIES * sizeof(uint4);
}

extern "C" int hqmq_launch_build_search_table(const float *cb, uint32_t S, uint32_t n_groups,
                                              void *table, cudaStream_t stream) {
    using namespace hqmq;
    const size_t smem = (size_t)24 * S * sizeof(double4);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(k_build_search_table, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return HQMQ_ERR_CUDA;
    dim3 grid(LUT_ENTRIES / BUILD_THREADS, n_groups);
    k_build_search_table<<<grid, BUILD_THREADS, smem, stream>>>(
        reinterpret_cast<const float4 *>(cb), S, reinterpret_cast<uint4 *>(table));
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

namespace hqmq {

template <int DT, int LIST, bool ENC, int BB>
static int launch_lut_bb(int B, int H, int T, int D, const void *x, const float *cb, uint32_t S,
                         uint32_t b, const void *table, const float *thr, int gran,
                         uint32_t *words, uint16_t *radius, const uint32_t *tile_off, uint64_t cap,
                         uint32_t *out_idx, uint16_t *out_val, hqmq_status *st, int sm_count,
                         cudaStream_t stream, const SpecArgs &sa) {
    const uint32_t gps = (uint32_t)(((uint64_t)T * D / 4) / 32);
    const uint32_t tps = (gps + TILE_GROUPS - 1) / TILE_GROUPS;
    const uint32_t n_tiles = (uint32_t)((uint64_t)B * H * tps);
    const size_t smem = (ENC ? enc_smem_bytes(S) : 0) +
                        (LIST == LIST_SPEC ? (size_t)(ENC_THREADS / 32) * STAGE * 4 : 0) +
                        (ENC && BB != 0 ? (size_t)(ENC_THREADS / 32) * TILE_CHUNKS * 2 : 0);
    auto kern = k_encode_lut<DT, LIST, ENC, BB>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return HQMQ_ERR_CUDA;
    // one CTA per SM, each a contiguous share of the call's tiles
    uint64_t ctas = (uint64_t)sm_count;
    const uint64_t want = ((uint64_t)n_tiles + 7) / 8;
    if (ctas > want) ctas = want;
    if (ctas < 1) ctas = 1;
    kern<<<(unsigned)ctas, ENC_THREADS, smem, stream>>>(
        x, H, gps, tps, n_tiles, reinterpret_cast<const float4 *>(cb), S, b,
        reinterpret_cast<const uint4 *>(table), thr, gran, words, radius, tile_off, cap, out_idx,
        out_val, reinterpret_cast<DevStatus *>(st), sa);
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

// Index widths 8 (S = 8..10) and 10 (S = 22..42) get kernels with constant
// shifts; others use the runtime width.
template <int DT, int LIST, bool ENC>
static int launch_lut(int B, int H, int T, int D, const void *x, const float *cb, uint32_t S,
                      uint32_t b, const void *table, const float *thr, int gran, uint32_t *words,
                      uint16_t *radius, const uint32_t *tile_off, uint64_t cap, uint32_t *out_idx,
                      uint16_t *out_val, hqmq_status *st, int sm_count, cudaStream_t stream,
                      const SpecArgs &sa) {
    if (ENC && b == 8)
        return launch_lut_bb<DT, LIST, ENC, 8>(B, H, T, D, x, cb, S, b, table, thr, gran, words,
                                               radius, tile_off, cap, out_idx, out_val, st,
                                               sm_count, stream, sa);
    if (ENC && b == 10)
        return launch_lut_bb<DT, LIST, ENC, 10>(B, H, T, D, x, cb, S, b, table, thr, gran, words,
                                                radius, tile_off, cap, out_idx, out_val, st,
                                                sm_count, stream, sa);
    return launch_lut_bb<DT, LIST, ENC, 0>(B, H, T, D, x, cb, S, b, table, thr, gran, words,
                                           radius, tile_off, cap, out_idx, out_val, st, sm_count,
                                           stream, sa);
}

template <int LIST, bool ENC>
static int launch_lut_dt(int dtype, int B, int H, int T, int D, const void *x, const float *cb,
                         uint32_t S, uint32_t b, const void *table, const float *thr, int gran,
                         uint32_t *words, uint16_t *radius, const uint32_t *tile_off, uint64_t cap,
                         uint32_t *out_idx, uint16_t *out_val, hqmq_status *st, int sm,
                         cudaStream_t stream, const SpecArgs &sa = SpecArgs{}) {
    if (dtype == HQMQ_BF16)
        return launch_lut<HQMQ_BF16, LIST, ENC>(B, H, T, D, x, cb, S, b, table, thr, gran, words,
                                                radius, tile_off, cap, out_idx, out_val, st, sm,
                                                stream, sa);
    return launch_lut<HQMQ_F32, LIST, ENC>(B, H, T, D, x, cb, S, b, table, thr, gran, words, radius,
                                           tile_off, cap, out_idx, out_val, st, sm, stream, sa);
}

}  // namespace hqmq

extern "C" int hqmq_launch_encode_lut(const void *x, int dtype, int B, int H, int T, int D,
                                      const float *cb, uint32_t S, uint32_t b, const void *table,
                                      const float *thr, int gran, uint32_t *words,
                                      uint16_t *radius, hqmq_status *st, int sm_count,
                                      cudaStream_t stream) {
    return hqmq::launch_lut_dt<0, true>(dtype, B, H, T, D, x, cb, S, b, table, thr, gran, words,
                                        radius, nullptr, 0, nullptr, nullptr, st, sm_count, stream);
}

// Pass C of the two-read Med3x: the ordered list (from exact thr and tile
// offsets) and, if table != NULL, the encode in the same read.
extern "C" int hqmq_launch_list_pass(const void *x, int dtype, int B, int H, int T, int D,
                                     const float *cb, uint32_t S, uint32_t b, const void *table,
                                     const float *thr, int gran, uint32_t *words,
                                     uint16_t *radius, const uint32_t *tile_off, uint64_t cap,
                                     uint32_t *out_idx, uint16_t *out_val, hqmq_status *st,
                                     int sm_count, cudaStream_t stream) {
    using namespace hqmq;
    const bool enc = table != nullptr;
    if (gran == HQMQ_GRAN_CHUNK) {
        return enc ? launch_lut_dt<HQMQ_GRAN_CHUNK + 1, true>(dtype, B, H, T, D, x, cb, S, b, table,
                                                             thr, gran, words, radius, tile_off,
                                                             cap, out_idx, out_val, st, sm_count,
                                                             stream)
                   : launch_lut_dt<HQMQ_GRAN_CHUNK + 1, false>(dtype, B, H, T, D, x, cb, S, b,
                                                              table, thr, gran, words, radius,
                                                              tile_off, cap, out_idx, out_val, st,
                                                              sm_count, stream);
    }
    return enc ? launch_lut_dt<HQMQ_GRAN_ELEMENT + 1, true>(dtype, B, H, T, D, x, cb, S, b, table,
                                                           thr, gran, words, radius, tile_off, cap,
                                                           out_idx, out_val, st, sm_count, stream)
               : launch_lut_dt<HQMQ_GRAN_ELEMENT + 1, false>(dtype, B, H, T, D, x, cb, S, b, table,
                                                            thr, gran, words, radius, tile_off,
                                                            cap, out_idx, out_val, st, sm_count,
                                                            stream);
}

// One-read chunk-mode Med3x, step B + speculative encode (after A + W).
extern "C" int hqmq_launch_spec_encode(const void *x, int dtype, int B, int H, int T, int D,
                                       const float *cb, uint32_t S, uint32_t b, const void *table,
                                       uint32_t *words, uint16_t *radius, void *ws, int sm_count,
                                       cudaStream_t stream) {
    using namespace hqmq;
    const SpecArgs sa = spec_args(reinterpret_cast<char *>(ws),
                                  fused_layout(B, H, T, D, HQMQ_GRAN_CHUNK));
    return launch_lut_dt<LIST_SPEC, true>(dtype, B, H, T, D, x, cb, S, b, table, nullptr,
                                          HQMQ_GRAN_CHUNK, words, radius, nullptr, 0, nullptr,
                                          nullptr, nullptr, sm_count, stream, sa);
}

// One-read chunk-mode Med3x, the list and the code fix-ups (after F + X + U + S).
extern "C" int hqmq_launch_fix_pass(const void *x, int dtype, int B, int H, int T, int D,
                                    const float *cb, uint32_t S, uint32_t b, const void *table,
                                    const float *thr, uint32_t *words, uint16_t *radius,
                                    const uint32_t *tile_off, uint64_t cap, uint32_t *out_idx,
                                    uint16_t *out_val, void *ws, hqmq_status *st, int sm_count,
                                    cudaStream_t stream, int use_cvals) {
    using namespace hqmq;
    (void)table;
    const SpecArgs sa = spec_args(reinterpret_cast<char *>(ws),
                                  fused_layout(B, H, T, D, HQMQ_GRAN_CHUNK));
    const uint32_t gps = (uint32_t)(((uint64_t)T * D / 4) / 32);
    const uint32_t tps = (gps + TILE_GROUPS - 1) / TILE_GROUPS;
    const uint32_t n_tiles = (uint32_t)((uint64_t)B * H * tps);
    uint64_t ctas = (uint64_t)sm_count * 8;
    const uint64_t want = ((uint64_t)n_tiles + FIX_THREADS / 32 - 1) / (FIX_THREADS / 32);
    if (ctas > want) ctas = want;
    if (ctas < 1) ctas = 1;
    const float4 *cb4 = reinterpret_cast<const float4 *>(cb);
    DevStatus *dst = reinterpret_cast<DevStatus *>(st);
    const cudaError_t e =
        dtype == HQMQ_BF16
            ? launch_pdl(k_list_fix<HQMQ_BF16>, dim3((unsigned)ctas), dim3(FIX_THREADS), 0, stream,
                         x, H, gps, tps, n_tiles, cb4, S, b, thr, words, radius, tile_off, cap,
                         out_idx, out_val, dst, sa, use_cvals)
            : launch_pdl(k_list_fix<HQMQ_F32>, dim3((unsigned)ctas), dim3(FIX_THREADS), 0, stream,
                         x, H, gps, tps, n_tiles, cb4, S, b, thr, words, radius, tile_off, cap,
                         out_idx, out_val, dst, sa, use_cvals);
    if (e != cudaSuccess) return HQMQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}
