// attention.cu -- decode-phase attention straight from HQMQ codes.
//
// The pages run their decoder inside the attention kernel (gist.science/nl,
// Technische Samenvatting, "Memory en Latentie"): the K and V caches stay
// compressed and each step decodes them on the fly.  This file computes, for
// one query token per sequence (GQA: G = Hq / Hk query heads per KV head),
//   o[b][hq] = sum_t softmax_t(scale <q[b][hq], K^[b][hk][t]>) V^[b][hk][t],
//   hk = hq / G,
// where K^ and V^ are exactly hqmq_decode's bf16 outputs (code, radius and
// outlier list).
//
// k_attn<R>: a CTA (8 warps) takes a contiguous range of 16-token blocks of
// one (b, hk); each warp a sub-range, with all G <= 8 query heads as the
// rows of a 16-row tile (rows >= G are zero).  The codes of a block are
// decoded in registers straight into mma.m16n8k16 operands, so neither K^
// nor V^ touches shared memory:
//   * scores S = Q K^T: K^ is the B operand; lane (n, q) = (lane / 4,
//     lane % 4) decodes chunks 8 q .. 8 q + 7 of tokens n and n + 8 and puts
//     chunk 8 q + ks in the k-slots of k-step ks (the order in which the 128
//     products of a dot product are summed is free; Q is loaded in the same
//     order).  bf16 x bf16 products are exact in the fp32 accumulator;
//   * online softmax in base 2 per query row (the C fragment of S holds, per
//     lane, exactly the B fragment of P^T that the next product needs);
//   * O^T += V^T P^T: V^ is the A operand; lane (n, q) decodes chunks 4 n ..
//     4 n + 3 of tokens 2 q, 2 q + 1, 2 q + 8, 2 q + 9, element 2 h + v of
//     chunk 4 n + i in slot n + 8 v of m-tile 2 i + h; P enters as two bf16
//     terms P_hi + P_lo (about 16 significant bits).
// The codeword table of each head lives in shared memory in R copies, lane
// l reading copy l % R (R = 8: the 8 lanes of a 16-byte phase never share a
// bank group).  Outlier lists: a chunk-mode K entry (its code has radius 0,
// so its decoded chunk is zero) enters the scores through extra mma k-steps,
// the CTA's query rows at the entry's chunk against the entry's values in
// its token's column; V entries, and both in element mode, are marked per
// block (slot map or bitmap) and patched into the decoded chunk before it
// enters the mma.  The warps' (max, sum, P V) partials are merged in shared
// memory; with several CTAs per (b, hk), the last one to finish merges the
// CTA partials.
#include <cuda_bf16.h>

#include "med3_window.cuh"

namespace hqmq {

constexpr int ATT_WARPS = 8;
constexpr int ATT_THREADS = ATT_WARPS * 32;
constexpr int ATT_D = 128;                    // head dimension (32 chunks = one packing group)
constexpr int ATT_BLK = 16;                   // tokens per decoded block
constexpr int ATT_PART = ATT_D + 2;           // floats per partial: max, sum, O[D]

struct CodesDev {
    const uint32_t *words;
    const uint16_t *radius;
    const float4 *cb;                          // this call's heads: [Hk][S]
    const uint32_t *out_idx;
    const uint16_t *out_val;
    const uint32_t *tile_off;                  // NULL: no list
    uint32_t cap32;
};

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

struct KVDev {
    const uint32_t *words;      // [groups][b]
    const uint16_t *radius;     // fp16 bits [chunks]
    const float4 *cb;           // [Hk][S]
    const uint32_t *out_idx;    // NULL: no list
    const uint16_t *out_val;
    const uint32_t *tile_off;   // list position of each 1024-chunk tile's first entry
    uint32_t cap32;
    int gran;
    const uint32_t *rwords;     // quantized radius: b-bit codes laid out like the indices
    const float *thr;           // [Hk]: the range of the codes
};

struct AttnArgs {
    const uint16_t *q;          // bf16 bits [B][Hk*G][128]
    const int *seq_len;         // [B] or NULL (= T)
    KVDev k, v;
    int B, Hk, G, T;
    uint32_t S, b;
    float sl2;                  // softmax scale * log2(e)
    int cph;                    // CTAs per (b, hk)
    uint32_t tiles_per_slab;
    void *o;                    // [B][Hk*G][128], bf16 or fp32
    int out_dtype;
    float *part;                // [B*Hk][cph][ATT_G][ATT_PART] when cph > 1
    uint32_t *done;             // [B*Hk] arrival counters, zero on entry
    DevStatus *st;              // (nothing is recorded)
};

constexpr int ATT_G = 8;                      // query rows per KV head (GQA group) handled
constexpr int LIST_WORDS = 64;                // bitmap words of one block (element mode)

// (r c0, r c1) with one packed instruction; each product is the IEEE
// round-to-nearest fp32 product (as __fmul_rn).
__device__ __forceinline__ float2 mul2(float r, float c0, float c1) {
    float2 o;
    asm("{.reg .b64 t, s;\n\tmov.b64 t, {%2, %3};\n\tmov.b64 s, {%4, %4};\n\t"
        "mul.rn.f32x2 t, t, s;\n\tmov.b64 {%0, %1}, t;}"
        : "=f"(o.x), "=f"(o.y)
        : "f"(c0), "f"(c1), "f"(r));
    return o;
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async8(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_wait1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// Index words one lane loads per token: K runs are 8 chunks (8 b bits from
// bit 8 q b of the token's group), V runs 4 chunks (from bit 4 n b).  With b
// known at compile time (BT = 8 or 10) exactly the words the run touches;
// BT = 0: up to 4 / 3 words, the unneeded ones predicated off.
template <int BT> struct Geo {
    static constexpr int KW = BT == 8 ? 2 : BT == 10 ? 3 : 4;
    static constexpr int VW = BT == 8 ? 1 : BT == 10 ? 2 : 3;
};

// What one lane loads for one 16-token block:
//   K: tokens t0 + n + 8 j (n = lane / 4, j = 0, 1), chunks 8 q .. 8 q + 7
//      (q = lane % 4): one 16-byte radius load and KW index words each;
//   V: tokens t0 + 2 q + (s & 1) + 8 (s >> 1) (s = 0..3), chunks 4 n .. 4 n + 3:
//      one 8-byte radius load and VW index words each.
template <int BT> struct BlockRegs {
    uint4 kr[2];
    uint32_t kw[2][Geo<BT>::KW];
    uint2 vr[4];
    uint32_t vw[4][Geo<BT>::VW];
    uint32_t krw[2][Geo<BT>::KW];             // RQ: radius-code words (same geometry)
    uint32_t vrw[4][Geo<BT>::VW];
};

// Per-lane base pointers of the block loads at token 0 of the slab: K
// token n, V token 2 q (the other tokens of a block are fixed offsets).
struct LanePtrs {
    const uint32_t *kw, *vw;
    const uint4 *kr;
    const uint2 *vr;
    const uint32_t *krw, *vrw;                // RQ: radius-code words
};

// Loads of the block starting at token t0 (tokens >= len read as zero);
// kneed / vneed: the words a run spans (BT = 0).
template <int BT, int RQ>
__device__ __forceinline__ void load_block(const LanePtrs &P, uint32_t b, int t0, int len,
                                           int lane, uint32_t kneed, uint32_t vneed,
                                           BlockRegs<BT> &R) {
    const int n = lane >> 2, q = lane & 3;
    const uint32_t tb = (uint32_t)t0 * b;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const bool ok = t0 + n + 8 * j < len;
        if (!RQ) R.kr[j] = ok ? __ldcs(P.kr + (size_t)(t0 + 8 * j) * 4) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t *w = P.kw + tb + 8 * j * b;
#pragma unroll
        for (int i = 0; i < Geo<BT>::KW; ++i)
            R.kw[j][i] = (ok && (BT || (uint32_t)i < kneed)) ? __ldg(w + i) : 0u;
        if (RQ) {
            const uint32_t *rw = P.krw + tb + 8 * j * b;
#pragma unroll
            for (int i = 0; i < Geo<BT>::KW; ++i)
                R.krw[j][i] = (ok && (BT || (uint32_t)i < kneed)) ? __ldcs(rw + i) : 0u;
        }
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int dt = (s & 1) + 8 * (s >> 1);
        const bool ok = t0 + 2 * q + dt < len;
        if (!RQ) R.vr[s] = ok ? __ldcs(P.vr + (size_t)(t0 + dt) * 8) : make_uint2(0u, 0u);
        const uint32_t *w = P.vw + tb + dt * b;
#pragma unroll
        for (int i = 0; i < Geo<BT>::VW; ++i)
            R.vw[s][i] = (ok && (BT || (uint32_t)i < vneed)) ? __ldg(w + i) : 0u;
        if (RQ) {
            const uint32_t *rw = P.vrw + tb + dt * b;
#pragma unroll
            for (int i = 0; i < Geo<BT>::VW; ++i)
                R.vrw[s][i] = (ok && (BT || (uint32_t)i < vneed)) ? __ldcs(rw + i) : 0u;
        }
    }
}

// A lane's run of indices: x = the run's words shifted so that index k sits
// at bits [k b, k b + b).  BT = 8 runs start on a word boundary.
template <int BT, int NW> struct Run {
    uint32_t x[NW];
    __device__ __forceinline__ void init(const uint32_t (&w)[NW], uint32_t o) {
        if constexpr (BT == 8) {
#pragma unroll
            for (int i = 0; i < NW; ++i) x[i] = w[i];
        } else {
#pragma unroll
            for (int i = 0; i + 1 < NW; ++i) x[i] = __funnelshift_r(w[i], w[i + 1], o);
            x[NW - 1] = w[NW - 1] >> o;
        }
    }
    __device__ __forceinline__ uint32_t get(int k, uint32_t b, uint32_t mask) const {
        if constexpr (BT > 0) {
            const int p = k * BT, wi = p >> 5, sh = p & 31;
            constexpr uint32_t m = (1u << BT) - 1u;
            if (sh + BT <= 32 || wi + 1 >= NW) return (x[wi] >> sh) & m;
            return __funnelshift_r(x[wi], x[wi + 1], sh) & m;
        } else {
            const uint32_t p = (uint32_t)k * b, wi = p >> 5, sh = p & 31;
            uint32_t lo = x[0], hi = NW > 1 ? x[1] : 0u;
#pragma unroll
            for (int i = 1; i < NW; ++i)
                if (wi == (uint32_t)i) {
                    lo = x[i];
                    hi = i + 1 < NW ? x[i + 1] : 0u;
                }
            return __funnelshift_r(lo, hi, sh) & mask;
        }
    }
};

// Outlier list of the current tile of one warp, per tensor: the first LC
// entries of each 32-token tile (one list tile) are copied to shared memory
// with cp.async one tile ahead.  Chunk-mode lists then get a per-block slot
// map; element-mode lists a per-block bitmap with the number of set bits
// before each word, so that an entry's list position is pos0 + rank (the
// list is in ascending index order without repeats).  Entries past LC in a
// tile are read from global memory.
template <int LC> struct WarpList {
    uint32_t idx[2][2][LC];                   // [tile parity][tensor]
    uint2 val[2][2][LC];                      // chunk mode: the 4 fp16 values
    // chunk-mode lists: per tensor one byte per chunk of the block, the
    // staged slot + 1 of its entry (255: past the staged part, 0: none);
    // element mode: per tensor a bitmap (64 words) and per-word prefix counts
    uint32_t aux[4 * LIST_WORDS];
    __device__ __forceinline__ uint32_t *bm(int t) { return aux + t * LIST_WORDS; }
    __device__ __forceinline__ uint32_t *pre(int t) { return aux + (2 + t) * LIST_WORDS; }
    __device__ __forceinline__ uint8_t *map(int t) {
        return reinterpret_cast<uint8_t *>(aux) + t * 512;
    }
};
static_assert(sizeof(WarpList<64>) == 48 * 64 + 1024, "per-warp list scratch");

struct ListView {
    bool any;                                 // the block has list entries
    uint32_t pos0;                            // list position of its first entry
};

// Starts the copy of the first LC entries [a, e) of a tile.
template <int LC>
__device__ __forceinline__ void stage_tile(const KVDev &X, uint32_t a, uint32_t e, uint32_t *sidx,
                                           uint2 *sval, int lane) {
    const uint32_t n = min(e - a, (uint32_t)LC);
    for (uint32_t k = (uint32_t)lane; k < n; k += 32) {
        cp_async4(sidx + k, X.out_idx + a + k);
        if (X.gran == HQMQ_GRAN_CHUNK) cp_async8(sval + k, X.out_val + (uint64_t)(a + k) * 4);
    }
}

// Chunk-mode lists: writes the block's slot map from the tile's entries
// [a, e); true if the block has entries.  Warp-collective.
template <int LC>
__device__ __forceinline__ bool map_block(const KVDev &X, const uint32_t *sidx, uint32_t a,
                                          uint32_t e, uint32_t u0, uint8_t *map, int lane) {
    if (a >= e) return false;
    __syncwarp();
    reinterpret_cast<uint4 *>(map)[lane] = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
    bool hit = false;
    for (uint32_t k = (uint32_t)lane; k < e - a; k += 32) {
        const uint32_t ix = k < (uint32_t)LC ? sidx[k] : __ldg(X.out_idx + a + k);
        const uint32_t loc = ix - u0;
        if (loc < 512u) {
            map[loc] = k < (uint32_t)LC ? (uint8_t)(k + 1) : (uint8_t)255;
            hit = true;
        }
    }
    const bool any = __any_sync(FULL, hit);
    __syncwarp();
    return any;
}

// fp16 x 4 -> bf16 x 4 (RN-even), in place, for n staged entries.
__device__ __forceinline__ uint2 f16x4_to_bf16x4(uint2 e) {
    return make_uint2(pack_bf16(f16_bits_to_f32(e.x & 0xFFFFu), f16_bits_to_f32(e.x >> 16)),
                      pack_bf16(f16_bits_to_f32(e.y & 0xFFFFu), f16_bits_to_f32(e.y >> 16)));
}
__device__ __forceinline__ void to_bf16x4(uint2 *sval, uint32_t n, int lane) {
    for (uint32_t k = (uint32_t)lane; k < n; k += 32) sval[k] = f16x4_to_bf16x4(sval[k]);
}

// The bf16 values of the chunk-mode entry of chunk `chunk`, which lies in
// the unstaged part [lo, e) of its tile: a binary search of the ascending
// list.
__device__ __noinline__ uint2 entry_past_stage(const KVDev &X, uint32_t lo, uint32_t e,
                                               uint32_t chunk) {
    uint32_t hi = e;
    while (lo < hi) {
        const uint32_t mid = (lo + hi) >> 1;
        if (__ldg(X.out_idx + mid) < chunk) lo = mid + 1;
        else hi = mid;
    }
    const uint32_t *vv = reinterpret_cast<const uint32_t *>(X.out_val + (uint64_t)lo * 4);
    return f16x4_to_bf16x4(make_uint2(__ldg(vv), __ldg(vv + 1)));
}

// Marks the entries of the tile [a, e) that fall in the block's units
// [u0, u0 + 512) (chunks) or [u0, u0 + 2048) (elements).  Warp-collective.
template <int LC>
__device__ __forceinline__ ListView block_bits(const KVDev &X, const uint32_t *sidx, uint32_t a,
                                               uint32_t e, uint32_t u0, uint32_t *bm,
                                               uint32_t *pre, int lane) {
    ListView L{false, 0u};
    if (a >= e) return L;
    const uint32_t span = X.gran == HQMQ_GRAN_ELEMENT ? 2048u : 512u;
    __syncwarp();
    bm[lane] = 0u;
    bm[lane + 32] = 0u;
    __syncwarp();
    uint32_t below = 0;
    for (uint32_t k = (uint32_t)lane; k < e - a; k += 32) {
        const uint32_t ix = k < (uint32_t)LC ? sidx[k] : __ldg(X.out_idx + a + k);
        if (ix < u0) {
            ++below;
        } else if (ix - u0 < span) {
            const uint32_t loc = ix - u0;
            atomicOr(bm + (loc >> 5), 1u << (loc & 31));
        }
    }
    below = __reduce_add_sync(FULL, below);
    __syncwarp();
    const uint32_t ca = __popc(bm[lane]), cb = __popc(bm[lane + 32]);
    uint32_t sa = ca, sb = cb;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t ua = __shfl_up_sync(FULL, sa, d), ub = __shfl_up_sync(FULL, sb, d);
        if (lane >= d) {
            sa += ua;
            sb += ub;
        }
    }
    const uint32_t tot_a = __shfl_sync(FULL, sa, 31), tot_b = __shfl_sync(FULL, sb, 31);
    pre[lane] = sa - ca;
    pre[lane + 32] = tot_a + sb - cb;
    __syncwarp();
    L.any = tot_a + tot_b > 0;
    L.pos0 = a + below;
    return L;
}

// List position of local bit p (set in the bitmap).
__device__ __forceinline__ uint32_t list_pos(const ListView &L, const uint32_t *bm,
                                             const uint32_t *pre, uint32_t p) {
    return L.pos0 + pre[p >> 5] + __popc(bm[p >> 5] & ((1u << (p & 31)) - 1u));
}

// The 4 fp16 values of the chunk-mode entry at list position pos.
template <int LC>
__device__ __forceinline__ uint2 chunk_entry(const KVDev &X, const uint2 *sval, uint32_t a,
                                             uint32_t pos) {
    if (pos - a < (uint32_t)LC) return sval[pos - a];
    const uint32_t *vv = reinterpret_cast<const uint32_t *>(X.out_val + (uint64_t)pos * 4);
    return make_uint2(__ldg(vv), __ldg(vv + 1));
}

// Decoded values of a listed chunk, as hqmq_decode writes them (before the
// bf16 rounding): chunk mode the entry's fp16 values; element mode
// fl32(r c_e) + v_e for each listed element (v holds fl32(r c_e) on entry).
template <int LC>
__device__ __forceinline__ void patch_values(const KVDev &X, const ListView &L, const uint32_t *bm,
                                             const uint32_t *pre, const uint2 *sval, uint32_t a,
                                             uint32_t lc, float (&v)[4]) {
    if (X.gran == HQMQ_GRAN_CHUNK) {
        if (!((bm[lc >> 5] >> (lc & 31)) & 1u)) return;
        const uint2 e = chunk_entry<LC>(X, sval, a, list_pos(L, bm, pre, lc));
        v[0] = f16_bits_to_f32(e.x & 0xFFFFu);
        v[1] = f16_bits_to_f32(e.x >> 16);
        v[2] = f16_bits_to_f32(e.y & 0xFFFFu);
        v[3] = f16_bits_to_f32(e.y >> 16);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t p = 4 * lc + i;
            if ((bm[p >> 5] >> (p & 31)) & 1u)
                v[i] = __fadd_rn(v[i], f16_bits_to_f32(__ldg(X.out_val + list_pos(L, bm, pre, p))));
        }
    }
}

// Codeword of index id (id <= 24 S; id == 24 S is the zero vector).  R > 0:
// from the shared-memory table holding R copies of each codeword, lane l
// reading copy l % R, so that the 8 lanes of one 16-byte-access phase hit 8
// different bank groups (R = 8: conflict-free); R == 0: computed from the
// head's codebook.
template <int R>
__device__ __forceinline__ float4 cw_lookup(const float4 *tab, const float4 *cb, uint32_t id,
                                            uint32_t nw, int lane) {
    if constexpr (R > 0)
        return tab[id * R + (uint32_t)(lane & (R - 1))];
    else
        return id < nw ? codeword((int)(id % 24u), __ldg(cb + id / 24u))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
}

// fl32(r c) of one chunk: (v0, v1, v2, v3).
__device__ __forceinline__ void scale_cw(float r, const float4 &cw, float (&v)[4]) {
    const float2 p01 = mul2(r, cw.x, cw.y), p23 = mul2(r, cw.z, cw.w);
    v[0] = p01.x;
    v[1] = p01.y;
    v[2] = p23.x;
    v[3] = p23.y;
}

// List handling of a kernel variant: no lists, chunk-mode lists (slot maps)
// or any lists (bitmaps; element mode).
constexpr int LM_NONE = 0, LM_CHUNK = 1, LM_ANY = 2;

template <int RK, int RV, int BT, int LM, int LC, int RQ>
__global__ void __launch_bounds__(ATT_THREADS, 1) k_attn(const AttnArgs a) {
    extern __shared__ float4 s_dyn[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = lane >> 2, q = lane & 3;
    const uint32_t nw = 24u * a.S;
    const uint32_t tabk = RK > 0 ? (nw + 1) * RK : 0u, tabv = RV > 0 ? (nw + 1) * RV : 0u;
    float4 *s_tk = s_dyn, *s_tv = s_dyn + tabk;
    WarpList<LC> &WL = reinterpret_cast<WarpList<LC> *>(s_dyn + tabk + tabv)[warp];
    // chunk-mode lists: the CTA's query rows in shared memory, bf16 [ATT_G][ATT_D]
    // (rows >= G zero), for the K list's score corrections
    uint16_t *s_q = reinterpret_cast<uint16_t *>(
        reinterpret_cast<WarpList<LC> *>(s_dyn + tabk + tabv) + ATT_WARPS);
    const int head = blockIdx.x / a.cph, cta = blockIdx.x % a.cph;
    const int bb = head / a.Hk, hk = head % a.Hk;
    const float4 *cbk = a.k.cb + (size_t)hk * a.S, *cbv = a.v.cb + (size_t)hk * a.S;
    if constexpr (RK > 0) {
        for (uint32_t i = threadIdx.x; i < tabk; i += ATT_THREADS) {
            const uint32_t id = i / (uint32_t)RK;
            s_tk[i] = id < nw ? codeword((int)(id % 24u), __ldg(cbk + id / 24u)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    if constexpr (RV > 0) {
        for (uint32_t i = threadIdx.x; i < tabv; i += ATT_THREADS) {
            const uint32_t id = i / (uint32_t)RV;
            s_tv[i] = id < nw ? codeword((int)(id % 24u), __ldg(cbv + id / 24u)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    int len = a.T;
    if (a.seq_len) len = max(0, min(__ldg(a.seq_len + bb), a.T));
    const int nblk = (len + ATT_BLK - 1) / ATT_BLK;
    const int c0 = (int)((int64_t)nblk * cta / a.cph), c1 = (int)((int64_t)nblk * (cta + 1) / a.cph);
    const int wb0 = c0 + (int)((int64_t)(c1 - c0) * warp / ATT_WARPS);
    const int wb1 = c0 + (int)((int64_t)(c1 - c0) * (warp + 1) / ATT_WARPS);

    // Q as the A operand of S = Q K^T: row n; the k-slots of k-step ks are the
    // 4 elements of chunk 8 q + ks (a0: elements 0, 1; a2: elements 2, 3)
    const int G = a.G;
    uint32_t aq[8][2];
    {
        const uint2 *qr = reinterpret_cast<const uint2 *>(
            a.q + (((size_t)bb * a.Hk + hk) * G + (n < G ? n : 0)) * ATT_D);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint2 v = n < G ? __ldg(qr + 8 * q + ks) : make_uint2(0u, 0u);
            aq[ks][0] = v.x;
            aq[ks][1] = v.y;
        }
    }
    const uint64_t slab = (uint64_t)bb * a.Hk + hk;
    const uint64_t slab_g0 = slab * (uint64_t)a.T;            // packing group of token 0
    const uint32_t b = BT ? (uint32_t)BT : a.b, mask = (1u << b) - 1u;
    const uint32_t kb0 = 8u * q * b, vb0 = 4u * n * b;
    const uint32_t kbo = kb0 & 31u, vbo = vb0 & 31u;
    const uint32_t kneed = (kbo + 8 * b + 31) >> 5, vneed = (vbo + 4 * b + 31) >> 5;
    const uint32_t tps = a.tiles_per_slab;
    const uint64_t tile0 = slab * tps;
    const bool klist = LM != LM_NONE && a.k.tile_off != nullptr;
    const bool vlist = LM != LM_NONE && a.v.tile_off != nullptr;
    const bool ke = LM == LM_ANY && a.k.gran == HQMQ_GRAN_ELEMENT;
    const bool ve = LM == LM_ANY && a.v.gran == HQMQ_GRAN_ELEMENT;
    // list position of the first entry of tile rel of this slab (capped)
    auto toff = [&](const KVDev &X, int rel) -> uint32_t {
        const uint32_t r = (uint32_t)min(max(rel, 0), (int)tps);
        return min(__ldg(X.tile_off + tile0 + r), X.cap32);
    };

    float m_run = -INFINITY, l_run = 0.f;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    uint32_t kt0 = 0, kt1 = 0, kt2 = 0, kt3 = 0, vt0 = 0, vt1 = 0, vt2 = 0, vt3 = 0;
    if constexpr (LM == LM_CHUNK) {
        if (threadIdx.x < ATT_G * ATT_D / 8) {                 // 16 bytes per thread
            const int row = threadIdx.x / (ATT_D / 8), c8 = threadIdx.x % (ATT_D / 8);
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (row < a.G)
                v = __ldg(reinterpret_cast<const uint4 *>(
                              a.q + (((size_t)bb * a.Hk + hk) * a.G + row) * ATT_D) + c8);
            reinterpret_cast<uint4 *>(s_q)[threadIdx.x] = v;
        }
    }
    __syncthreads();                                           // tables ready

    LanePtrs P;
    P.kw = a.k.words + (slab_g0 + n) * b + (kb0 >> 5);
    P.vw = a.v.words + (slab_g0 + 2 * q) * b + (vb0 >> 5);
    P.kr = RQ ? nullptr : reinterpret_cast<const uint4 *>(a.k.radius + (slab_g0 + n) * 32) + q;
    P.vr = RQ ? nullptr : reinterpret_cast<const uint2 *>(a.v.radius + (slab_g0 + 2 * q) * 32) + n;
    P.krw = RQ ? a.k.rwords + (slab_g0 + n) * b + (kb0 >> 5) : nullptr;
    P.vrw = RQ ? a.v.rwords + (slab_g0 + 2 * q) * b + (vb0 >> 5) : nullptr;
    const float dk = RQ ? qr_delta(__ldg(a.k.thr + hk), nw) : 0.0f;   // radius steps (RQ)
    const float dv = RQ ? qr_delta(__ldg(a.v.thr + hk), nw) : 0.0f;
    BlockRegs<BT> cur, nxt;
    if (wb0 < wb1) load_block<BT, RQ>(P, b, wb0 * ATT_BLK, len, lane, kneed, vneed, cur);
    for (int blk = wb0; blk < wb1; ++blk) {
        const int t0 = blk * ATT_BLK;
        if (blk + 1 < wb1) load_block<BT, RQ>(P, b, t0 + ATT_BLK, len, lane, kneed, vneed, nxt);
        const int tau = t0 >> 5, par = tau & 1;
        if ((klist || vlist) && (blk == wb0 || (t0 & 31) == 0)) {
            // entering list tile tau: stage tile tau + 1, make sure tau is in
            __syncwarp();
            if (blk == wb0) {
                if (klist) {
                    kt0 = toff(a.k, tau);
                    kt1 = toff(a.k, tau + 1);
                    kt2 = toff(a.k, tau + 2);
                    stage_tile<LC>(a.k, kt0, kt1, WL.idx[par][0], WL.val[par][0], lane);
                }
                if (vlist) {
                    vt0 = toff(a.v, tau);
                    vt1 = toff(a.v, tau + 1);
                    vt2 = toff(a.v, tau + 2);
                    stage_tile<LC>(a.v, vt0, vt1, WL.idx[par][1], WL.val[par][1], lane);
                }
                cp_commit();
            } else {
                kt0 = kt1; kt1 = kt2; kt2 = kt3;
                vt0 = vt1; vt1 = vt2; vt2 = vt3;
            }
            if (klist) stage_tile<LC>(a.k, kt1, kt2, WL.idx[par ^ 1][0], WL.val[par ^ 1][0], lane);
            if (vlist) stage_tile<LC>(a.v, vt1, vt2, WL.idx[par ^ 1][1], WL.val[par ^ 1][1], lane);
            cp_commit();
            if (klist) kt3 = toff(a.k, tau + 3);
            if (vlist) vt3 = toff(a.v, tau + 3);
            cp_wait1();
            __syncwarp();
            if constexpr (LM == LM_CHUNK) {
                // the staged fp16 values of tile tau -> the bf16 that hqmq_decode writes
                if (klist) to_bf16x4(WL.val[par][0], min(kt1 - kt0, (uint32_t)LC), lane);
                if (vlist) to_bf16x4(WL.val[par][1], min(vt1 - vt0, (uint32_t)LC), lane);
                __syncwarp();
            }
        }
        const uint32_t u0 = (uint32_t)((slab_g0 + (uint64_t)t0) * 32);   // the block's first chunk
        bool kany = false, vany = false;
        uint32_t kbs = 0, kbe = 0;                             // LM_CHUNK: the block's K entries
        ListView LK{false, 0u}, LV{false, 0u};
        if constexpr (LM == LM_CHUNK) {
            if (klist && kt1 > kt0) {
                // the block's K entries: tile positions [kbs, kbe) (the list is
                // in ascending chunk order; the tile holds two blocks)
                uint32_t lo = 0, in = 0;
                for (uint32_t k = (uint32_t)lane; k < kt1 - kt0; k += 32) {
                    const uint32_t ix = k < (uint32_t)LC ? WL.idx[par][0][k] : __ldg(a.k.out_idx + kt0 + k);
                    lo += ix < u0 ? 1u : 0u;
                    in += ix - u0 < 512u ? 1u : 0u;
                }
                kbs = __reduce_add_sync(FULL, lo);
                kbe = kbs + __reduce_add_sync(FULL, in);
            }
            if (vlist) vany = map_block<LC>(a.v, WL.idx[par][1], vt0, vt1, u0, WL.map(1), lane);
        } else if constexpr (LM == LM_ANY) {
            if (klist) LK = block_bits<LC>(a.k, WL.idx[par][0], kt0, kt1, ke ? 4 * u0 : u0, WL.bm(0), WL.pre(0), lane);
            if (vlist) LV = block_bits<LC>(a.v, WL.idx[par][1], vt0, vt1, ve ? 4 * u0 : u0, WL.bm(1), WL.pre(1), lane);
            kany = LK.any;
            vany = LV.any;
        }

        // ---- scores: K^ decoded straight into B fragments; even and odd
        //      k-steps accumulate separately (two short mma chains) ----
        float sc[2][4], sd[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
            sd[j][0] = sd[j][1] = sd[j][2] = sd[j][3] = 0.f;
            Run<BT, Geo<BT>::KW> rk, rkr;
            rk.init(cur.kw[j], kbo);
            if (RQ) rkr.init(cur.krw[j], kbo);
            const uint32_t rr[4] = {cur.kr[j].x, cur.kr[j].y, cur.kr[j].z, cur.kr[j].w};
            // radius of K chunk 8 q + ks: fp16, or from its code (RQ)
            auto krad = [&](int ks) -> float {
                return RQ ? qr_radius(rkr.get(ks, b, mask), nw, dk)
                          : f16_bits_to_f32((rr[ks >> 1] >> (16 * (ks & 1))) & 0xFFFFu);
            };
            uint32_t kf0[8], kf1[8];
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t id = min(rk.get(ks, b, mask), nw);
                const float r = krad(ks);
                float v[4];
                scale_cw(r, cw_lookup<RK>(s_tk, cbk, id, nw, lane), v);
                kf0[ks] = pack_bf16(v[0], v[1]);
                kf1[ks] = pack_bf16(v[2], v[3]);
            }
            if (kany) {
                // (chunk-mode K lists are applied as score corrections below)
                const uint32_t tl = (uint32_t)(n + 8 * j);
                if constexpr (LM == LM_ANY) {
                    const uint32_t lb = ke ? WL.bm(0)[tl * 4 + q] : (WL.bm(0)[tl] >> (8 * q)) & 0xFFu;
                    if (lb) {
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks) {
                            if (!(ke ? (lb >> (4 * ks)) & 15u : (lb >> ks) & 1u)) continue;
                            float v[4] = {0.f, 0.f, 0.f, 0.f};
                            if (ke) {
                                const uint32_t id = min(rk.get(ks, b, mask), nw);
                                const float r = krad(ks);
                                scale_cw(r, cw_lookup<RK>(s_tk, cbk, id, nw, lane), v);
                            }
                            patch_values<LC>(a.k, LK, WL.bm(0), WL.pre(0), WL.val[par][0], kt0,
                                             tl * 32 + 8 * q + ks, v);
                            kf0[ks] = pack_bf16(v[0], v[1]);
                            kf1[ks] = pack_bf16(v[2], v[3]);
                        }
                    }
                }
            }
#pragma unroll
            for (int ks = 0; ks < 8; ks += 2) {
                mma_bf16(sc[j], aq[ks][0], 0u, aq[ks][1], 0u, kf0[ks], kf1[ks]);
                mma_bf16(sd[j], aq[ks + 1][0], 0u, aq[ks + 1][1], 0u, kf0[ks + 1], kf1[ks + 1]);
            }
        }

        // ---- chunk-mode K list: a listed chunk's code has radius 0, so its
        //      decoded K^ is zero above; its values enter the scores as extra
        //      k-steps: A = the query rows at the entries' chunks, B = each
        //      entry's 4 values in the column of its token (4 entries per step)
        if constexpr (LM == LM_CHUNK) {
            for (uint32_t e0 = kbs; e0 < kbe; e0 += 4) {           // (warp-uniform)
                const uint32_t e = e0 + (uint32_t)q;
                uint32_t tok = 0xFFu, c = 0u;
                uint2 v = make_uint2(0u, 0u);
                if (e < kbe) {
                    uint32_t ix;
                    if (e < (uint32_t)LC) {
                        ix = WL.idx[par][0][e];
                        v = WL.val[par][0][e];                      // (already bf16)
                    } else {
                        ix = __ldg(a.k.out_idx + kt0 + e);
                        const uint32_t *vv = reinterpret_cast<const uint32_t *>(
                            a.k.out_val + (uint64_t)(kt0 + e) * 4);
                        v = f16x4_to_bf16x4(make_uint2(__ldg(vv), __ldg(vv + 1)));
                    }
                    tok = (ix - u0) >> 5;
                    c = (ix - u0) & 31u;
                }
                const uint2 qa = *reinterpret_cast<const uint2 *>(s_q + n * ATT_D + 4 * c);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const bool hit = tok == (uint32_t)(n + 8 * j);
                    mma_bf16(sc[j], qa.x, 0u, qa.y, 0u, hit ? v.x : 0u, hit ? v.y : 0u);
                }
            }
        }

        // ---- online softmax (base 2) for row n; this lane holds tokens
        //      t0 + 8 j + 2 q + e ----
        float xs[4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                xs[2 * j + e] = t0 + 8 * j + 2 * q + e < len ? (sc[j][e] + sd[j][e]) * a.sl2 : -INFINITY;
        float bmax = fmaxf(fmaxf(xs[0], xs[1]), fmaxf(xs[2], xs[3]));
        bmax = fmaxf(bmax, __shfl_xor_sync(FULL, bmax, 1));
        bmax = fmaxf(bmax, __shfl_xor_sync(FULL, bmax, 2));
        const float m_new = fmaxf(m_run, bmax);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float corr = exp2f(m_run - m_use);
        m_run = m_new;
        float p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = exp2f(xs[i] - m_use);
        // P = P_hi + P_lo in bf16: the B fragments of O^T += V^T P^T
        const uint32_t ph0 = pack_bf16(p[0], p[1]), ph1 = pack_bf16(p[2], p[3]);
        const uint32_t pl0 = pack_bf16(p[0] - bf16_lo(ph0), p[1] - bf16_hi(ph0));
        const uint32_t pl1 = pack_bf16(p[2] - bf16_lo(ph1), p[3] - bf16_hi(ph1));
        const float lsum = ((bf16_lo(ph0) + bf16_lo(pl0)) + (bf16_hi(ph0) + bf16_hi(pl0))) +
                           ((bf16_lo(ph1) + bf16_lo(pl1)) + (bf16_hi(ph1) + bf16_hi(pl1)));
        l_run = l_run * corr + lsum;
        // this lane's accumulators hold rows 2 q and 2 q + 1
        const float ca = __shfl_sync(FULL, corr, 8 * q), cbr = __shfl_sync(FULL, corr, 8 * q + 4);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const float2 r02 = mul2(ca, acc[mt][0], acc[mt][2]);
            const float2 r13 = mul2(cbr, acc[mt][1], acc[mt][3]);
            acc[mt][0] = r02.x;
            acc[mt][2] = r02.y;
            acc[mt][1] = r13.x;
            acc[mt][3] = r13.y;
        }

        // ---- O^T += V^T P^T: V^ decoded straight into A fragments; tile
        //      2 i + h, slot n + 8 v holds element 2 h + v of chunk 4 n + i ----
        Run<BT, Geo<BT>::VW> rv[4], rvr[4];
        uint32_t lv[4] = {0u, 0u, 0u, 0u}, lvor = 0;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            rv[s].init(cur.vw[s], vbo);
            if (RQ) rvr[s].init(cur.vrw[s], vbo);
            if (vany) {
                const uint32_t tl = (uint32_t)(2 * q + (s & 1) + 8 * (s >> 1));
                if constexpr (LM == LM_CHUNK)
                    lv[s] = *reinterpret_cast<const uint32_t *>(WL.map(1) + tl * 32 + 4 * n);
                else if constexpr (LM == LM_ANY)
                    lv[s] = ve ? (WL.bm(1)[tl * 4 + (n >> 1)] >> (16 * (n & 1))) & 0xFFFFu
                               : (WL.bm(1)[tl] >> (4 * n)) & 0xFu;
                lvor |= lv[s];
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float v[4][4];
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint32_t id = min(rv[s].get(i, b, mask), nw);
                const uint32_t rw = i < 2 ? cur.vr[s].x : cur.vr[s].y;
                const float r = RQ ? qr_radius(rvr[s].get(i, b, mask), nw, dv)
                                   : f16_bits_to_f32((rw >> (16 * (i & 1))) & 0xFFFFu);
                scale_cw(r, cw_lookup<RV>(s_tv, cbv, id, nw, lane), v[s]);
            }
            if constexpr (LM == LM_CHUNK) {
                if ((lvor >> (8 * i)) & 0xFFu) {
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        const uint32_t slot = (lv[s] >> (8 * i)) & 0xFFu;
                        if (!slot) continue;
                        const uint32_t tl = (uint32_t)(2 * q + (s & 1) + 8 * (s >> 1));
                        const uint2 e = slot != 255u ? WL.val[par][1][slot - 1]
                                                     : entry_past_stage(a.v, vt0 + LC, vt1,
                                                                        u0 + tl * 32 + 4 * n + i);
                        v[s][0] = bf16_lo(e.x);
                        v[s][1] = bf16_hi(e.x);
                        v[s][2] = bf16_lo(e.y);
                        v[s][3] = bf16_hi(e.y);
                    }
                }
            } else if constexpr (LM == LM_ANY) {
                if (lvor & (ve ? 0xFu << (4 * i) : 1u << i)) {
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        if (!(ve ? (lv[s] >> (4 * i)) & 15u : (lv[s] >> i) & 1u)) continue;
                        const uint32_t tl = (uint32_t)(2 * q + (s & 1) + 8 * (s >> 1));
                        patch_values<LC>(a.v, LV, WL.bm(1), WL.pre(1), WL.val[par][1], vt0,
                                         tl * 32 + 4 * n + i, v[s]);
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t a0 = pack_bf16(v[0][2 * h], v[1][2 * h]);
                const uint32_t a1 = pack_bf16(v[0][2 * h + 1], v[1][2 * h + 1]);
                const uint32_t a2 = pack_bf16(v[2][2 * h], v[3][2 * h]);
                const uint32_t a3 = pack_bf16(v[2][2 * h + 1], v[3][2 * h + 1]);
                mma_bf16(acc[2 * i + h], a0, a1, a2, a3, ph0, ph1);
                mma_bf16(acc[2 * i + h], a0, a1, a2, a3, pl0, pl1);
            }
        }
        cur = nxt;
    }

    // ---- merge the warps' partials (the tables are no longer read) ----
    float lrow = l_run;
    lrow += __shfl_xor_sync(FULL, lrow, 1);
    lrow += __shfl_xor_sync(FULL, lrow, 2);
    __syncthreads();
    float *s_m = reinterpret_cast<float *>(s_dyn);
    float *s_l = s_m + ATT_WARPS * ATT_G;
    float *s_o = s_l + ATT_WARPS * ATT_G;                      // [warp][row][D]
    if (q == 0) {
        s_m[warp * ATT_G + n] = m_run;
        s_l[warp * ATT_G + n] = lrow;
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int row = 2 * q + (e & 1);
            const int dim = 16 * n + 4 * (mt >> 1) + 2 * (mt & 1) + (e >> 1);
            s_o[(warp * ATT_G + row) * ATT_D + dim] = acc[mt][e];
        }
    __syncthreads();
    const size_t orow0 = ((size_t)bb * a.Hk + hk) * G;        // first query head of this KV head
    float *part = a.part + ((size_t)head * a.cph + cta) * ATT_G * ATT_PART;
    for (int idx = threadIdx.x; idx < ATT_G * ATT_D; idx += ATT_THREADS) {
        const int row = idx / ATT_D, dim = idx % ATT_D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < ATT_WARPS; ++w) M = fmaxf(M, s_m[w * ATT_G + row]);
        const float mu = M == -INFINITY ? 0.f : M;
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < ATT_WARPS; ++w) {
            const float f = exp2f(s_m[w * ATT_G + row] - mu);
            L += s_l[w * ATT_G + row] * f;
            O += s_o[(w * ATT_G + row) * ATT_D + dim] * f;
        }
        if (a.cph == 1) {
            if (row < G) {
                const float val = L > 0.f ? O / L : 0.f;
                if (a.out_dtype == HQMQ_BF16)
                    reinterpret_cast<__nv_bfloat16 *>(a.o)[(orow0 + row) * ATT_D + dim] = __float2bfloat16_rn(val);
                else
                    reinterpret_cast<float *>(a.o)[(orow0 + row) * ATT_D + dim] = val;
            }
        } else {
            part[row * ATT_PART + 2 + dim] = O;
            if (dim == 0) {
                part[row * ATT_PART] = M;
                part[row * ATT_PART + 1] = L;
            }
        }
    }
    if (a.cph == 1) return;

    // ---- the last CTA of this (b, hk) merges the cph partials ----
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(a.done + head, 1u) == (unsigned)(a.cph - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const float *pall = a.part + (size_t)head * a.cph * ATT_G * ATT_PART;
    for (int idx = threadIdx.x; idx < G * ATT_D; idx += ATT_THREADS) {
        const int row = idx / ATT_D, dim = idx % ATT_D;
        float M = -INFINITY;
        for (int c = 0; c < a.cph; ++c) M = fmaxf(M, __ldcg(pall + ((size_t)c * ATT_G + row) * ATT_PART));
        const float mu = M == -INFINITY ? 0.f : M;
        float L = 0.f, O = 0.f;
        for (int c = 0; c < a.cph; ++c) {
            const float *pc = pall + ((size_t)c * ATT_G + row) * ATT_PART;
            const float f = exp2f(__ldcg(pc) - mu);
            L += __ldcg(pc + 1) * f;
            O += __ldcg(pc + 2 + dim) * f;
        }
        const float val = L > 0.f ? O / L : 0.f;
        if (a.out_dtype == HQMQ_BF16)
            reinterpret_cast<__nv_bfloat16 *>(a.o)[(orow0 + row) * ATT_D + dim] = __float2bfloat16_rn(val);
        else
            reinterpret_cast<float *>(a.o)[(orow0 + row) * ATT_D + dim] = val;
    }
    if (threadIdx.x == 0) a.done[head] = 0u;                  // ready for the next call
}

constexpr uint32_t ATT_MAX_PARTS = 1024;      // CTA partials a workspace holds

inline uint64_t attn_align256(uint64_t v) { return (v + 255) & ~(uint64_t)255; }

// Dynamic shared memory of k_attn<RK, RV, *, LM, LC> for S codewords per head.
inline size_t attn_smem(uint32_t S, int RK, int RV, int LM, int LC) {
    const size_t tab = (size_t)(24u * S + 1u) * (RK + RV) * sizeof(float4);
    const size_t list = LM == LM_NONE ? 0 : (size_t)ATT_WARPS * (48 * LC + 1024) +
                                            (LM == LM_CHUNK ? (size_t)ATT_G * ATT_D * 2 : 0);
    const size_t merge = (size_t)(2 * ATT_WARPS * ATT_G + ATT_WARPS * ATT_G * ATT_D) * sizeof(float);
    return tab + list > merge ? tab + list : merge;
}

inline KVDev kv_dev(const hqmq_kv_codes *c) {
    KVDev d;
    d.words = c->idx_words;
    d.radius = c->radius;
    d.cb = reinterpret_cast<const float4 *>(c->codebook);
    d.out_idx = c->out_idx;
    d.out_val = c->out_val;
    d.tile_off = c->out_idx && c->cap > 0 ? c->tile_off : nullptr;
    d.cap32 = c->cap < 0xFFFFFFFFull ? (uint32_t)c->cap : 0xFFFFFFFFu;
    d.gran = c->gran;
    d.rwords = c->rcode_words;
    d.thr = c->thr;
    return d;
}

// CTAs per (b, hk): the smallest count that fills at least 95% of the
// resident CTA slots of its last wave, else the best fill; every warp keeps
// at least two 16-token blocks.
inline int attn_plan(int n_heads, int T, int slots) {
    const int nblk = (T + ATT_BLK - 1) / ATT_BLK;
    int cmax = nblk / (2 * ATT_WARPS);
    if ((uint32_t)n_heads >= ATT_MAX_PARTS) cmax = 1;
    else if (cmax > (int)(ATT_MAX_PARTS / n_heads)) cmax = (int)(ATT_MAX_PARTS / n_heads);
    if (cmax < 1) cmax = 1;
    int best = 1;
    double best_eff = 0.0;
    for (int c = 1; c <= cmax; ++c) {
        const double work = (double)n_heads * c;
        const double waves = ceil(work / slots);
        const double eff = work / (waves * slots);
        if (eff >= 0.95) return c;
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
            best = c;
        }
    }
    return best;
}

template <int RK, int RV, int BT, int LM, int LC, int RQ>
static int launch_attn1(AttnArgs &a, int sm_count, cudaStream_t stream) {
    auto kern = k_attn<RK, RV, BT, LM, LC, RQ>;
    const size_t smem = attn_smem(a.S, RK, RV, LM, LC);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return HQMQ_ERR_CUDA;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, ATT_THREADS, smem) !=
            cudaSuccess || occ < 1)
        occ = 1;
    const int n_heads = a.B * a.Hk;
    a.cph = attn_plan(n_heads, a.T, sm_count * occ);
    if (a.cph > 1 && cudaMemsetAsync(a.done, 0, (size_t)n_heads * sizeof(uint32_t), stream) !=
                         cudaSuccess)
        return HQMQ_ERR_CUDA;
    kern<<<(unsigned)(n_heads * a.cph), ATT_THREADS, smem, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

template <int RK, int RV, int BT, int LM, int LC>
static int launch_attn(AttnArgs &a, int sm_count, cudaStream_t stream) {
    if (a.k.rwords) return launch_attn1<RK, RV, BT, LM, LC, 1>(a, sm_count, stream);
    return launch_attn1<RK, RV, BT, LM, LC, 0>(a, sm_count, stream);
}

}  // namespace hqmq

extern "C" uint64_t hqmq_attn_workspace_bytes(int B, int Hk) {
    using namespace hqmq;
    const uint64_t n_heads = (uint64_t)B * Hk;
    const uint64_t parts = n_heads >= ATT_MAX_PARTS ? 0 : ATT_MAX_PARTS;
    return attn_align256(n_heads * sizeof(uint32_t)) + parts * ATT_G * ATT_PART * sizeof(float);
}

extern "C" int hqmq_launch_attention(const uint16_t *q, const int *seq_len, const hqmq_kv_codes *k,
                                     const hqmq_kv_codes *v, uint32_t S, uint32_t b, int B,
                                     int Hk, int G, int T, float scale, void *o, int out_dtype,
                                     void *ws, hqmq_status *st, int sm_count, int smem_optin,
                                     cudaStream_t stream) {
    using namespace hqmq;
    AttnArgs a;
    a.q = q;
    a.seq_len = seq_len;
    a.k = kv_dev(k);
    a.v = kv_dev(v);
    a.B = B;
    a.Hk = Hk;
    a.G = G;
    a.T = T;
    a.S = S;
    a.b = b;
    a.sl2 = (float)((double)scale * 1.4426950408889634);
    a.cph = 1;
    a.tiles_per_slab = (uint32_t)((T + 31) / 32);
    a.o = o;
    a.out_dtype = out_dtype;
    a.done = reinterpret_cast<uint32_t *>(ws);
    a.part = reinterpret_cast<float *>(reinterpret_cast<char *>(ws) +
                                       attn_align256((uint64_t)B * Hk * sizeof(uint32_t)));
    a.st = reinterpret_cast<DevStatus *>(st);
    // list handling: none, chunk-mode slot maps, or bitmaps (element mode)
    const bool kl = k->out_idx && k->cap > 0, vl = v->out_idx && v->cap > 0;
    const bool any_elem = (kl && k->gran == HQMQ_GRAN_ELEMENT) || (vl && v->gran == HQMQ_GRAN_ELEMENT);
    const int lm = !kl && !vl ? LM_NONE : any_elem ? LM_ANY : LM_CHUNK;
    const size_t opt = (size_t)smem_optin;
    // the index widths of S = 8 and S = 32 (b = 8, 10): 8 K-table copies
    // (conflict-free lookups), 8 or 4 V-table copies, 192 staged entries
    if (b == 8 && attn_smem(S, 8, 8, LM_ANY, 192) <= opt) {
        if (lm == LM_NONE) return launch_attn<8, 8, 8, LM_NONE, 192>(a, sm_count, stream);
        if (lm == LM_CHUNK && attn_smem(S, 8, 8, LM_CHUNK, 192) <= opt)
            return launch_attn<8, 8, 8, LM_CHUNK, 192>(a, sm_count, stream);
        return launch_attn<8, 8, 8, LM_ANY, 192>(a, sm_count, stream);
    }
    if (b == 10 && attn_smem(S, 8, 4, LM_ANY, 192) <= opt) {
        // without lists there is no list scratch: 8 V-table copies fit too
        if (lm == LM_NONE && attn_smem(S, 8, 8, LM_NONE, 192) <= opt)
            return launch_attn<8, 8, 10, LM_NONE, 192>(a, sm_count, stream);
        if (lm == LM_NONE) return launch_attn<8, 4, 10, LM_NONE, 192>(a, sm_count, stream);
        if (lm == LM_CHUNK && attn_smem(S, 8, 4, LM_CHUNK, 192) <= opt)
            return launch_attn<8, 4, 10, LM_CHUNK, 192>(a, sm_count, stream);
        return launch_attn<8, 4, 10, LM_ANY, 192>(a, sm_count, stream);
    }
    // any other S: the most table copies that fit, 64 staged entries
    if (attn_smem(S, 8, 8, LM_ANY, 64) <= opt) return launch_attn<8, 8, 0, LM_ANY, 64>(a, sm_count, stream);
    if (attn_smem(S, 4, 4, LM_ANY, 64) <= opt) return launch_attn<4, 4, 0, LM_ANY, 64>(a, sm_count, stream);
    if (attn_smem(S, 2, 2, LM_ANY, 64) <= opt) return launch_attn<2, 2, 0, LM_ANY, 64>(a, sm_count, stream);
    if (attn_smem(S, 1, 1, LM_ANY, 64) <= opt) return launch_attn<1, 1, 0, LM_ANY, 64>(a, sm_count, stream);
    return launch_attn<0, 0, 0, LM_ANY, 64>(a, sm_count, stream);
}
