// decode.cu -- HQMQ decode: unpack -> quaternion product -> scale -> outliers.
//
// x_hat = r (q_p q_s): the stored fp16 radius times the effective codeword
// (gist.science/nl, Technische Samenvatting, Methodologie and section 1); the
// Med3x outliers kept in fp16 (section 3) are restored.  The pages run this
// inside their attention kernel ("Memory en Latentie"); here it is a
// standalone streaming kernel that writes the dense bf16 (or fp32) tensor.
//
// k_decode: each CTA owns one slab (b, h), builds that head's 24 S codeword
// table in shared memory once (S <= 170; larger S recomputes the codeword
// per chunk) and streams its chunks in units of 8 packing groups: the unit's
// index words staged in shared memory, one radius pair per lane and 64
// chunks, 8 products and one 16-byte (bf16) store per chunk pair; no block
// barriers after the table build.  Outlier list entries overwrite their
// chunk (chunk mode) or add the fp16 value to the recomputed fl32(r * c) of
// their element (element mode):
//  * with the list's tile offsets (the list position of each 1024-chunk
//    tile's first entry), inside k_decode: the warp that wrote a 256-chunk
//    quarter writes the entries of that quarter after a __syncwarp();
//  * without them, in a second launch, k_decode_outliers (one thread per
//    entry).
#include "med3_window.cuh"

namespace hqmq {

constexpr int DEC_THREADS = 256;
constexpr int OUT_THREADS = 256;

__device__ __forceinline__ uint32_t get_index(const uint32_t *__restrict__ words, uint64_t grp,
                                              uint32_t k, uint32_t b) {
    const uint32_t *w = words + grp * b;
    uint32_t bit = k * b;
    uint32_t o = bit & 31u;
    uint64_t v = __ldg(w + (bit >> 5));
    if (o + b > 32u) v |= (uint64_t)__ldg(w + (bit >> 5) + 1) << 32;
    return (uint32_t)(v >> o) & ((1u << b) - 1u);
}

// fl32(fl32(r c_e) + v) of element e of chunk j, r and c from the chunk's
// code (the main pass's product), v the list's fp16 value; a bad index gives
// r = 0.  RQ: r from the chunk's radius code (rwords, delta).
template <int RQ>
__device__ __forceinline__ float element_with_outlier(const uint32_t *__restrict__ words,
                                                     const uint16_t *__restrict__ radius,
                                                     const uint32_t *__restrict__ rwords,
                                                     float delta,
                                                     const float4 *__restrict__ cb, uint32_t S,
                                                     uint32_t b, uint64_t j, int e, uint32_t v16) {
    const uint32_t ix = get_index(words, j >> 5, (uint32_t)(j & 31u), b);
    float r = RQ ? qr_radius(get_index(rwords, j >> 5, (uint32_t)(j & 31u), b), 24u * S, delta)
                 : f16_bits_to_f32(__ldg(radius + j));
    float c = 0.0f;
    if (ix < 24u * S) {
        const float4 cw = codeword((int)(ix % 24u), __ldg(cb + ix / 24u));
        c = e == 0 ? cw.x : e == 1 ? cw.y : e == 2 ? cw.z : cw.w;
    } else {
        r = 0.0f;
    }
    return __fadd_rn(__fmul_rn(r, c), f16_bits_to_f32(v16));
}

// Main pass: every chunk -> round(fl32(r * c_i)).  A warp takes units of
// DEC_UNIT packing groups (256 chunks) of one slab: it stages the unit's
// index words in shared memory (coalesced loads) and loads the unit's radii
// (lane k: chunks 2k and 2k+1 of each 64-chunk half, one 4-byte load each,
// all in flight); per half, lane k extracts its two indices from the staged
// words, multiplies and stores its two chunks with one 16-byte (bf16) store
// (a warp store covers the half's 64 chunks).
// LISTED: 0 = no list here, HQMQ_GRAN_CHUNK + 1 / HQMQ_GRAN_ELEMENT + 1 =
// apply the list of that granularity through its tile offsets: after a unit's
// stores and a __syncwarp(), the warp writes the entries of its tile that
// fall inside the unit.
constexpr int DEC_UNIT = 8;                      // packing groups per unit
// RQ: quantized-radius mode, the radius of a chunk is fl32(k delta_h) with k
// its b-bit radius code (rwords, laid out like the index words).
template <int OUT_DT, bool TABLE, int LISTED, int RQ>
__global__ void __launch_bounds__(DEC_THREADS, 8)
k_decode(const uint32_t *__restrict__ words, const uint16_t *__restrict__ radius,
         const float4 *__restrict__ cb_all, uint32_t S, uint32_t b, int H,
         uint32_t chunks_per_slab, void *__restrict__ y, DevStatus *st,
         const uint32_t *__restrict__ tile_off, uint32_t tiles_per_slab,
         const uint32_t *__restrict__ out_idx, const uint16_t *__restrict__ out_val,
         uint32_t cap32, const uint32_t *__restrict__ rwords, const float *__restrict__ thr) {
    extern __shared__ float4 s_dyn[];
    pdl_wait();                                    // (launched with launch_pdl)
    const uint32_t n_words = 24u * S;
    float4 *s_tab = s_dyn;                         // [24 S] if TABLE
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t *s_w = reinterpret_cast<uint32_t *>(s_dyn + (TABLE ? n_words : 0)) +
                    (uint32_t)warp * DEC_UNIT * b;  // this warp's staged words
    uint32_t *s_rw = s_w + (DEC_THREADS / 32) * DEC_UNIT * b;   // its staged radius codes (RQ)
    const int slab = blockIdx.y;
    const int h = slab % H;
    const float4 *cb = cb_all + (size_t)h * S;
    const float delta = RQ ? qr_delta(__ldg(thr + h), n_words) : 0.0f;
    if (TABLE) {
        for (uint32_t i = threadIdx.x; i < n_words; i += DEC_THREADS)
            s_tab[i] = codeword((int)(i % 24u), __ldg(cb + i / 24u));
        __syncthreads();
    }
    const uint32_t gps = chunks_per_slab / 32;
    const uint64_t gs0 = (uint64_t)slab * gps;     // the slab's first packing group
    const uint32_t n_units = (gps + DEC_UNIT - 1) / DEC_UNIT;
    const uint32_t mask = (1u << b) - 1u;
    const uint32_t warp_g = blockIdx.x * (DEC_THREADS / 32) + (uint32_t)warp;
    const uint32_t n_warps = gridDim.x * (DEC_THREADS / 32);
    unsigned n_bad = 0;
    for (uint32_t un = warp_g; un < n_units; un += n_warps) {
        const uint32_t g0 = un * DEC_UNIT;
        const uint32_t ng = min((uint32_t)DEC_UNIT, gps - g0);
        const uint64_t gg0 = gs0 + g0;             // global packing group of the unit
        // lane k: chunks 2k, 2k+1 of each 64-chunk half of the unit (u < 4):
        // one 4-byte radius pair, one 16-byte (bf16) store per lane
        uint32_t rr[DEC_UNIT / 2];
#pragma unroll
        for (int u = 0; u < DEC_UNIT / 2; ++u)     // radius pairs: all in flight
            rr[u] = (!RQ && (uint32_t)(u * 64 + 2 * lane) < ng * 32u)
                        ? __ldcs(reinterpret_cast<const uint32_t *>(radius + gg0 * 32) + u * 32 + lane)
                        : 0u;
        __syncwarp();                              // (the previous unit's reads of s_w)
        for (uint32_t i = lane; i < ng * b; i += 32) {
            s_w[i] = __ldg(words + gg0 * b + i);
            if (RQ) s_rw[i] = __ldcs(rwords + gg0 * b + i);
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < DEC_UNIT / 2; ++u) {
            if ((uint32_t)(2 * u) >= ng) break;
            const uint32_t c = (uint32_t)u * 64 + 2u * lane;        // chunk within the unit
            // (a unit with an odd number of groups ends inside its last half:
            // lanes past it neither load nor store)
            const bool live = c < ng * 32u;
            uint32_t ixs[2], rks[2] = {0u, 0u};
            if (b <= 16) {                         // both indices from one 64-bit window
                const uint32_t bit = c * b, o = bit & 31u;
                const uint32_t *sw = s_w + (bit >> 5);
                const uint64_t w64 = (uint64_t)sw[0] | ((uint64_t)(o + 2 * b > 32u ? sw[1] : 0u) << 32);
                ixs[0] = (uint32_t)(w64 >> o) & mask;
                ixs[1] = (uint32_t)(w64 >> (o + b)) & mask;
                if (RQ) {
                    const uint32_t *sr = s_rw + (bit >> 5);
                    const uint64_t r64 = (uint64_t)sr[0] | ((uint64_t)(o + 2 * b > 32u ? sr[1] : 0u) << 32);
                    rks[0] = (uint32_t)(r64 >> o) & mask;
                    rks[1] = (uint32_t)(r64 >> (o + b)) & mask;
                }
            } else {
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                    const uint32_t bit = (c + v) * b, o = bit & 31u;
                    const uint32_t *sw = s_w + (bit >> 5);
                    ixs[v] = __funnelshift_r(sw[0], o + b > 32u ? sw[1] : 0u, o) & mask;
                    if (RQ) {
                        const uint32_t *sr = s_rw + (bit >> 5);
                        rks[v] = __funnelshift_r(sr[0], o + b > 32u ? sr[1] : 0u, o) & mask;
                    }
                }
            }
            float out[8];
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                float r = RQ ? qr_radius(rks[v], n_words, delta)
                             : f16_bits_to_f32(v ? (rr[u] >> 16) : (rr[u] & 0xFFFFu));
                float4 cw;
                if (ixs[v] < n_words) {
                    cw = TABLE ? s_tab[ixs[v]] : codeword((int)(ixs[v] % 24u), __ldg(cb + ixs[v] / 24u));
                } else {
                    cw = make_float4(0.f, 0.f, 0.f, 0.f);
                    r = 0.0f;
                    n_bad += live ? 1u : 0u;
                }
                out[4 * v] = __fmul_rn(r, cw.x);
                out[4 * v + 1] = __fmul_rn(r, cw.y);
                out[4 * v + 2] = __fmul_rn(r, cw.z);
                out[4 * v + 3] = __fmul_rn(r, cw.w);
            }
            const uint64_t j = gg0 * 32 + c;
            if (!live) {
            } else if (OUT_DT == HQMQ_BF16) {
                __nv_bfloat162 a0 = __floats2bfloat162_rn(out[0], out[1]);
                __nv_bfloat162 a1 = __floats2bfloat162_rn(out[2], out[3]);
                __nv_bfloat162 a2 = __floats2bfloat162_rn(out[4], out[5]);
                __nv_bfloat162 a3 = __floats2bfloat162_rn(out[6], out[7]);
                uint4 q;
                q.x = *reinterpret_cast<uint32_t *>(&a0);
                q.y = *reinterpret_cast<uint32_t *>(&a1);
                q.z = *reinterpret_cast<uint32_t *>(&a2);
                q.w = *reinterpret_cast<uint32_t *>(&a3);
                reinterpret_cast<uint4 *>(y)[j >> 1] = q;
            } else {
                float4 *yp = reinterpret_cast<float4 *>(y) + j;
                yp[0] = make_float4(out[0], out[1], out[2], out[3]);
                yp[1] = make_float4(out[4], out[5], out[6], out[7]);
            }
        }
        if (LISTED) {
            // the list entries of this unit [q0, q1) (chunk indices), from
            // its tile's list range; ordered after the warp's stores above
            __syncwarp();
            const uint64_t q0 = gg0 * 32, q1 = (gg0 + ng) * 32;
            const uint64_t gt = (uint64_t)slab * tiles_per_slab + g0 / TILE_GROUPS;
            const uint32_t a = __ldg(tile_off + gt);
            uint32_t e = __ldg(tile_off + gt + 1);
            if (e > cap32) e = cap32;
            for (uint32_t k0 = a; k0 < e; k0 += 32) {
                const uint32_t k = k0 + (uint32_t)lane;
                if (k >= e) break;
                const uint32_t qi = __ldg(out_idx + k);
                if (LISTED == HQMQ_GRAN_CHUNK + 1) {
                    if (qi < q0 || qi >= q1) continue;
                    const uint32_t *vv = reinterpret_cast<const uint32_t *>(out_val + (uint64_t)k * 4);
                    const uint32_t v01 = __ldg(vv), v23 = __ldg(vv + 1);
                    const float f0 = f16_bits_to_f32(v01 & 0xFFFFu), f1 = f16_bits_to_f32(v01 >> 16);
                    const float f2 = f16_bits_to_f32(v23 & 0xFFFFu), f3 = f16_bits_to_f32(v23 >> 16);
                    if (OUT_DT == HQMQ_BF16) {
                        __nv_bfloat162 a0 = __floats2bfloat162_rn(f0, f1);
                        __nv_bfloat162 a1 = __floats2bfloat162_rn(f2, f3);
                        uint2 o;
                        o.x = *reinterpret_cast<uint32_t *>(&a0);
                        o.y = *reinterpret_cast<uint32_t *>(&a1);
                        reinterpret_cast<uint2 *>(y)[qi] = o;
                    } else {
                        reinterpret_cast<float4 *>(y)[qi] = make_float4(f0, f1, f2, f3);
                    }
                } else {
                    const uint64_t jq = qi >> 2;
                    if (jq < q0 || jq >= q1) continue;
                    const float val = element_with_outlier<RQ>(words, radius, rwords, delta, cb, S,
                                                               b, jq, (int)(qi & 3u),
                                                               __ldg(out_val + k));
                    if (OUT_DT == HQMQ_BF16)
                        reinterpret_cast<__nv_bfloat16 *>(y)[qi] = __float2bfloat16_rn(val);
                    else
                        reinterpret_cast<float *>(y)[qi] = val;
                }
            }
        }
    }
    unsigned nb = __reduce_add_sync(FULL, n_bad);
    if (lane == 0 && nb && st) atomicOr(&st->flags, HQMQ_FLAG_BAD_INDEX);
}

// Outlier pass, one thread per list entry below cap (after the main pass, on
// the same stream).  Chunk mode: the chunk becomes round(fp16 values).
// Element mode: the element becomes round(fl32(fl32(r * c_e) + v)), with
// r * c_e recomputed from the chunk's code exactly as the main pass does.
// Entries whose index lies outside the tensor are skipped.
template <int OUT_DT, int GRAN>
__global__ void __launch_bounds__(OUT_THREADS)
k_decode_outliers(const uint32_t *__restrict__ words, const uint16_t *__restrict__ radius,
                  const float4 *__restrict__ cb_all, uint32_t S, uint32_t b, int H,
                  uint32_t chunks_per_slab, uint64_t n_chunks,
                  const uint32_t *__restrict__ out_idx, const uint16_t *__restrict__ out_val,
                  const uint32_t *__restrict__ slab_off, uint64_t n_slabs, uint64_t cap,
                  void *__restrict__ y) {
    uint64_t n = slab_off[n_slabs];
    if (n > cap) n = cap;
    const uint64_t stride = (uint64_t)gridDim.x * OUT_THREADS;
    for (uint64_t q0 = (uint64_t)blockIdx.x * OUT_THREADS + threadIdx.x; q0 < n;
         q0 += 4 * stride) {
        uint32_t ev[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {                 // four independent entries in flight
            const uint64_t q = q0 + u * stride;
            ev[u] = q < n ? __ldg(out_idx + q) : 0xFFFFFFFFu;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint64_t q = q0 + u * stride;
            if (q >= n) break;
            const uint64_t e = ev[u];
            if (GRAN == HQMQ_GRAN_CHUNK) {
                if (e >= n_chunks) continue;
                const uint32_t *vv = reinterpret_cast<const uint32_t *>(out_val + q * 4);
                const uint32_t v01 = __ldg(vv), v23 = __ldg(vv + 1);
                const float f0 = f16_bits_to_f32(v01 & 0xFFFFu), f1 = f16_bits_to_f32(v01 >> 16);
                const float f2 = f16_bits_to_f32(v23 & 0xFFFFu), f3 = f16_bits_to_f32(v23 >> 16);
                if (OUT_DT == HQMQ_BF16) {
                    __nv_bfloat162 a0 = __floats2bfloat162_rn(f0, f1);
                    __nv_bfloat162 a1 = __floats2bfloat162_rn(f2, f3);
                    uint2 o;
                    o.x = *reinterpret_cast<uint32_t *>(&a0);
                    o.y = *reinterpret_cast<uint32_t *>(&a1);
                    reinterpret_cast<uint2 *>(y)[e] = o;
                } else {
                    reinterpret_cast<float4 *>(y)[e] = make_float4(f0, f1, f2, f3);
                }
            } else {
                if (e >= 4 * n_chunks) continue;
                const uint64_t j = e >> 2;
                const int i = (int)(e & 3u);
                const int h = (int)((j / chunks_per_slab) % (uint64_t)H);
                const uint32_t ix = get_index(words, j >> 5, (uint32_t)(j & 31u), b);
                float r = f16_bits_to_f32(__ldg(radius + j));
                float c = 0.0f;
                if (ix < 24u * S) {
                    const float4 cw = codeword((int)(ix % 24u), __ldg(cb_all + (size_t)h * S + ix / 24u));
                    c = i == 0 ? cw.x : i == 1 ? cw.y : i == 2 ? cw.z : cw.w;
                } else {
                    r = 0.0f;
                }
                const float val = __fadd_rn(__fmul_rn(r, c), f16_bits_to_f32(__ldg(out_val + q)));
                if (OUT_DT == HQMQ_BF16)
                    reinterpret_cast<__nv_bfloat16 *>(y)[e] = __float2bfloat16_rn(val);
                else
                    reinterpret_cast<float *>(y)[e] = val;
            }
        }
    }
}

template <int OUT_DT, bool TABLE, int LISTED, int RQ = 0>
static int launch_main(const uint32_t *words, const uint16_t *radius, const float *cb, uint32_t S,
                       uint32_t b, int B, int H, uint32_t cps, void *y, hqmq_status *st,
                       const uint32_t *tile_off, const uint32_t *out_idx, const uint16_t *out_val,
                       uint64_t cap, int sm_count, cudaStream_t stream,
                       const uint32_t *rwords = nullptr, const float *thr = nullptr) {
    auto kern = k_decode<OUT_DT, TABLE, LISTED, RQ>;
    const size_t smem = (TABLE ? (size_t)24 * S * sizeof(float4) : 0) +
                        (size_t)(RQ ? 2 : 1) * (DEC_THREADS / 32) * DEC_UNIT * b * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return HQMQ_ERR_CUDA;
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, DEC_THREADS, smem) !=
            cudaSuccess || occ < 1)
        occ = 1;
    const int n_slabs = B * H;
    const uint32_t gps = cps / 32;
    const uint64_t units = (gps + DEC_UNIT - 1) / DEC_UNIT;
    const uint64_t want = (units + DEC_THREADS / 32 - 1) / (DEC_THREADS / 32);
    const uint64_t fill = ((uint64_t)sm_count * occ + n_slabs - 1) / n_slabs;
    uint64_t gx = want < fill ? want : fill;
    if (gx < 1) gx = 1;
    const uint32_t tps = (gps + TILE_GROUPS - 1) / TILE_GROUPS;
    const uint32_t cap32 = cap < 0xFFFFFFFFull ? (uint32_t)cap : 0xFFFFFFFFu;
    dim3 grid((unsigned)gx, (unsigned)n_slabs);
    if (launch_pdl(kern, grid, dim3(DEC_THREADS), smem, stream, words, radius,
                   reinterpret_cast<const float4 *>(cb), S, b, H, cps, y,
                   reinterpret_cast<DevStatus *>(st), tile_off, tps, out_idx, out_val, cap32,
                   rwords, thr) != cudaSuccess)
        return HQMQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

template <int OUT_DT, bool TABLE>
static int launch_main_l(int listed, const uint32_t *words, const uint16_t *radius,
                         const float *cb, uint32_t S, uint32_t b, int B, int H, uint32_t cps,
                         void *y, hqmq_status *st, const uint32_t *tile_off,
                         const uint32_t *out_idx, const uint16_t *out_val, uint64_t cap, int sm,
                         cudaStream_t stream) {
    if (listed == HQMQ_GRAN_CHUNK + 1)
        return launch_main<OUT_DT, TABLE, HQMQ_GRAN_CHUNK + 1>(
            words, radius, cb, S, b, B, H, cps, y, st, tile_off, out_idx, out_val, cap, sm, stream);
    if (listed == HQMQ_GRAN_ELEMENT + 1)
        return launch_main<OUT_DT, TABLE, HQMQ_GRAN_ELEMENT + 1>(
            words, radius, cb, S, b, B, H, cps, y, st, tile_off, out_idx, out_val, cap, sm, stream);
    return launch_main<OUT_DT, TABLE, 0>(words, radius, cb, S, b, B, H, cps, y, st, nullptr,
                                         nullptr, nullptr, 0, sm, stream);
}

template <int OUT_DT>
static int launch_out(int gran, const uint32_t *words, const uint16_t *radius, const float *cb,
                      uint32_t S, uint32_t b, int B, int H, uint32_t cps,
                      const uint32_t *out_idx, const uint16_t *out_val, const uint32_t *slab_off,
                      uint64_t cap, void *y, int sm_count, cudaStream_t stream) {
    const uint64_t n_slabs = (uint64_t)B * H;
    const uint64_t n_chunks = n_slabs * cps;
    // the list length is only known on the device: size the grid for cap
    uint64_t blocks = (cap + OUT_THREADS - 1) / OUT_THREADS;
    const uint64_t max_blocks = (uint64_t)sm_count * 8;
    if (blocks > max_blocks) blocks = max_blocks;
    if (blocks < 1) blocks = 1;
    const float4 *cb4 = reinterpret_cast<const float4 *>(cb);
    if (gran == HQMQ_GRAN_CHUNK)
        k_decode_outliers<OUT_DT, HQMQ_GRAN_CHUNK><<<(unsigned)blocks, OUT_THREADS, 0, stream>>>(
            words, radius, cb4, S, b, H, cps, n_chunks, out_idx, out_val, slab_off, n_slabs, cap,
            y);
    else
        k_decode_outliers<OUT_DT, HQMQ_GRAN_ELEMENT><<<(unsigned)blocks, OUT_THREADS, 0, stream>>>(
            words, radius, cb4, S, b, H, cps, n_chunks, out_idx, out_val, slab_off, n_slabs, cap,
            y);
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}

template <int OUT_DT>
static int launch_all(bool table, int gran, const uint32_t *words, const uint16_t *radius,
                      const float *cb, uint32_t S, uint32_t b, const uint32_t *out_idx,
                      const uint16_t *out_val, const uint32_t *slab_off, const uint32_t *tile_off,
                      uint64_t cap, int B, int H, uint32_t cps, void *y, hqmq_status *st, int sm,
                      cudaStream_t stream) {
    const bool has_list = out_idx != nullptr && cap > 0;
    // with the list's tile offsets the main pass applies the list itself
    const int listed = has_list && tile_off ? gran + 1 : 0;
    int rc = table ? launch_main_l<OUT_DT, true>(listed, words, radius, cb, S, b, B, H, cps, y, st,
                                                 tile_off, out_idx, out_val, cap, sm, stream)
                   : launch_main_l<OUT_DT, false>(listed, words, radius, cb, S, b, B, H, cps, y,
                                                  st, tile_off, out_idx, out_val, cap, sm, stream);
    if (rc != HQMQ_OK || !has_list || listed) return rc;
    return launch_out<OUT_DT>(gran, words, radius, cb, S, b, B, H, cps, out_idx, out_val, slab_off,
                              cap, y, sm, stream);
}

}  // namespace hqmq

extern "C" int hqmq_launch_decode(const uint32_t *words, const uint16_t *radius, const float *cb,
                                  uint32_t S, uint32_t b, const uint32_t *out_idx,
                                  const uint16_t *out_val, const uint32_t *slab_off,
                                  const uint32_t *tile_off, uint64_t cap, int gran, int B, int H,
                                  int T, int D, void *y, int out_dtype, hqmq_status *st,
                                  int sm_count, cudaStream_t stream) {
    using namespace hqmq;
    const uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    const bool table = S <= 170;
    if (out_dtype == HQMQ_BF16)
        return launch_all<HQMQ_BF16>(table, gran, words, radius, cb, S, b, out_idx, out_val,
                                     slab_off, tile_off, cap, B, H, cps, y, st, sm_count, stream);
    return launch_all<HQMQ_F32>(table, gran, words, radius, cb, S, b, out_idx, out_val, slab_off,
                                tile_off, cap, B, H, cps, y, st, sm_count, stream);
}

// Quantized-radius decode: as hqmq_launch_decode, the radius of chunk j being
// fl32(k_j delta_h) (k_j its radius code, delta_h = fl32(thr_h / (24 S - 1))).
// A list needs its tile offsets (applied in the main pass).
extern "C" int hqmq_launch_decode_qr(const uint32_t *words, const uint32_t *rwords, const float *thr,
                                     const float *cb, uint32_t S, uint32_t b,
                                     const uint32_t *out_idx, const uint16_t *out_val,
                                     const uint32_t *tile_off, uint64_t cap, int gran, int B, int H,
                                     int T, int D, void *y, int out_dtype, hqmq_status *st,
                                     int sm_count, cudaStream_t stream) {
    using namespace hqmq;
    const uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    const bool table = S <= 170;
    const bool listed = out_idx != nullptr && cap > 0 && tile_off != nullptr;
    const int L = listed ? gran + 1 : 0;
#define HQMQ_QR_LAUNCH(DT, TB, LS)                                                              \
    return launch_main<DT, TB, LS, 1>(words, nullptr, cb, S, b, B, H, cps, y, st,               \
                                      LS ? tile_off : nullptr, LS ? out_idx : nullptr,           \
                                      LS ? out_val : nullptr, LS ? cap : 0, sm_count, stream,    \
                                      rwords, thr)
    if (out_dtype == HQMQ_BF16) {
        if (table) {
            if (L == HQMQ_GRAN_CHUNK + 1) HQMQ_QR_LAUNCH(HQMQ_BF16, true, HQMQ_GRAN_CHUNK + 1);
            if (L == HQMQ_GRAN_ELEMENT + 1) HQMQ_QR_LAUNCH(HQMQ_BF16, true, HQMQ_GRAN_ELEMENT + 1);
            HQMQ_QR_LAUNCH(HQMQ_BF16, true, 0);
        }
        if (L == HQMQ_GRAN_CHUNK + 1) HQMQ_QR_LAUNCH(HQMQ_BF16, false, HQMQ_GRAN_CHUNK + 1);
        if (L == HQMQ_GRAN_ELEMENT + 1) HQMQ_QR_LAUNCH(HQMQ_BF16, false, HQMQ_GRAN_ELEMENT + 1);
        HQMQ_QR_LAUNCH(HQMQ_BF16, false, 0);
    }
    if (table) {
        if (L == HQMQ_GRAN_CHUNK + 1) HQMQ_QR_LAUNCH(HQMQ_F32, true, HQMQ_GRAN_CHUNK + 1);
        if (L == HQMQ_GRAN_ELEMENT + 1) HQMQ_QR_LAUNCH(HQMQ_F32, true, HQMQ_GRAN_ELEMENT + 1);
        HQMQ_QR_LAUNCH(HQMQ_F32, true, 0);
    }
    if (L == HQMQ_GRAN_CHUNK + 1) HQMQ_QR_LAUNCH(HQMQ_F32, false, HQMQ_GRAN_CHUNK + 1);
    if (L == HQMQ_GRAN_ELEMENT + 1) HQMQ_QR_LAUNCH(HQMQ_F32, false, HQMQ_GRAN_ELEMENT + 1);
    HQMQ_QR_LAUNCH(HQMQ_F32, false, 0);
#undef HQMQ_QR_LAUNCH
}
