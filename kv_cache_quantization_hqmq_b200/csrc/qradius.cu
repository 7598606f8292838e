// qradius.cu -- quantized radius: the fp16 radius of a bulk chunk as a b-bit
// level code.
//
// The pages' bit budget is about 2 log2(24 S) bits per chunk (3.79 bits per
// element at S = 8: arXiv 2605.27646 abstract), i.e. a radius code with as
// many levels as there are codewords.  With Med3x every bulk chunk has
// r <= thr_h (gist.science/nl, Technische Samenvatting, section 3), so the
// radius is quantized uniformly on [0, thr_h] into L = 24 S levels:
//   inv_h = fl32((L - 1) / thr_h), k = min(L - 1, floor(fl32(fl32(r inv_h) + 1/2)))
// (0 for a NaN radius, and for every chunk of a head whose thr is not a
// positive finite value); the code is stored in b = ceil(log2(24 S)) bits,
// packed like the indices (LSB first, b words per 32 chunks).  Decode uses
// r = fl32(k fl32(thr_h / (L - 1))).
#include "med3_window.cuh"

namespace hqmq {

constexpr int QR_THREADS = 256;

constexpr int QR_GROUPS = 4;                    // packing groups per warp pass

// Level of one fp16 radius for inverse step inv (see the file comment).
__device__ __forceinline__ uint32_t radius_level(uint16_t r16, float inv, uint32_t L) {
    const float q = __fmul_rn(f16_bits_to_f32(r16), inv);
    if (!(q == q)) return 0u;
    const float kf = floorf(__fadd_rn(q, 0.5f));
    const float lm1 = (float)(L - 1u);
    return kf >= lm1 ? L - 1u : (kf > 0.0f ? (uint32_t)kf : 0u);
}

// A warp takes QR_GROUPS packing groups of 32 chunks per pass (all radius
// loads in flight first): lane k quantizes chunk k of each and ORs its b bits
// into the warp's shared output words, which lanes < b store.
__global__ void __launch_bounds__(QR_THREADS)
k_quantize_radius(const uint16_t *__restrict__ radius, const float *__restrict__ thr, uint32_t H,
                  uint32_t groups_per_slab, uint32_t n_groups, uint32_t L, uint32_t b,
                  uint32_t *__restrict__ rwords) {
    __shared__ uint32_t s_out[QR_THREADS / 32][QR_GROUPS][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t stride = gridDim.x * (QR_THREADS / 32) * QR_GROUPS;
    const float lm1 = (float)(L - 1u);
    const uint32_t bit = (uint32_t)lane * b, w = bit >> 5, o = bit & 31u;
    for (uint32_t g0 = (blockIdx.x * (QR_THREADS / 32) + warp) * QR_GROUPS; g0 < n_groups;
         g0 += stride) {
        uint16_t r[QR_GROUPS];
#pragma unroll
        for (int u = 0; u < QR_GROUPS; ++u)
            r[u] = g0 + u < n_groups ? __ldcs(radius + (size_t)(g0 + u) * 32 + lane) : (uint16_t)0;
        __syncwarp();
#pragma unroll
        for (int u = 0; u < QR_GROUPS; ++u) s_out[warp][u][lane] = 0u;
        __syncwarp();
#pragma unroll
        for (int u = 0; u < QR_GROUPS; ++u) {
            if (g0 + u >= n_groups) break;
            const uint32_t h = ((g0 + u) / groups_per_slab) % H;
            const float t = __ldg(thr + h);
            const float inv = (t > 0.0f && !isinf(t) && L >= 2u) ? __fdiv_rn(lm1, t) : 0.0f;
            const uint32_t k = radius_level(r[u], inv, L);
            atomicOr(&s_out[warp][u][w], k << o);
            if (o + b > 32u) atomicOr(&s_out[warp][u][w + 1], k >> (32u - o));
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < QR_GROUPS; ++u)
            if (g0 + u < n_groups && (uint32_t)lane < b)
                rwords[(size_t)(g0 + u) * b + lane] = s_out[warp][u][lane];
    }
}

}  // namespace hqmq

extern "C" int hqmq_launch_quantize_radius(const uint16_t *radius, const float *thr, int B, int H,
                                           int T, int D, uint32_t S, uint32_t b, uint32_t *rwords,
                                           int sm_count, cudaStream_t stream) {
    using namespace hqmq;
    const uint32_t cps = (uint32_t)((uint64_t)T * D / 4);
    const uint32_t n_groups = (uint32_t)((uint64_t)B * H * cps / 32);   // < 2^27 by the shape rules
    uint64_t blocks = (n_groups + (QR_THREADS / 32) * QR_GROUPS - 1) / ((QR_THREADS / 32) * QR_GROUPS);
    const uint64_t max_blocks = (uint64_t)sm_count * 8;
    if (blocks > max_blocks) blocks = max_blocks;
    if (blocks < 1) blocks = 1;
    k_quantize_radius<<<(unsigned)blocks, QR_THREADS, 0, stream>>>(radius, thr, (uint32_t)H, cps / 32,
                                                                   n_groups, 24u * S, b, rwords);
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}
