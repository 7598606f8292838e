// codebook.cu -- secondary codebook generator.
//
// HQMQ's secondary codebook is S random unit quaternions per (layer, head,
// role), drawn with no calibration data and seeded (gist.science/nl, Technische
// Samenvatting, section 1; arXiv 2605.27646 abstract).  A normalised Gaussian
// 4-vector is Haar-uniform on S^3.  The generator is counter-based, so every
// (group, s) is drawn independently by one thread and any sub-range of groups
// reproduces the same rows.
#include "hqmq_device.cuh"

namespace hqmq {

// Philox4x32-10 (Salmon et al., SC'11): ten rounds of the multiply-xor S-box
// with multipliers 0xD2511F53 / 0xCD9E8D57; the key is bumped by the Weyl
// constants 0x9E3779B9 / 0xBB67AE85 between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        uint32_t lo_a = 0xD2511F53u * c.x, hi_a = __umulhi(0xD2511F53u, c.x);
        uint32_t lo_b = 0xCD9E8D57u * c.z, hi_b = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi_b ^ c.y ^ k0, lo_b, hi_a ^ c.w ^ k1, lo_a);
    }
    return c;
}

__global__ void k_codebook(uint64_t seed, uint32_t S, uint32_t n_groups, uint32_t group0,
                           float4 *__restrict__ out) {
    uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (uint64_t)n_groups * S) return;
    uint32_t gl = (uint32_t)(i / S), s = (uint32_t)(i % S);
    uint4 v = philox4x32_10(make_uint4(s, group0 + gl, 0u, 0u), (uint32_t)seed,
                            (uint32_t)(seed >> 32));
    const double two_pi = 6.283185307179586;     // fp64 nearest to 2 pi
    const double scale = 2.3283064365386963e-10;  // 2^-32
    // u = (v + 1/2) 2^-32 in (0, 1): both steps are exact in fp64
    double u0 = __dmul_rn((double)v.x + 0.5, scale);
    double u1 = __dmul_rn((double)v.y + 0.5, scale);
    double u2 = __dmul_rn((double)v.z + 0.5, scale);
    double u3 = __dmul_rn((double)v.w + 0.5, scale);
    // Box & Muller (1958): two independent N(0,1) per pair of uniforms
    double rad0 = __dsqrt_rn(-2.0 * log(u0));
    double rad1 = __dsqrt_rn(-2.0 * log(u2));
    double th0 = __dmul_rn(two_pi, u1);
    double th1 = __dmul_rn(two_pi, u3);
    double z0 = __dmul_rn(rad0, cos(th0));
    double z1 = __dmul_rn(rad0, sin(th0));
    double z2 = __dmul_rn(rad1, cos(th1));
    double z3 = __dmul_rn(rad1, sin(th1));
    double n2 = __dadd_rn(__dadd_rn(__dadd_rn(__dmul_rn(z0, z0), __dmul_rn(z1, z1)),
                                    __dmul_rn(z2, z2)),
                          __dmul_rn(z3, z3));
    double n = __dsqrt_rn(n2);
    float4 q;
    if (!(n > 1e-300)) {
        q = make_float4(1.0f, 0.0f, 0.0f, 0.0f);
    } else {
        q = make_float4((float)__ddiv_rn(z0, n), (float)__ddiv_rn(z1, n),
                        (float)__ddiv_rn(z2, n), (float)__ddiv_rn(z3, n));
    }
    out[i] = q;
}

}  // namespace hqmq

extern "C" int hqmq_launch_codebook(uint64_t seed, uint32_t S, uint32_t n_groups, uint32_t group0,
                                    float *d_codebook, cudaStream_t stream) {
    uint64_t n = (uint64_t)n_groups * S;
    int threads = 256;
    uint64_t blocks = (n + threads - 1) / threads;
    if (blocks > 0x7FFFFFFFull) return HQMQ_ERR_ARG;
    hqmq::k_codebook<<<(unsigned)blocks, threads, 0, stream>>>(
        seed, S, n_groups, group0, reinterpret_cast<float4 *>(d_codebook));
    return cudaGetLastError() == cudaSuccess ? HQMQ_OK : HQMQ_ERR_CUDA;
}
