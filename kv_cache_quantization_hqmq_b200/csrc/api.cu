// api.cu -- the extern "C" entry points of libhqmq declared in include/hqmq.h:
// argument validation (synchronous, before anything is enqueued) and the
// dispatch to the kernels of codebook.cu, med3.cu, encode.cu and decode.cu.
#include <cuda_runtime.h>

#include <atomic>

#include "../../include/hqmq.h"

extern "C" int hqmq_launch_codebook(uint64_t seed, uint32_t S, uint32_t n_groups, uint32_t group0,
                                    float *d_codebook, cudaStream_t stream);
extern "C" int hqmq_launch_encode(const void *x, int dtype, int B, int H, int T, int D,
                                  const float *cb, uint32_t S, uint32_t b, const float *thr,
                                  int gran, uint32_t *words, uint16_t *radius, hqmq_status *st,
                                  int sm_count, cudaStream_t stream);
extern "C" int hqmq_launch_decode(const uint32_t *words, const uint16_t *radius, const float *cb,
                                  uint32_t S, uint32_t b, const uint32_t *out_idx,
                                  const uint16_t *out_val, const uint32_t *slab_off, const uint32_t *tile_off, uint64_t cap,
                                  int gran, int B, int H, int T, int D, void *y, int out_dtype,
                                  hqmq_status *st, int sm_count, cudaStream_t stream);
extern "C" uint64_t hqmq_med3_workspace_bytes(int B, int H, int T, int D);
extern "C" int hqmq_launch_outlier_extract(const void *x, int dtype, int B, int H, int T, int D,
                                           float C, int gran, float *rmed, float *thr,
                                           uint32_t *out_idx, uint16_t *out_val,
                                           uint32_t *slab_off, uint64_t cap, void *ws,
                                           hqmq_status *st, int sm_count, cudaStream_t stream);

extern "C" uint64_t hqmq_window_workspace_bytes(int B, int H, int T, int D, int gran);
extern "C" int hqmq_launch_med3_window(const void *x, int dtype, int B, int H, int T, int D,
                                       float C, int gran, float *rmed, float *thr,
                                       uint32_t *slab_off, uint32_t *tile_off_out, uint64_t cap,
                                       void *ws, hqmq_status *st, int sm_count,
                                       cudaStream_t stream, const uint32_t **tile_off,
                                       uint32_t *tiles_per_slab);
extern "C" uint64_t hqmq_list_tile_count(int B, int H, int T, int D);
extern "C" int hqmq_launch_med3_front(const void *x, int dtype, int B, int H, int T, int D,
                                      float C, int gran, void *ws, int pass_b, int sm_count,
                                      cudaStream_t stream);
extern "C" int hqmq_launch_med3_finish(const void *x, int dtype, int B, int H, int T, int D,
                                       float C, int gran, float *rmed, float *thr,
                                       uint32_t *slab_off, uint32_t *tile_off_out, uint64_t cap,
                                       void *ws, hqmq_status *st, int sm_count,
                                       cudaStream_t stream, const uint32_t **tile_off,
                                       uint32_t *tiles_per_slab);
extern "C" int hqmq_spec_encode_supported(uint32_t b);
extern "C" int hqmq_launch_table_encode_units(const void *x, int dtype, int B, int H, int T, int D,
                                              const float *cb, uint32_t S, uint32_t b,
                                              const void *table, uint32_t *words,
                                              uint16_t *radius, hqmq_status *st, int sm_count,
                                              cudaStream_t stream);
extern "C" int hqmq_launch_spec_encode_units(const void *x, int dtype, int B, int H, int T, int D,
                                             const float *cb, uint32_t S, uint32_t b,
                                             const void *table, uint32_t *words, uint16_t *radius,
                                             void *ws, int sm_count, cudaStream_t stream);
extern "C" int hqmq_launch_spec_encode(const void *x, int dtype, int B, int H, int T, int D,
                                       const float *cb, uint32_t S, uint32_t b, const void *table,
                                       uint32_t *words, uint16_t *radius, void *ws, int sm_count,
                                       cudaStream_t stream);
extern "C" int hqmq_launch_fix_pass(const void *x, int dtype, int B, int H, int T, int D,
                                    const float *cb, uint32_t S, uint32_t b, const void *table,
                                    const float *thr, uint32_t *words, uint16_t *radius,
                                    const uint32_t *tile_off, uint64_t cap, uint32_t *out_idx,
                                    uint16_t *out_val, void *ws, hqmq_status *st, int sm_count,
                                    cudaStream_t stream,
                                    int use_cvals);
extern "C" int hqmq_launch_list_pass(const void *x, int dtype, int B, int H, int T, int D,
                                     const float *cb, uint32_t S, uint32_t b, const void *table,
                                     const float *thr, int gran, uint32_t *words,
                                     uint16_t *radius, const uint32_t *tile_off, uint64_t cap,
                                     uint32_t *out_idx, uint16_t *out_val, hqmq_status *st,
                                     int sm_count, cudaStream_t stream);
extern "C" uint64_t hqmq_lut_bytes_per_group(uint32_t S);
extern "C" uint64_t hqmq_attn_workspace_bytes(int B, int Hk);
extern "C" uint64_t hqmq_thr_extract_workspace_bytes(int B, int H, int T, int D);
extern "C" int hqmq_launch_append(const void *x, int dtype, int n_calls, int B, int H, int T, int D,
                                  const float *thr, int gran, const float *cb, uint32_t S,
                                  uint32_t b, uint32_t *words, uint16_t *radius, uint32_t *out_idx,
                                  uint16_t *out_val, uint32_t *slab_off, uint32_t *tile_off,
                                  uint32_t cap, hqmq_status *st, cudaStream_t stream);
extern "C" int hqmq_launch_outlier_extract_thr(const void *x, int dtype, int B, int H, int T, int D,
                                               const float *thr, int gran, uint32_t *out_idx,
                                               uint16_t *out_val, uint32_t *slab_off,
                                               uint32_t *tile_off, uint64_t cap, void *ws,
                                               hqmq_status *st, cudaStream_t stream);
extern "C" int hqmq_launch_quantize_radius(const uint16_t *radius, const float *thr, int B, int H,
                                           int T, int D, uint32_t S, uint32_t b, uint32_t *rwords,
                                           int sm_count, cudaStream_t stream);
extern "C" uint64_t hqmq_launch_joint_words(int B, int H, int T, int D, uint32_t S);
extern "C" void hqmq_launch_joint_block(uint32_t S, uint32_t *n, uint32_t *w);
extern "C" int hqmq_launch_pack_joint(const uint32_t *iw, const uint32_t *kw, uint32_t S, int B,
                                      int H, int T, int D, uint32_t *joint, hqmq_status *st,
                                      int sm_count, cudaStream_t stream);
extern "C" int hqmq_launch_list_flags(const uint32_t *out_idx, const uint32_t *total,
                                      uint64_t cap, uint64_t n_chunks, uint32_t *flags,
                                      int sm_count, cudaStream_t stream);
extern "C" int hqmq_launch_decode_joint(const uint32_t *joint, const float *thr, const float *cb,
                                        uint32_t S, const uint32_t *flags, const uint16_t *out_val,
                                        const uint32_t *tile_off, uint64_t cap, int B, int H,
                                        int T, int D, void *y, int out_dtype, int sm_count,
                                        cudaStream_t stream);
extern "C" int hqmq_launch_decode_qr(const uint32_t *words, const uint32_t *rwords, const float *thr,
                                     const float *cb, uint32_t S, uint32_t b,
                                     const uint32_t *out_idx, const uint16_t *out_val,
                                     const uint32_t *tile_off, uint64_t cap, int gran, int B, int H,
                                     int T, int D, void *y, int out_dtype, hqmq_status *st,
                                     int sm_count, cudaStream_t stream);
extern "C" int hqmq_launch_attention(const uint16_t *q, const int *seq_len, const hqmq_kv_codes *k,
                                     const hqmq_kv_codes *v, uint32_t S, uint32_t b, int B,
                                     int Hk, int G, int T, float scale, void *o, int out_dtype,
                                     void *ws, hqmq_status *st, int sm_count, int smem_optin,
                                     cudaStream_t stream);
extern "C" int hqmq_launch_build_search_table(const float *cb, uint32_t S, uint32_t n_groups,
                                              void *table, cudaStream_t stream);
extern "C" int hqmq_launch_encode_lut(const void *x, int dtype, int B, int H, int T, int D,
                                      const float *cb, uint32_t S, uint32_t b, const void *table,
                                      const float *thr, int gran, uint32_t *words,
                                      uint16_t *radius, hqmq_status *st, int sm_count,
                                      cudaStream_t stream);

namespace {

constexpr uint32_t S_MAX = 65535;
constexpr uint32_t JOINT_MAX_S = 2730;        // joint code: L^2 = (24 S)^2 < 2^32

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape rules shared by every call: positive sizes, D % 4 == 0, whole packing
// groups per slab ((T*D/4) % 32 == 0), at most 65535 slabs (grid y), and
// fewer than 2^32 elements (32-bit flat element indices).
bool shape_ok(int B, int H, int T, int D) {
    if (B <= 0 || H <= 0 || T <= 0 || D <= 0) return false;
    if (D % 4 != 0) return false;
    uint64_t cps = (uint64_t)T * D / 4;
    if (cps % 32 != 0) return false;
    if ((uint64_t)B * H > 65535) return false;
    if ((uint64_t)B * H * T * D >= (1ull << 32)) return false;
    return true;
}

bool dtype_ok(int d) { return d == HQMQ_BF16 || d == HQMQ_F32; }
bool gran_ok(int g) { return g == HQMQ_GRAN_CHUNK || g == HQMQ_GRAN_ELEMENT; }

// SM count of the current device, cached per device id.
int sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (dev >= 0 && dev < 64) {
        int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Opt-in shared memory per block of the current device, cached per device id.
int smem_optin() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (dev >= 0 && dev < 64) {
        int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return -1;
    if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// A coded cache of hqmq_attention_decode: pointers present and aligned.
int kv_codes_check(const hqmq_kv_codes *c) {
    if (!c || !c->idx_words || !c->codebook) return HQMQ_ERR_ARG;
    if (c->rcode_words ? !c->thr : !c->radius) return HQMQ_ERR_ARG;
    if (!aligned(c->rcode_words, 4) || !aligned(c->thr, 4)) return HQMQ_ERR_ALIGN;
    if (c->out_idx && (!c->out_val || !c->tile_off || !gran_ok(c->gran))) return HQMQ_ERR_ARG;
    if (!aligned(c->idx_words, 4) || !aligned(c->radius, 16) || !aligned(c->codebook, 16) ||
        !aligned(c->out_idx, 4) || !aligned(c->out_val, 8) || !aligned(c->tile_off, 4))
        return HQMQ_ERR_ALIGN;
    return HQMQ_OK;
}

}  // namespace

extern "C" {

const char *hqmq_version(void) { return "hqmq-b200 1.0"; }

const char *hqmq_error_string(int err) {
    switch (err) {
        case HQMQ_OK: return "ok";
        case HQMQ_ERR_ARG: return "invalid argument";
        case HQMQ_ERR_ALIGN: return "misaligned pointer";
        case HQMQ_ERR_CUDA: return "CUDA error";
        case HQMQ_ERR_WORKSPACE: return "workspace too small";
        default: return "unknown error";
    }
}

uint32_t hqmq_index_bits(uint32_t S) {
    if (S < 1 || S > S_MAX) return 0;
    uint64_t n = 24ull * S;
    uint32_t b = 0;
    while ((1ull << b) < n) ++b;
    return b;
}

uint64_t hqmq_index_words(int B, int H, int T, int D, uint32_t S) {
    uint32_t b = hqmq_index_bits(S);
    if (!b || !shape_ok(B, H, T, D)) return 0;
    return ((uint64_t)B * H * T * D / 128) * b;
}

int hqmq_make_codebook(uint64_t seed, uint32_t S, uint32_t n_groups, uint32_t group0,
                       float *d_codebook, void *stream) {
    if (S < 1 || S > S_MAX || n_groups < 1 || !d_codebook) return HQMQ_ERR_ARG;
    if ((uint64_t)group0 + n_groups > (1ull << 32)) return HQMQ_ERR_ARG;
    if (!aligned(d_codebook, 16)) return HQMQ_ERR_ALIGN;
    return hqmq_launch_codebook(seed, S, n_groups, group0, d_codebook, (cudaStream_t)stream);
}

uint64_t hqmq_outlier_workspace_size(int B, int H, int T, int D, int gran) {
    if (!shape_ok(B, H, T, D) || !gran_ok(gran)) return 0;
    return hqmq_window_workspace_bytes(B, H, T, D, gran);
}

int hqmq_outlier_extract(const void *d_x, int dtype, int B, int H, int T, int D, float C,
                         int gran, float *d_rmed, float *d_thr, uint32_t *d_out_idx,
                         uint16_t *d_out_val, uint32_t *d_slab_off, uint32_t *d_tile_off,
                         uint64_t cap, void *d_ws, uint64_t ws_bytes, hqmq_status *d_status,
                         void *stream) {
    if (!shape_ok(B, H, T, D) || !dtype_ok(dtype) || !gran_ok(gran)) return HQMQ_ERR_ARG;
    if (!(C > 0.0f) || !(C < 3.0e38f)) return HQMQ_ERR_ARG;
    if (!d_x || !d_rmed || !d_thr || !d_slab_off || !d_ws) return HQMQ_ERR_ARG;
    if (cap > 0 && (!d_out_idx || !d_out_val)) return HQMQ_ERR_ARG;
    if (!aligned(d_x, 16) || !aligned(d_rmed, 4) || !aligned(d_thr, 4) ||
        !aligned(d_slab_off, 4) || !aligned(d_tile_off, 16) || !aligned(d_ws, 256) ||
        !aligned(d_out_idx, 4) || !aligned(d_out_val, 4) || !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    if (ws_bytes < hqmq_window_workspace_bytes(B, H, T, D, gran)) return HQMQ_ERR_WORKSPACE;
    int sm = sm_count();
    if (sm <= 0) return HQMQ_ERR_CUDA;
    const uint32_t *tile_off = nullptr;
    uint32_t tps = 0;
    int rc = hqmq_launch_med3_window(d_x, dtype, B, H, T, D, C, gran, d_rmed, d_thr, d_slab_off,
                                     d_tile_off, cap, d_ws, d_status, sm, (cudaStream_t)stream,
                                     &tile_off, &tps);
    if (rc != HQMQ_OK) return rc;
    return hqmq_launch_list_pass(d_x, dtype, B, H, T, D, nullptr, 1, 5, nullptr, d_thr, gran,
                                 nullptr, nullptr, tile_off, cap, d_out_idx, d_out_val, d_status,
                                 sm, (cudaStream_t)stream);
}

uint64_t hqmq_encode_med3_workspace_size(int B, int H, int T, int D, int gran) {
    return hqmq_outlier_workspace_size(B, H, T, D, gran);
}

int hqmq_encode_med3(const void *d_x, int dtype, int B, int H, int T, int D, float C, int gran,
                     const float *d_codebook, uint32_t S, const void *d_table,
                     uint32_t *d_idx_words, uint16_t *d_radius, float *d_rmed, float *d_thr,
                     uint32_t *d_out_idx, uint16_t *d_out_val, uint32_t *d_slab_off,
                     uint32_t *d_tile_off, uint64_t cap, void *d_ws, uint64_t ws_bytes,
                     hqmq_status *d_status, void *stream) {
    if (!shape_ok(B, H, T, D) || !dtype_ok(dtype) || !gran_ok(gran)) return HQMQ_ERR_ARG;
    if (!(C > 0.0f) || !(C < 3.0e38f)) return HQMQ_ERR_ARG;
    if (S < 1 || S > S_MAX) return HQMQ_ERR_ARG;
    if (d_table && hqmq_lut_bytes_per_group(S) == 0) return HQMQ_ERR_ARG;
    if (!d_x || !d_codebook || !d_idx_words || !d_radius || !d_rmed || !d_thr || !d_slab_off ||
        !d_ws)
        return HQMQ_ERR_ARG;
    if (cap > 0 && (!d_out_idx || !d_out_val)) return HQMQ_ERR_ARG;
    if (!aligned(d_x, 16) || !aligned(d_codebook, 16) || !aligned(d_table, 16) ||
        !aligned(d_idx_words, 4) || !aligned(d_radius, 4) || !aligned(d_rmed, 4) ||
        !aligned(d_thr, 4) || !aligned(d_slab_off, 4) || !aligned(d_tile_off, 16) ||
        !aligned(d_ws, 256) ||
        !aligned(d_out_idx, 4) || !aligned(d_out_val, 4) || !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    if (ws_bytes < hqmq_window_workspace_bytes(B, H, T, D, gran)) return HQMQ_ERR_WORKSPACE;
    int sm = sm_count();
    if (sm <= 0) return HQMQ_ERR_CUDA;
    const uint32_t *tile_off = nullptr;
    uint32_t tps = 0;
    const uint32_t b = hqmq_index_bits(S);
    cudaStream_t s = (cudaStream_t)stream;
    if (d_table && gran == HQMQ_GRAN_CHUNK) {
        // one read of x: the encode pass also does pass B's work and encodes
        // speculatively; the fix-up pass then reads only the chunks that may
        // be outliers
        int rc = hqmq_launch_med3_front(d_x, dtype, B, H, T, D, C, gran, d_ws, 0, sm, s);
        if (rc == HQMQ_OK)
            rc = hqmq_spec_encode_supported(b)
                     ? hqmq_launch_spec_encode_units(d_x, dtype, B, H, T, D, d_codebook, S, b,
                                                     d_table, d_idx_words, d_radius, d_ws, sm, s)
                     : hqmq_launch_spec_encode(d_x, dtype, B, H, T, D, d_codebook, S, b, d_table,
                                               d_idx_words, d_radius, d_ws, sm, s);
        if (rc == HQMQ_OK)
            rc = hqmq_launch_med3_finish(d_x, dtype, B, H, T, D, C, gran, d_rmed, d_thr,
                                         d_slab_off, d_tile_off, cap, d_ws, d_status, sm, s,
                                         &tile_off, &tps);
        if (rc == HQMQ_OK)
            rc = hqmq_launch_fix_pass(d_x, dtype, B, H, T, D, d_codebook, S, b, d_table, d_thr,
                                      d_idx_words, d_radius, tile_off, cap, d_out_idx, d_out_val,
                                      d_ws, d_status, sm, s, hqmq_spec_encode_supported(b));
        return rc;
    }
    int rc = hqmq_launch_med3_window(d_x, dtype, B, H, T, D, C, gran, d_rmed, d_thr, d_slab_off,
                                     d_tile_off, cap, d_ws, d_status, sm, s, &tile_off, &tps);
    if (rc != HQMQ_OK) return rc;
    if (d_table)   // list and encode in the same (second) read of x
        return hqmq_launch_list_pass(d_x, dtype, B, H, T, D, d_codebook, S, b, d_table, d_thr,
                                     gran, d_idx_words, d_radius, tile_off, cap, d_out_idx,
                                     d_out_val, d_status, sm, (cudaStream_t)stream);
    rc = hqmq_launch_list_pass(d_x, dtype, B, H, T, D, nullptr, 1, 5, nullptr, d_thr, gran,
                               nullptr, nullptr, tile_off, cap, d_out_idx, d_out_val, d_status,
                               sm, (cudaStream_t)stream);
    if (rc != HQMQ_OK) return rc;
    return hqmq_launch_encode(d_x, dtype, B, H, T, D, d_codebook, S, b, d_thr, gran, d_idx_words,
                              d_radius, d_status, sm, (cudaStream_t)stream);
}

int hqmq_encode(const void *d_x, int dtype, int B, int H, int T, int D, const float *d_codebook,
                uint32_t S, const float *d_thr, int gran, uint32_t *d_idx_words,
                uint16_t *d_radius, hqmq_status *d_status, void *stream) {
    if (!shape_ok(B, H, T, D) || !dtype_ok(dtype) || !gran_ok(gran)) return HQMQ_ERR_ARG;
    if (S < 1 || S > S_MAX) return HQMQ_ERR_ARG;
    if (!d_x || !d_codebook || !d_idx_words || !d_radius) return HQMQ_ERR_ARG;
    if (!aligned(d_x, 16) || !aligned(d_codebook, 16) || !aligned(d_idx_words, 4) ||
        !aligned(d_radius, 4) || !aligned(d_thr, 4) || !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    int sm = sm_count();
    if (sm <= 0) return HQMQ_ERR_CUDA;
    return hqmq_launch_encode(d_x, dtype, B, H, T, D, d_codebook, S, hqmq_index_bits(S), d_thr,
                              gran, d_idx_words, d_radius, d_status, sm, (cudaStream_t)stream);
}

int hqmq_decode(const uint32_t *d_idx_words, const uint16_t *d_radius, const float *d_codebook,
                uint32_t S, const uint32_t *d_out_idx, const uint16_t *d_out_val,
                const uint32_t *d_slab_off, const uint32_t *d_tile_off, uint64_t cap, int gran,
                int B, int H, int T, int D, void *d_y, int out_dtype, hqmq_status *d_status,
                void *stream) {
    if (!shape_ok(B, H, T, D) || !dtype_ok(out_dtype) || !gran_ok(gran)) return HQMQ_ERR_ARG;
    if (S < 1 || S > S_MAX) return HQMQ_ERR_ARG;
    if (!d_idx_words || !d_radius || !d_codebook || !d_y) return HQMQ_ERR_ARG;
    if (d_out_idx && (!d_out_val || !d_slab_off)) return HQMQ_ERR_ARG;
    if (!aligned(d_idx_words, 4) || !aligned(d_radius, 4) || !aligned(d_codebook, 16) ||
        !aligned(d_y, 16) || !aligned(d_out_idx, 4) || !aligned(d_out_val, 4) ||
        !aligned(d_slab_off, 4) || !aligned(d_tile_off, 4) || !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    int sm = sm_count();
    if (sm <= 0) return HQMQ_ERR_CUDA;
    return hqmq_launch_decode(d_idx_words, d_radius, d_codebook, S, hqmq_index_bits(S), d_out_idx,
                              d_out_val, d_slab_off, d_out_idx ? d_tile_off : nullptr, cap, gran,
                              B, H, T, D, d_y, out_dtype, d_status, sm, (cudaStream_t)stream);
}

uint64_t hqmq_search_table_bytes(uint32_t S) { return hqmq_lut_bytes_per_group(S); }

uint64_t hqmq_list_tiles(int B, int H, int T, int D) {
    if (!shape_ok(B, H, T, D)) return 0;
    return hqmq_list_tile_count(B, H, T, D);
}

int hqmq_make_search_table(const float *d_codebook, uint32_t S, uint32_t n_groups,
                           void *d_table, void *stream) {
    if (hqmq_lut_bytes_per_group(S) == 0 || n_groups < 1 || n_groups > 65535) return HQMQ_ERR_ARG;
    if (!d_codebook || !d_table) return HQMQ_ERR_ARG;
    if (!aligned(d_codebook, 16) || !aligned(d_table, 16)) return HQMQ_ERR_ALIGN;
    return hqmq_launch_build_search_table(d_codebook, S, n_groups, d_table, (cudaStream_t)stream);
}

int hqmq_encode_lut(const void *d_x, int dtype, int B, int H, int T, int D,
                    const float *d_codebook, uint32_t S, const void *d_table, const float *d_thr,
                    int gran, uint32_t *d_idx_words, uint16_t *d_radius, hqmq_status *d_status,
                    void *stream) {
    if (!shape_ok(B, H, T, D) || !dtype_ok(dtype) || !gran_ok(gran)) return HQMQ_ERR_ARG;
    if (hqmq_lut_bytes_per_group(S) == 0) return HQMQ_ERR_ARG;
    if (!d_x || !d_codebook || !d_table || !d_idx_words || !d_radius) return HQMQ_ERR_ARG;
    if (!aligned(d_x, 16) || !aligned(d_codebook, 16) || !aligned(d_table, 16) ||
        !aligned(d_idx_words, 4) || !aligned(d_radius, 4) || !aligned(d_thr, 4) ||
        !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    int sm = sm_count();
    if (sm <= 0) return HQMQ_ERR_CUDA;
    const uint32_t b = hqmq_index_bits(S);
    if (!d_thr && hqmq_spec_encode_supported(b))
        return hqmq_launch_table_encode_units(d_x, dtype, B, H, T, D, d_codebook, S, b, d_table,
                                              d_idx_words, d_radius, d_status, sm,
                                              (cudaStream_t)stream);
    return hqmq_launch_encode_lut(d_x, dtype, B, H, T, D, d_codebook, S, b, d_table, d_thr, gran,
                                  d_idx_words, d_radius, d_status, sm, (cudaStream_t)stream);
}

uint64_t hqmq_attention_workspace_size(int B, int Hk) {
    if (B <= 0 || Hk <= 0 || (uint64_t)B * Hk > 65535) return 0;
    return hqmq_attn_workspace_bytes(B, Hk);
}

int hqmq_attention_decode(const uint16_t *d_q, const int32_t *d_seq_len, const hqmq_kv_codes *k,
                          const hqmq_kv_codes *v, uint32_t S, int B, int Hq, int Hk, int T, int D,
                          float scale, void *d_o, int out_dtype, void *d_ws, uint64_t ws_bytes,
                          hqmq_status *d_status, void *stream) {
    if (D != 128 || !shape_ok(B, Hk, T, D) || !dtype_ok(out_dtype)) return HQMQ_ERR_ARG;
    if (Hq <= 0 || Hq % Hk != 0 || Hq / Hk > 8) return HQMQ_ERR_ARG;
    if (S < 1 || S > S_MAX || !(scale == scale) || scale - scale != 0.0f) return HQMQ_ERR_ARG;
    if (!d_q || !d_o || !d_ws) return HQMQ_ERR_ARG;
    int rc = kv_codes_check(k);
    if (rc == HQMQ_OK) rc = kv_codes_check(v);
    if (rc != HQMQ_OK) return rc;
    if ((k->rcode_words == nullptr) != (v->rcode_words == nullptr)) return HQMQ_ERR_ARG;
    if (!aligned(d_q, 8) || !aligned(d_o, 4) || !aligned(d_seq_len, 4) || !aligned(d_ws, 256) ||
        !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    if (ws_bytes < hqmq_attn_workspace_bytes(B, Hk)) return HQMQ_ERR_WORKSPACE;
    const int sm = sm_count(), optin = smem_optin();
    if (sm <= 0 || optin <= 0) return HQMQ_ERR_CUDA;
    return hqmq_launch_attention(d_q, d_seq_len, k, v, S, hqmq_index_bits(S), B, Hk, Hq / Hk, T,
                                 scale, d_o, out_dtype, d_ws, d_status, sm, optin,
                                 (cudaStream_t)stream);
}

int hqmq_quantize_radius(const uint16_t *d_radius, const float *d_thr, int B, int H, int T, int D,
                         uint32_t S, uint32_t *d_rcode_words, void *stream) {
    if (!shape_ok(B, H, T, D) || S < 1 || S > S_MAX) return HQMQ_ERR_ARG;
    if (!d_radius || !d_thr || !d_rcode_words) return HQMQ_ERR_ARG;
    if (!aligned(d_radius, 2) || !aligned(d_thr, 4) || !aligned(d_rcode_words, 4))
        return HQMQ_ERR_ALIGN;
    const int sm = sm_count();
    if (sm <= 0) return HQMQ_ERR_CUDA;
    return hqmq_launch_quantize_radius(d_radius, d_thr, B, H, T, D, S, hqmq_index_bits(S),
                                       d_rcode_words, sm, (cudaStream_t)stream);
}

int hqmq_decode_qradius(const uint32_t *d_idx_words, const uint32_t *d_rcode_words,
                        const float *d_thr, const float *d_codebook, uint32_t S,
                        const uint32_t *d_out_idx, const uint16_t *d_out_val,
                        const uint32_t *d_tile_off, uint64_t cap, int gran, int B, int H, int T,
                        int D, void *d_y, int out_dtype, hqmq_status *d_status, void *stream) {
    if (!shape_ok(B, H, T, D) || !dtype_ok(out_dtype) || !gran_ok(gran)) return HQMQ_ERR_ARG;
    if (S < 1 || S > S_MAX) return HQMQ_ERR_ARG;
    if (!d_idx_words || !d_rcode_words || !d_thr || !d_codebook || !d_y) return HQMQ_ERR_ARG;
    if (d_out_idx && (!d_out_val || !d_tile_off)) return HQMQ_ERR_ARG;
    if (!aligned(d_idx_words, 4) || !aligned(d_rcode_words, 4) || !aligned(d_thr, 4) ||
        !aligned(d_codebook, 16) || !aligned(d_y, 16) || !aligned(d_out_idx, 4) ||
        !aligned(d_out_val, 4) || !aligned(d_tile_off, 4) || !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    const int sm = sm_count();
    if (sm <= 0) return HQMQ_ERR_CUDA;
    return hqmq_launch_decode_qr(d_idx_words, d_rcode_words, d_thr, d_codebook, S,
                                 hqmq_index_bits(S), d_out_idx, d_out_val,
                                 d_out_idx ? d_tile_off : nullptr, cap, gran, B, H, T, D, d_y,
                                 out_dtype, d_status, sm, (cudaStream_t)stream);
}

static bool joint_S_ok(uint32_t S) { return S >= 1 && S <= JOINT_MAX_S; }

void hqmq_joint_block(uint32_t S, uint32_t *chunks_per_block, uint32_t *bits_per_block) {
    uint32_t n = 0, w = 0;
    if (joint_S_ok(S)) hqmq_launch_joint_block(S, &n, &w);
    if (chunks_per_block) *chunks_per_block = n;
    if (bits_per_block) *bits_per_block = w;
}

uint64_t hqmq_joint_words(int B, int H, int T, int D, uint32_t S) {
    if (!shape_ok(B, H, T, D) || !joint_S_ok(S)) return 0;
    return hqmq_launch_joint_words(B, H, T, D, S);
}

int hqmq_pack_joint(const uint32_t *d_idx_words, const uint32_t *d_rcode_words, uint32_t S, int B,
                    int H, int T, int D, uint32_t *d_joint, hqmq_status *d_status, void *stream) {
    if (!shape_ok(B, H, T, D) || !joint_S_ok(S)) return HQMQ_ERR_ARG;
    if (!d_idx_words || !d_rcode_words || !d_joint) return HQMQ_ERR_ARG;
    if (!aligned(d_idx_words, 4) || !aligned(d_rcode_words, 4) || !aligned(d_joint, 4) ||
        !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    const int sm = sm_count();
    if (sm <= 0) return HQMQ_ERR_CUDA;
    return hqmq_launch_pack_joint(d_idx_words, d_rcode_words, S, B, H, T, D, d_joint, d_status,
                                  sm, (cudaStream_t)stream);
}

int hqmq_list_flags(const uint32_t *d_out_idx, const uint32_t *d_slab_off, uint64_t cap, int B,
                    int H, int T, int D, uint32_t *d_flags, void *stream) {
    if (!shape_ok(B, H, T, D)) return HQMQ_ERR_ARG;
    if (!d_slab_off || !d_flags || (cap > 0 && !d_out_idx)) return HQMQ_ERR_ARG;
    if (!aligned(d_out_idx, 4) || !aligned(d_slab_off, 4) || !aligned(d_flags, 4))
        return HQMQ_ERR_ALIGN;
    const int sm = sm_count();
    if (sm <= 0) return HQMQ_ERR_CUDA;
    const uint64_t n_chunks = (uint64_t)B * H * T * D / 4;
    return hqmq_launch_list_flags(d_out_idx, d_slab_off + (size_t)B * H, cap, n_chunks, d_flags,
                                  sm, (cudaStream_t)stream);
}

int hqmq_decode_joint(const uint32_t *d_joint, const float *d_thr, const float *d_codebook,
                      uint32_t S, const uint32_t *d_flags, const uint16_t *d_out_val,
                      const uint32_t *d_tile_off, uint64_t cap, int B, int H, int T, int D,
                      void *d_y, int out_dtype, void *stream) {
    if (!shape_ok(B, H, T, D) || !dtype_ok(out_dtype) || !joint_S_ok(S)) return HQMQ_ERR_ARG;
    if (!d_joint || !d_thr || !d_codebook || !d_y) return HQMQ_ERR_ARG;
    if (d_flags && (!d_tile_off || (cap > 0 && !d_out_val))) return HQMQ_ERR_ARG;
    if (!aligned(d_joint, 4) || !aligned(d_thr, 4) || !aligned(d_codebook, 16) ||
        !aligned(d_y, out_dtype == HQMQ_BF16 ? 8 : 16) || !aligned(d_flags, 4) ||
        !aligned(d_out_val, 4) || !aligned(d_tile_off, 4))
        return HQMQ_ERR_ALIGN;
    const int sm = sm_count();
    if (sm <= 0) return HQMQ_ERR_CUDA;
    return hqmq_launch_decode_joint(d_joint, d_thr, d_codebook, S, d_flags, d_out_val, d_tile_off,
                                    cap, B, H, T, D, d_y, out_dtype, sm, (cudaStream_t)stream);
}

uint64_t hqmq_outlier_extract_given_thr_workspace_size(int B, int H, int T, int D) {
    if (!shape_ok(B, H, T, D)) return 0;
    return hqmq_thr_extract_workspace_bytes(B, H, T, D);
}

int hqmq_outlier_extract_given_thr(const void *d_x, int dtype, int B, int H, int T, int D,
                                   const float *d_thr, int gran, uint32_t *d_out_idx,
                                   uint16_t *d_out_val, uint32_t *d_slab_off,
                                   uint32_t *d_tile_off, uint64_t cap, void *d_ws,
                                   uint64_t ws_bytes, hqmq_status *d_status, void *stream) {
    if (!shape_ok(B, H, T, D) || !dtype_ok(dtype) || !gran_ok(gran)) return HQMQ_ERR_ARG;
    if (!d_x || !d_thr || !d_slab_off || !d_ws || (cap > 0 && (!d_out_idx || !d_out_val)))
        return HQMQ_ERR_ARG;
    if (!aligned(d_x, 16) || !aligned(d_thr, 4) || !aligned(d_out_idx, 4) ||
        !aligned(d_out_val, 4) || !aligned(d_slab_off, 4) || !aligned(d_tile_off, 4) ||
        !aligned(d_ws, 256) || !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    if (ws_bytes < hqmq_thr_extract_workspace_bytes(B, H, T, D)) return HQMQ_ERR_WORKSPACE;
    return hqmq_launch_outlier_extract_thr(d_x, dtype, B, H, T, D, d_thr, gran, d_out_idx,
                                           d_out_val, d_slab_off, d_tile_off, cap, d_ws, d_status,
                                           (cudaStream_t)stream);
}

int hqmq_append_batch(const void *d_x, int dtype, int n_calls, int B, int H, int T, int D,
                      const float *d_thr, int gran, const float *d_codebook, uint32_t S,
                      uint32_t *d_idx_words, uint16_t *d_radius, uint32_t *d_out_idx,
                      uint16_t *d_out_val, uint32_t *d_slab_off, uint32_t *d_tile_off,
                      uint64_t cap, hqmq_status *d_status, void *stream) {
    if (!shape_ok(B, H, T, D) || !dtype_ok(dtype) || !gran_ok(gran)) return HQMQ_ERR_ARG;
    if (n_calls < 1 || n_calls > (1 << 30) || S < 1 || S > S_MAX) return HQMQ_ERR_ARG;
    if ((uint64_t)H * S * 16 > 160 * 1024) return HQMQ_ERR_ARG;   // codebooks of a call in smem
    if (cap >= (1ull << 32)) return HQMQ_ERR_ARG;
    if (!d_x || !d_thr || !d_codebook || !d_idx_words || !d_radius || !d_slab_off)
        return HQMQ_ERR_ARG;
    if (cap > 0 && (!d_out_idx || !d_out_val)) return HQMQ_ERR_ARG;
    if (!aligned(d_x, 16) || !aligned(d_thr, 4) || !aligned(d_codebook, 16) ||
        !aligned(d_idx_words, 4) || !aligned(d_radius, 2) || !aligned(d_out_idx, 4) ||
        !aligned(d_out_val, 8) || !aligned(d_slab_off, 4) || !aligned(d_tile_off, 4) ||
        !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    return hqmq_launch_append(d_x, dtype, n_calls, B, H, T, D, d_thr, gran, d_codebook, S,
                              hqmq_index_bits(S), d_idx_words, d_radius, d_out_idx, d_out_val,
                              d_slab_off, d_tile_off, (uint32_t)cap, d_status,
                              (cudaStream_t)stream);
}

}  // extern "C"
