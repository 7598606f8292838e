// med3_noalloc.cu -- hqmq_outlier_extract_noalloc: the Med3x step without a
// caller-provided workspace.
//
// The regular entry point takes its scratch (radix histograms, selection
// state, per-tile outlier counts and offsets) from a workspace the caller
// allocates.  Some callers cannot allocate device memory at all -- a serving
// engine that has reserved all of the GPU's memory for its own pool, or a hook
// that runs where a cudaMalloc/cudaFree (which may synchronise the device)
// is not allowed.  For them this file keeps the scratch in a fixed
// file-scope device array of HQMQ_NOALLOC_SCRATCH_BYTES bytes, which every
// GPU that loads the library holds until the process exits.
//
// In host code the array's name is only a host-side stand-in; its device
// address is obtained once per device with cudaGetSymbolAddress (on the
// first call made on that device, with that device current) and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/hqmq.h"

extern "C" uint64_t hqmq_med3_workspace_bytes(int B, int H, int T, int D);
extern "C" int hqmq_launch_outlier_extract(const void *x, int dtype, int B, int H, int T, int D,
                                           float C, int gran, float *rmed, float *thr,
                                           uint32_t *out_idx, uint16_t *out_val,
                                           uint32_t *slab_off, uint64_t cap, void *ws,
                                           hqmq_status *st, int sm_count, cudaStream_t stream);

static __device__ __align__(256) unsigned char g_med3_scratch[HQMQ_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int MAX_DEV = 64;
std::mutex g_mu;
void *g_ptr[MAX_DEV];
int g_sms[MAX_DEV];

// Device address of the scratch array and the SM count of the current
// device, looked up once per device.
int scratch_for_current_device(void **ptr, int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEV) return HQMQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_med3_scratch) != cudaSuccess || !p) return HQMQ_ERR_CUDA;
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return HQMQ_ERR_CUDA;
        g_ptr[dev] = p;
        g_sms[dev] = n;
    }
    *ptr = g_ptr[dev];
    *sms = g_sms[dev];
    return HQMQ_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" HQMQ_API int hqmq_outlier_extract_noalloc(const void *d_x, int dtype, int B, int H,
                                                    int T, int D, float C, int gran,
                                                    float *d_rmed, float *d_thr,
                                                    uint32_t *d_out_idx, uint16_t *d_out_val,
                                                    uint32_t *d_slab_off, uint64_t cap,
                                                    hqmq_status *d_status, void *stream) {
    // same argument rules as hqmq_outlier_extract; the scratch need is that of
    // the compact three-pass radix selection this entry point runs
    if (hqmq_outlier_workspace_size(B, H, T, D, gran) == 0) return HQMQ_ERR_ARG;
    const uint64_t need = hqmq_med3_workspace_bytes(B, H, T, D);
    if (dtype != HQMQ_BF16 && dtype != HQMQ_F32) return HQMQ_ERR_ARG;
    if (!(C > 0.0f) || !(C < 3.0e38f)) return HQMQ_ERR_ARG;
    if (!d_x || !d_rmed || !d_thr || !d_slab_off) return HQMQ_ERR_ARG;
    if (cap > 0 && (!d_out_idx || !d_out_val)) return HQMQ_ERR_ARG;
    if (!aligned(d_x, 16) || !aligned(d_rmed, 4) || !aligned(d_thr, 4) ||
        !aligned(d_slab_off, 4) || !aligned(d_out_idx, 4) || !aligned(d_out_val, 4) ||
        !aligned(d_status, 8))
        return HQMQ_ERR_ALIGN;
    if (need > HQMQ_NOALLOC_SCRATCH_BYTES) return HQMQ_ERR_WORKSPACE;
    void *ws = nullptr;
    int sms = 0;
    int rc = scratch_for_current_device(&ws, &sms);
    if (rc != HQMQ_OK) return rc;
    // every scratch word the kernels read is cleared or written first by
    // this call (the histograms are zeroed by a memset on `stream`)
    return hqmq_launch_outlier_extract(d_x, dtype, B, H, T, D, C, gran, d_rmed, d_thr, d_out_idx,
                                       d_out_val, d_slab_off, cap, ws, d_status, sms,
                                       (cudaStream_t)stream);
}
