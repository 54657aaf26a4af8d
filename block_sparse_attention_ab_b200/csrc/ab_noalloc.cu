// ab_noalloc.cu -- ab_score_noalloc: the IBCS scoring call for callers that cannot
// allocate device memory (see include/ab_attn.h). Its scratch -- mean keys, centroids,
// cluster weights and the bf16 terms of the mean keys -- lives in a fixed array in the
// library's own device memory.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/ab_attn.h"
#include "ab_kernels.h"

namespace {

constexpr size_t kScratchBytes = (size_t)AB_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// One copy per device that loads the library, resident until the process exits.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of g_scratch on the current device. In host code the symbol is only a
// host-side stand-in, so the address is looked up once per device (with that device
// current) and cached.
// A failed lookup keeps its CUDA error for ab_last_cuda_error; a device ordinal past the
// cache (more than kMaxDevices GPUs) is AB_ERR_RANGE.
ab_status scratch_on_current_device(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return ab::status_of(e);
    if (dev < 0 || dev >= kMaxDevices) return AB_ERR_RANGE;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_scratch);
        if (e != cudaSuccess) return ab::status_of(e);
        if (!ptr) return ab::status_of(cudaErrorInvalidSymbol);
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return AB_OK;
}

// The body of ab_score_noalloc.
ab_status score_noalloc(const void *q, const void *k, ab_shape s, int n_clusters, int iters,
                        float *scores, int *dev_flag, void *stream)
{
    if (!q || !k || !scores) return AB_ERR_NULL;
    if (s.B <= 0 || s.H <= 0 || s.N <= 0 || s.N_pad <= 0 || s.d <= 0) return AB_ERR_SHAPE;
    if (s.N_pad % AB_BLOCK != 0 || s.N > s.N_pad || s.N_pad - s.N >= AB_BLOCK) return AB_ERR_SHAPE;
    if (s.dtype != AB_BF16) return AB_ERR_DTYPE;
    if (s.d != 64 && s.d != 128) return AB_ERR_UNSUPPORTED;
    if (s.N_pad / AB_BLOCK > AB_MAX_BLOCKS || (long long)s.B * s.H > 65535LL) return AB_ERR_RANGE;
    if (n_clusters < 1 || n_clusters > 8) return AB_ERR_UNSUPPORTED;
    if (iters < 1 || iters > 1000) return AB_ERR_RANGE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(scores)) return AB_ERR_ALIGN;

    const ab::ScoreLayout L = ab::score_layout((size_t)s.B * s.H, (size_t)s.N_pad / AB_BLOCK,
                                               (size_t)s.N_pad / AB_BLOCK, (size_t)s.d,
                                               (size_t)n_clusters);
    if (L.total > kScratchBytes) return AB_ERR_WORKSPACE;

    void *base = nullptr;
    ab_status st = scratch_on_current_device(&base);
    if (st != AB_OK) return st;
    // Every region below is fully written by a kernel before any kernel reads it, so
    // nothing left by an earlier call needs clearing.
    uint8_t *ws = static_cast<uint8_t *>(base);
    float *kb = reinterpret_cast<float *>(ws + L.kbar);
    float *ce = reinterpret_cast<float *>(ws + L.cent);
    float *cw = reinterpret_cast<float *>(ws + L.cw);
    void *kt = ws + L.kbar_terms;
    float *ks = reinterpret_cast<float *>(ws + L.kscale);
    const int BH = s.B * s.H, nb = s.N_pad / AB_BLOCK;
    cudaStream_t cs = (cudaStream_t)stream;
    cudaError_t e = ab::launch_meankey(k, kb, kt, ks, BH, s.N, s.N_pad, s.d, cs);
    if (e == cudaSuccess)
        e = ab::launch_kmeans(q, ce, cw, nullptr, BH, s.N, s.N_pad, s.d, n_clusters, iters,
                              dev_flag, cs);
    if (e == cudaSuccess)
        e = ab::launch_score(ce, cw, kt, ks, scores, BH, nb, nb, nb, s.d, n_clusters, dev_flag, cs);
    return ab::status_of(e);
}

}  // namespace

extern "C" ab_status ab_score_noalloc(const void *q, const void *k, ab_shape s, int n_clusters,
                                      int iters, float *scores, int *dev_flag, void *stream)
{
    nvtxRangePushA("ab_score_noalloc");
    const ab_status st = score_noalloc(q, k, s, n_clusters, iters, scores, dev_flag, stream);
    nvtxRangePop();
    return st;
}
