// ab_api.cu -- the C ABI declared in include/ab_attn.h: host-side argument checks,
// workspace carving, and kernel launches on the caller's stream. No device memory is
// allocated here; the only state kept between calls is one side stream and two events
// per device for ab_score's concurrent mean-key pass.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/ab_attn.h"
#include "ab_kernels.h"

namespace ab {

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

ab_status status_of(cudaError_t e)
{
    if (e == cudaSuccess) return AB_OK;
    g_last_cuda_error = e;
    return AB_ERR_CUDA;
}

}  // namespace ab

namespace {

// NVTX range around each entry point (host side: argument checks and launches), so a
// timeline profiler shows which call enqueued which kernels. No cost without a tool.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ab_status check_shape(const ab_shape &s)
{
    if (s.B <= 0 || s.H <= 0 || s.N <= 0 || s.N_pad <= 0 || s.d <= 0) return AB_ERR_SHAPE;
    if (s.N_pad % AB_BLOCK != 0 || s.N > s.N_pad || s.N_pad - s.N >= AB_BLOCK) return AB_ERR_SHAPE;
    if (s.dtype != AB_BF16) return AB_ERR_DTYPE;
    if (s.d != 64 && s.d != 128) return AB_ERR_UNSUPPORTED;
    if (s.N_pad / AB_BLOCK > AB_MAX_BLOCKS) return AB_ERR_RANGE;
    // grid and index arithmetic stay in int / size_t ranges
    if ((long long)s.B * s.H > 65535LL) return AB_ERR_RANGE;
    return AB_OK;
}

ab::ScoreLayout score_layout(const ab_shape &s, int C, int unit = AB_BLOCK)
{
    return ab::score_layout((size_t)s.B * s.H, (size_t)s.N_pad / AB_BLOCK, (size_t)s.N_pad / unit,
                            (size_t)s.d, (size_t)C);
}

// key units accepted by the unit entry points: 128-token blocks (at most AB_MAX_BLOCKS
// per head, checked with the shape) or 4-token units (at most AB_MAX_UNITS per head)
ab_status check_unit(const ab_shape &s, int unit)
{
    if (unit != AB_BLOCK && unit != AB_UNIT4) return AB_ERR_UNSUPPORTED;
    if (s.N_pad / unit > AB_MAX_UNITS) return AB_ERR_RANGE;
    return AB_OK;
}

ab_status cuda_status(cudaError_t e) { return ab::status_of(e); }

// ab_score's mean keys (an HBM-bound read of K) and k-means (a latency-bound chain over Q)
// are independent: the mean keys run on a side stream forked from the caller's stream by
// an event and joined back by another before the block score. One side stream and two
// events per device, created on the device's first ab_score call and kept until exit; the
// mutex makes a call's record-wait-launch sequence atomic across host threads.
constexpr int kMaxSideDevices = 64;

struct SideStream {
    std::mutex mu;
    bool ready = false;
    cudaStream_t st = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};

SideStream g_side[kMaxSideDevices];

cudaError_t side_init(SideStream &ss)
{
    if (ss.ready) return cudaSuccess;
    cudaError_t e = cudaStreamCreateWithFlags(&ss.st, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming);
    if (e == cudaSuccess) ss.ready = true;
    return e;
}

// Mean keys and k-means of one ab_score call: concurrently through the device's side
// stream, or in sequence on the caller's stream while that stream is being captured
// into a graph (or on a device past the side-stream table).
template <typename MeanKey, typename KMeans>
cudaError_t meankey_and_kmeans(cudaStream_t cs, MeanKey meankey, KMeans kmeans)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(cs, &cap);
    if (e != cudaSuccess) {
        // the query is refused for the legacy stream while another stream captures in
        // global mode: clear that error (only it) and launch in order
        (void)cudaGetLastError();
        cap = cudaStreamCaptureStatusActive;
    }
    if (cap != cudaStreamCaptureStatusNone || dev < 0 || dev >= kMaxSideDevices) {
        e = meankey(cs);
        return e == cudaSuccess ? kmeans(cs) : e;
    }
    // k-means is enqueued first so that its CTAs take the SMs and the mean-key CTAs fill
    // the resources they leave (one per SM)
    SideStream &ss = g_side[dev];
    std::lock_guard<std::mutex> lock(ss.mu);
    e = side_init(ss);
    if (e == cudaSuccess) e = cudaEventRecord(ss.fork, cs);
    if (e == cudaSuccess) e = kmeans(cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.st, ss.fork, 0);
    if (e == cudaSuccess) e = meankey(ss.st);
    if (e == cudaSuccess) e = cudaEventRecord(ss.join, ss.st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ss.join, 0);
    return e;
}

ab_status attn_common(const void *q, const void *k, const void *v, ab_shape s, int unit,
                      const int32_t *idx, const int32_t *cnt, const float *w, void *out,
                      ab_dtype out_dtype, float *lse, int *dev_flag, void *stream,
                      unsigned long long wait_ns = 0)
{
    if (!q || !k || !v || !idx || !cnt || !out) return AB_ERR_NULL;
    ab_status st = check_shape(s);
    if (st != AB_OK) return st;
    st = check_unit(s, unit);
    if (st != AB_OK) return st;
    if (out_dtype != AB_BF16 && out_dtype != AB_F32) return AB_ERR_DTYPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(idx) ||
        !aligned16(cnt) || (w && !aligned16(w)) || (lse && !aligned16(lse)))
        return AB_ERR_ALIGN;
    ab::AttnLaunch a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.idx = idx;
    a.cnt = cnt;
    a.w = w;
    a.out = out;
    a.out_f32 = out_dtype == AB_F32;
    a.lse = lse;
    a.flag = dev_flag;
    a.B = s.B;
    a.H = s.H;
    a.N = s.N;
    a.N_pad = s.N_pad;
    a.d = s.d;
    a.unit = unit;
    a.grid_override = 0;
    a.wait_ns = wait_ns;
    return cuda_status(ab::launch_attn(a, (cudaStream_t)stream));
}

}  // namespace

extern "C" {

ab_status ab_score_workspace_size(ab_shape s, int n_clusters, size_t *bytes)
{
    if (!bytes) return AB_ERR_NULL;
    *bytes = 0;
    ab_status st = check_shape(s);
    if (st != AB_OK) return st;
    if (n_clusters < 1 || n_clusters > 8) return AB_ERR_UNSUPPORTED;
    *bytes = score_layout(s, n_clusters).total;
    return AB_OK;
}

ab_status ab_score_units_workspace_size(ab_shape s, int n_clusters, int key_unit, size_t *bytes)
{
    if (!bytes) return AB_ERR_NULL;
    *bytes = 0;
    ab_status st = check_shape(s);
    if (st != AB_OK) return st;
    st = check_unit(s, key_unit);
    if (st != AB_OK) return st;
    if (n_clusters < 1 || n_clusters > 8) return AB_ERR_UNSUPPORTED;
    *bytes = score_layout(s, n_clusters, key_unit).total;
    return AB_OK;
}

ab_status ab_score(const void *q, const void *k, ab_shape s, int n_clusters, int iters,
                   float *scores, float *kbar, float *centroids, float *cweights,
                   uint8_t *assign, void *workspace, size_t workspace_bytes, int *dev_flag,
                   void *stream)
{
    NvtxRange nvtx("ab_score");
    return ab_score_units(q, k, s, n_clusters, iters, AB_BLOCK, scores, kbar, centroids, cweights,
                          assign, workspace, workspace_bytes, dev_flag, stream);
}

ab_status ab_score_units(const void *q, const void *k, ab_shape s, int n_clusters, int iters,
                         int key_unit, float *scores, float *kbar, float *centroids,
                         float *cweights, uint8_t *assign, void *workspace,
                         size_t workspace_bytes, int *dev_flag, void *stream)
{
    NvtxRange nvtx("ab_score_units");
    if (!q || !k || !scores) return AB_ERR_NULL;
    ab_status st = check_shape(s);
    if (st != AB_OK) return st;
    st = check_unit(s, key_unit);
    if (st != AB_OK) return st;
    if (n_clusters < 1 || n_clusters > 8) return AB_ERR_UNSUPPORTED;
    if (iters < 1 || iters > 1000) return AB_ERR_RANGE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(scores) || (kbar && !aligned16(kbar)) ||
        (centroids && !aligned16(centroids)) || (cweights && !aligned16(cweights)) ||
        !aligned16(workspace))
        return AB_ERR_ALIGN;
    const ab::ScoreLayout L = score_layout(s, n_clusters, key_unit);
    if (!workspace || workspace_bytes < L.total) return AB_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *kb = kbar ? kbar : reinterpret_cast<float *>(ws + L.kbar);
    float *ce = centroids ? centroids : reinterpret_cast<float *>(ws + L.cent);
    float *cw = cweights ? cweights : reinterpret_cast<float *>(ws + L.cw);
    const int BH = s.B * s.H, nqb = s.N_pad / AB_BLOCK, nku = s.N_pad / key_unit;
    const int nku_valid = (s.N + key_unit - 1) / key_unit;  // units holding a valid token
    cudaStream_t cs = (cudaStream_t)stream;
    void *kt = ws + L.kbar_terms;
    float *ks = reinterpret_cast<float *>(ws + L.kscale);
    cudaError_t e = meankey_and_kmeans(
        cs,
        [&](cudaStream_t st) {
            return ab::launch_meankey_units(k, kb, kt, ks, BH, s.N, s.N_pad, s.d, key_unit, st);
        },
        [&](cudaStream_t st) {
            return ab::launch_kmeans(q, ce, cw, assign, BH, s.N, s.N_pad, s.d, n_clusters, iters,
                                     dev_flag, st);
        });
    if (e == cudaSuccess)
        e = ab::launch_score(ce, cw, kt, ks, scores, BH, nqb, nku, nku_valid, s.d, n_clusters,
                             dev_flag, cs);
    return cuda_status(e);
}

ab_status ab_select(const float *scores, int B, int H, int nqb, int nkb, int budget,
                    ab_mode mode, uint64_t seed, int32_t *idx, int32_t *cnt, float *w, double *p,
                    int *dev_flag, void *stream)
{
    NvtxRange nvtx("ab_select");
    if (!scores || !idx || !cnt) return AB_ERR_NULL;
    if (mode == AB_MODE_SIP && !w) return AB_ERR_NULL;
    if (mode != AB_MODE_SIP && mode != AB_MODE_TOPK) return AB_ERR_UNSUPPORTED;
    if (B <= 0 || H <= 0 || nqb <= 0 || nkb <= 0) return AB_ERR_SHAPE;
    if (nkb > AB_MAX_UNITS || budget < 1) return AB_ERR_RANGE;
    if ((long long)B * H * nqb > 2147483647LL) return AB_ERR_RANGE;
    if (!aligned16(scores) || !aligned16(idx) || !aligned16(cnt) || (w && !aligned16(w)) ||
        (p && !aligned16(p)))
        return AB_ERR_ALIGN;
    const int K = budget < nkb ? budget : nkb;
    cudaStream_t cs = (cudaStream_t)stream;
    cudaError_t e;
    if (mode == AB_MODE_SIP)
        e = ab::launch_sip(scores, B * H, H, 0, nqb, nkb, K, seed, idx, cnt, w, p, dev_flag, cs);
    else
        e = ab::launch_topk(scores, B, H, nqb, nkb, K, idx, cnt, w, dev_flag, cs);
    return cuda_status(e);
}

ab_status ab_attn_fwd(const void *q, const void *k, const void *v, ab_shape s, const int32_t *idx,
                      const int32_t *cnt, const float *w, void *out, ab_dtype out_dtype,
                      float *lse, int *dev_flag, void *stream)
{
    NvtxRange nvtx("ab_attn_fwd");
    if (!w) return AB_ERR_NULL;
    return attn_common(q, k, v, s, AB_BLOCK, idx, cnt, w, out, out_dtype, lse, dev_flag, stream);
}

ab_status ab_attn_units_fwd(const void *q, const void *k, const void *v, ab_shape s, int key_unit,
                            const int32_t *idx, const int32_t *cnt, const float *w, void *out,
                            ab_dtype out_dtype, float *lse, int *dev_flag, void *stream)
{
    NvtxRange nvtx("ab_attn_units_fwd");
    if (!w) return AB_ERR_NULL;
    return attn_common(q, k, v, s, key_unit, idx, cnt, w, out, out_dtype, lse, dev_flag, stream);
}

ab_status ab_attn_units_topk_fwd(const void *q, const void *k, const void *v, ab_shape s,
                                 int key_unit, const int32_t *idx, const int32_t *cnt, void *out,
                                 ab_dtype out_dtype, float *lse, int *dev_flag, void *stream)
{
    NvtxRange nvtx("ab_attn_units_topk_fwd");
    return attn_common(q, k, v, s, key_unit, idx, cnt, nullptr, out, out_dtype, lse, dev_flag,
                       stream);
}

ab_status ab_attn_topk_fwd(const void *q, const void *k, const void *v, ab_shape s,
                           const int32_t *idx, const int32_t *cnt, void *out, ab_dtype out_dtype,
                           float *lse, int *dev_flag, void *stream)
{
    NvtxRange nvtx("ab_attn_topk_fwd");
    return attn_common(q, k, v, s, AB_BLOCK, idx, cnt, nullptr, out, out_dtype, lse, dev_flag,
                       stream);
}

ab_status ab_selftest_attn_wait_limit(const void *q, const void *k, const void *v, ab_shape s,
                                      int key_unit, const int32_t *idx, const int32_t *cnt,
                                      const float *w, void *out, ab_dtype out_dtype, float *lse,
                                      int *dev_flag, int limit_ns, void *stream)
{
    NvtxRange nvtx("ab_selftest_attn_wait_limit");
    if (!dev_flag) return AB_ERR_NULL;
    if (limit_ns < 1 || limit_ns > 1000000000) return AB_ERR_RANGE;
    return attn_common(q, k, v, s, key_unit, idx, cnt, w, out, out_dtype, lse, dev_flag, stream,
                       (unsigned long long)limit_ns);
}

ab_status ab_check_flag(const int *dev_flag, int *host_flag, void *stream)
{
    NvtxRange nvtx("ab_check_flag");
    if (!dev_flag || !host_flag) return AB_ERR_NULL;
    cudaError_t e = cudaMemcpyAsync(host_flag, dev_flag, sizeof(int), cudaMemcpyDeviceToHost,
                                    (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e);
    if (*host_flag == 0) return AB_OK;
    if (*host_flag & AB_FLAG_TIMEOUT) return AB_ERR_TIMEOUT;
    return AB_ERR_DEVICE_FLAG;
}

const char *ab_status_str(ab_status s)
{
    switch (s) {
    case AB_OK: return "AB_OK";
    case AB_ERR_NULL: return "AB_ERR_NULL";
    case AB_ERR_SHAPE: return "AB_ERR_SHAPE";
    case AB_ERR_DTYPE: return "AB_ERR_DTYPE";
    case AB_ERR_UNSUPPORTED: return "AB_ERR_UNSUPPORTED";
    case AB_ERR_RANGE: return "AB_ERR_RANGE";
    case AB_ERR_CUDA: return "AB_ERR_CUDA";
    case AB_ERR_DEVICE_FLAG: return "AB_ERR_DEVICE_FLAG";
    case AB_ERR_TIMEOUT: return "AB_ERR_TIMEOUT";
    case AB_ERR_ALIGN: return "AB_ERR_ALIGN";
    case AB_ERR_WORKSPACE: return "AB_ERR_WORKSPACE";
    }
    return "AB_ERR_UNKNOWN";
}

const char *ab_last_cuda_error(void) { return cudaGetErrorString(ab::g_last_cuda_error); }

int ab_version(void) { return 100; }

}  // extern "C"
