// ab_host.cu -- ab_forward_host: the whole hot path (IBCS block scores, SIP or top-k
// selection, block-sparse attention) for Q, K, V in host memory, with O returned to host
// memory. The (b, h) head pairs go through in chunks, and the copies of one chunk overlap
// the computation of its neighbours:
//
//   copy-in stream   H2D(0) H2D(1)         H2D(2)          ...
//   caller's stream         compute(0)     compute(1)      compute(2) ...
//   copy-out stream                        D2H(0)          D2H(1)     ...
//
// Two device slots per tensor (Q, K, V in; O out) carry the chunks; events order a slot's
// reuse after the work that last read it. Every stage works per (b, h), and SIP keys its
// random numbers by the global (b, h), so the result is the one the device calls give on
// the whole tensors.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/ab_attn.h"
#include "ab_kernels.h"

namespace {

constexpr int kMaxDevices = 64;

// Streams and events of the copy pipeline, created on a device's first use and kept
// until process exit. The mutex makes one call's enqueue sequence atomic, so concurrent
// calls from several host threads never interleave their records and waits on the
// shared events (their copies then queue on the same copy streams).
struct HostPipe {
    std::mutex mu;
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr;
    cudaEvent_t copied_in[2] = {}, computed[2] = {}, copied_out[2] = {};
};

HostPipe g_pipes[kMaxDevices];

cudaError_t pipe_init(HostPipe &hp)
{
    if (hp.ready) return cudaSuccess;
    cudaError_t e = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming);
    for (int s = 0; s < 2 && e == cudaSuccess; ++s) {
        e = cudaEventCreateWithFlags(&hp.copied_in[s], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.computed[s], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.copied_out[s], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) hp.ready = true;
    return e;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Device workspace of one call: two slots of Q, K, V and O for `ch` head pairs, then the
// scoring workspace, scores and the plan of one chunk.
struct HostLayout {
    size_t q[2], k[2], v[2], o[2], score_ws, score_ws_bytes, scores, idx, cnt, w, total;
};

HostLayout host_layout(const ab_shape &s, int C, int ch, size_t out_elem)
{
    HostLayout L{};
    const size_t tok = (size_t)ch * s.N_pad * s.d;  // elements of one tensor chunk
    const size_t nqb = (size_t)s.N_pad / AB_BLOCK, nkb = nqb;
    size_t off = 0;
    for (int b = 0; b < 2; ++b) {
        L.q[b] = off;
        off = up256(off + tok * 2);
        L.k[b] = off;
        off = up256(off + tok * 2);
        L.v[b] = off;
        off = up256(off + tok * 2);
        L.o[b] = off;
        off = up256(off + tok * out_elem);
    }
    L.score_ws = off;
    L.score_ws_bytes = ab::score_layout((size_t)ch, nqb, nkb, (size_t)s.d, (size_t)C).total;
    off = up256(off + L.score_ws_bytes);
    L.scores = off;
    off = up256(off + (size_t)ch * nqb * nkb * 4);
    L.idx = off;
    off = up256(off + (size_t)ch * nqb * nkb * 4);
    L.cnt = off;
    off = up256(off + (size_t)ch * nqb * 4);
    L.w = off;
    off = up256(off + (size_t)ch * nqb * nkb * 4);
    L.total = off;
    return L;
}

ab_status host_args(const ab_shape &s, int n_clusters, int chunk_heads, ab_dtype out_dtype)
{
    if (s.B <= 0 || s.H <= 0 || s.N <= 0 || s.N_pad <= 0 || s.d <= 0) return AB_ERR_SHAPE;
    if (s.N_pad % AB_BLOCK != 0 || s.N > s.N_pad || s.N_pad - s.N >= AB_BLOCK) return AB_ERR_SHAPE;
    if (s.dtype != AB_BF16 || (out_dtype != AB_BF16 && out_dtype != AB_F32)) return AB_ERR_DTYPE;
    if (s.d != 64 && s.d != 128) return AB_ERR_UNSUPPORTED;
    if (n_clusters < 1 || n_clusters > 8) return AB_ERR_UNSUPPORTED;
    if (s.N_pad / AB_BLOCK > AB_MAX_BLOCKS || (long long)s.B * s.H > 65535LL) return AB_ERR_RANGE;
    if (chunk_heads < 1 || chunk_heads > s.B * s.H) return AB_ERR_RANGE;
    return AB_OK;
}

}  // namespace

extern "C" {

ab_status ab_forward_host_workspace_size(ab_shape s, int n_clusters, int chunk_heads,
                                         ab_dtype out_dtype, size_t *bytes)
{
    if (!bytes) return AB_ERR_NULL;
    *bytes = 0;
    const ab_status st = host_args(s, n_clusters, chunk_heads, out_dtype);
    if (st != AB_OK) return st;
    *bytes = host_layout(s, n_clusters, chunk_heads, out_dtype == AB_F32 ? 4 : 2).total;
    return AB_OK;
}

ab_status ab_forward_host(const void *q_host, const void *k_host, const void *v_host, ab_shape s,
                          int n_clusters, int iters, ab_mode mode, int budget, uint64_t seed,
                          void *o_host, ab_dtype out_dtype, int chunk_heads, void *workspace,
                          size_t workspace_bytes, int *dev_flag, void *stream)
{
    nvtxRangePushA("ab_forward_host");
    struct Pop {
        ~Pop() { nvtxRangePop(); }
    } pop;
    if (!q_host || !k_host || !v_host || !o_host) return AB_ERR_NULL;
    ab_status st = host_args(s, n_clusters, chunk_heads, out_dtype);
    if (st != AB_OK) return st;
    if (iters < 1 || iters > 1000 || budget < 1) return AB_ERR_RANGE;
    if (mode != AB_MODE_SIP && mode != AB_MODE_TOPK) return AB_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return AB_ERR_ALIGN;
    const size_t out_elem = out_dtype == AB_F32 ? 4 : 2;
    const HostLayout L = host_layout(s, n_clusters, chunk_heads, out_elem);
    if (!workspace || workspace_bytes < L.total) return AB_ERR_WORKSPACE;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return ab::status_of(e);
    if (dev < 0 || dev >= kMaxDevices) return AB_ERR_UNSUPPORTED;
    HostPipe &hp = g_pipes[dev];
    std::lock_guard<std::mutex> lock(hp.mu);
    e = pipe_init(hp);
    if (e != cudaSuccess) return ab::status_of(e);

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    cudaStream_t cs = (cudaStream_t)stream;
    const int BH = s.B * s.H, nqb = s.N_pad / AB_BLOCK, nkb = nqb;
    const size_t row_elems = (size_t)s.N_pad * s.d;  // elements of one head pair
    float *scores = reinterpret_cast<float *>(ws + L.scores);
    int32_t *idx = reinterpret_cast<int32_t *>(ws + L.idx);
    int32_t *cnt = reinterpret_cast<int32_t *>(ws + L.cnt);
    float *w = reinterpret_cast<float *>(ws + L.w);
    const int K = budget < nkb ? budget : nkb;
    // the copies start after the work already on the caller's stream (it may still read
    // the workspace)
    e = cudaEventRecord(hp.start, cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.in, hp.start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.out, hp.start, 0);
    const int n_chunks = (BH + chunk_heads - 1) / chunk_heads;
    for (int c = 0; c < n_chunks && e == cudaSuccess && st == AB_OK; ++c) {
        const int slot = c & 1;
        const int bh0 = c * chunk_heads;
        const int nh = BH - bh0 < chunk_heads ? BH - bh0 : chunk_heads;
        const size_t in_bytes = (size_t)nh * row_elems * 2, out_bytes = (size_t)nh * row_elems * out_elem;
        void *qd = ws + L.q[slot], *kd = ws + L.k[slot], *vd = ws + L.v[slot], *od = ws + L.o[slot];
        // copy in: the slot's tensors were last read by the computation of chunk c - 2
        if (c >= 2) e = cudaStreamWaitEvent(hp.in, hp.computed[slot], 0);
        const size_t in_off = (size_t)bh0 * row_elems * 2;
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(qd, static_cast<const uint8_t *>(q_host) + in_off, in_bytes,
                                cudaMemcpyHostToDevice, hp.in);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(kd, static_cast<const uint8_t *>(k_host) + in_off, in_bytes,
                                cudaMemcpyHostToDevice, hp.in);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(vd, static_cast<const uint8_t *>(v_host) + in_off, in_bytes,
                                cudaMemcpyHostToDevice, hp.in);
        if (e == cudaSuccess) e = cudaEventRecord(hp.copied_in[slot], hp.in);
        // compute on the caller's stream: the slot's O was last read by the copy-out of
        // chunk c - 2
        if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, hp.copied_in[slot], 0);
        if (e == cudaSuccess && c >= 2) e = cudaStreamWaitEvent(cs, hp.copied_out[slot], 0);
        if (e != cudaSuccess) break;
        ab_shape cshape = s;
        cshape.B = 1;
        cshape.H = nh;
        st = ab_score(qd, kd, cshape, n_clusters, iters, scores, nullptr, nullptr, nullptr, nullptr,
                      ws + L.score_ws, L.score_ws_bytes, dev_flag, stream);
        if (st != AB_OK) break;
        if (mode == AB_MODE_SIP)
            e = ab::launch_sip(scores, nh, s.H, bh0, nqb, nkb, K, seed, idx, cnt, w, nullptr, dev_flag, cs);
        else
            e = ab::launch_topk(scores, 1, nh, nqb, nkb, K, idx, cnt, w, dev_flag, cs);
        if (e != cudaSuccess) break;
        st = mode == AB_MODE_SIP
                 ? ab_attn_fwd(qd, kd, vd, cshape, idx, cnt, w, od, out_dtype, nullptr, dev_flag, stream)
                 : ab_attn_topk_fwd(qd, kd, vd, cshape, idx, cnt, od, out_dtype, nullptr, dev_flag, stream);
        if (st != AB_OK) break;
        e = cudaEventRecord(hp.computed[slot], cs);
        // copy out
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.out, hp.computed[slot], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(static_cast<uint8_t *>(o_host) + (size_t)bh0 * row_elems * out_elem, od,
                                out_bytes, cudaMemcpyDeviceToHost, hp.out);
        if (e == cudaSuccess) e = cudaEventRecord(hp.copied_out[slot], hp.out);
    }
    // the caller's stream completes after everything enqueued on the copy streams (the
    // last copies out; on an early error, whatever was already queued)
    cudaError_t j = cudaEventRecord(hp.copied_in[0], hp.in);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(cs, hp.copied_in[0], 0);
    if (j == cudaSuccess) j = cudaEventRecord(hp.copied_out[0], hp.out);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(cs, hp.copied_out[0], 0);
    if (st != AB_OK) return st;
    return ab::status_of(e != cudaSuccess ? e : j);
}

}  // extern "C"
