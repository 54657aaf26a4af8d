/*
 * ab_attn.h -- C ABI of the AB-Attention hot path on NVIDIA B200 (sm_100a).
 *
 * The method is described on the news page "AB-Attention ускорил генерацию видео до
 * 2,23× и пропускает 92% внимания" (app.hamidun.com), section «Три приёма AB-Attention»:
 * score key blocks (IBCS), sample them (SIP), and run softmax attention over the
 * sampled blocks, gathered by index, with a logit shift. The page's section «Где
 * ломаются прежние разреженные схемы» describes the top-k baseline.
 *
 * Conventions shared by every call
 *   - Token tensors Q, K, V, O are contiguous bf16 arrays [B, H, N_pad, d] (BHND,
 *     row-major). N is the number of valid tokens, N_pad = N rounded up to a multiple
 *     of 128 (the block size). Rows t >= N are never read as data (the kernels treat
 *     them as absent) and are written as 0 on output.
 *   - n_qb = n_kb = N_pad / 128 query / key blocks of 128 tokens each.
 *   - Every pointer argument except `stream` (and the host buffers of ab_forward_host)
 *     is a DEVICE pointer on the current device, allocated and owned by the caller,
 *     16-byte aligned. The calls allocate no device memory; the host-side work is
 *     argument validation, building TMA tensor maps and enqueueing kernels (and, for
 *     the attention calls, one 16-byte memset; for ab_attn_bwd, one memset of part of
 *     its workspace; for ab_forward_host, the copies).
 *   - Library-owned device state: two file-scope __device__ arrays exist once on every
 *     GPU that loads the library, from load until process exit: the attention
 *     kernels' 4096 claim slots (16 bytes each; see "Scheduling" at ab_attn_fwd) and
 *     the AB_NOALLOC_SCRATCH_BYTES scratch of ab_score_noalloc; and on the host, the
 *     copy streams and events of ab_forward_host and one side stream and two events
 *     per device for ab_score (created on first use). Nothing else persists between
 *     calls.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call only
 *     enqueues work on it and returns; results are ready when the stream is.
 *   - Argument errors are reported synchronously by the return value and nothing is
 *     enqueued. Problems only the device can see (a bad score, an out-of-range block
 *     index, a bounded wait that gave up) are OR-ed as AB_FLAG_* bits into the
 *     optional `dev_flag` int (caller-allocated, caller-zeroed); read it back with
 *     ab_check_flag().
 */
#ifndef AB_ATTN_H
#define AB_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    AB_OK = 0,
    AB_ERR_NULL = 1,        /* a required pointer is NULL */
    AB_ERR_SHAPE = 2,       /* inconsistent or non-positive sizes */
    AB_ERR_DTYPE = 3,       /* token tensors must be AB_BF16 */
    AB_ERR_UNSUPPORTED = 4, /* head dim other than 64 / 128, clusters outside 1..8, ... */
    AB_ERR_RANGE = 5,       /* budget < 1, iters < 1, too many blocks */
    AB_ERR_CUDA = 6,        /* a CUDA runtime / driver call or launch failed */
    AB_ERR_DEVICE_FLAG = 7, /* ab_check_flag: the device flag is non-zero */
    AB_ERR_TIMEOUT = 8,     /* ab_check_flag: a kernel's bounded wait gave up */
    AB_ERR_ALIGN = 9,       /* a pointer is not 16-byte aligned */
    AB_ERR_WORKSPACE = 10   /* workspace NULL or smaller than ab_score_workspace_size */
} ab_status;

typedef enum { AB_F32 = 0, AB_BF16 = 1 } ab_dtype;

typedef enum {
    AB_MODE_SIP = 0, /* sampling with inclusion-probability weights */
    AB_MODE_TOPK = 1 /* deterministic top-k, all weights 1 */
} ab_mode;

/* Shape of the token tensors (BHND, contiguous). dtype must be AB_BF16. */
typedef struct {
    int32_t B, H, N, N_pad, d;
    int32_t dtype; /* ab_dtype */
} ab_shape;

/* Bits OR-ed into *dev_flag by the kernels. */
#define AB_FLAG_BAD_SCORE 1u  /* ab_select: a score is NaN, infinite, < 0 or > 2, or a
                                 SIP row's exact fixed-point sum needs more than 64 bits */
#define AB_FLAG_BAD_INDEX 2u  /* ab_attn_*: a cnt or idx entry outside its range */
#define AB_FLAG_BAD_WEIGHT 4u /* ab_attn_fwd: a weight is NaN, infinite or <= 0 */
#define AB_FLAG_TIMEOUT 8u    /* a bounded in-kernel wait gave up (pipeline stalled) */
#define AB_FLAG_SCHED_COLLISION 16u /* ab_attn_*: another attention call used the same
                                       claim slot while this one ran (see "Scheduling" at
                                       ab_attn_fwd); this call's output is unreliable */

/* Limits: head dim d in {64, 128}; 1 <= n_kb <= 8192 (N_pad <= 1,048,576). */
#define AB_BLOCK 128
#define AB_MAX_BLOCKS 8192
/* The page's fine-grained key/value selection unit (section «Три приёма AB-Attention»,
 * third technique): 4 tokens. With it at most AB_MAX_UNITS units per head
 * (N_pad <= 262144); ab_select takes rows of up to AB_MAX_UNITS entries. */
#define AB_UNIT4 4
#define AB_MAX_UNITS 65536

/*
 * ab_score_workspace_size -- bytes of device scratch ab_score() needs for shape `s`
 * and `n_clusters`: the mean keys [B,H,n_kb,d] fp32, the centroids [B,H,n_qb,C,d] fp32,
 * the cluster weights [B,H,n_qb,C] fp32, the two fp16 terms of each mean key scaled by a
 * power of two [2,B,H,n_kb,d] (operands of the tensor-core block score) and each mean
 * key's unscale factor fp32 [B,H,n_kb rounded up to 256], each region 256-byte aligned.
 * Returns AB_ERR_* for an invalid shape; *bytes is then 0.
 */
ab_status ab_score_workspace_size(ab_shape s, int n_clusters, size_t *bytes);

/*
 * ab_score -- IBCS block scores (page section «Три приёма AB-Attention», first
 * technique). For every query block qb of 128 tokens:
 *   1. kbar_j = mean of the valid keys of key block j;
 *   2. k-means of the block's valid queries into C = n_clusters clusters, `iters`
 *      Lloyd iterations (assign to the nearest centroid in squared Euclidean
 *      distance, ties to the lowest cluster; update to the member mean, an empty
 *      cluster keeps its centroid); the initial centroid c is the query at
 *      block-local index c*floor(n_v/C) (min(c, n_v-1) when n_v < C); the weight of a
 *      cluster is its share of the block's valid queries;
 *   3. scores[qb][j] = sum_c w_c softmax_j(cent_c . kbar_j / sqrt(d)), the softmax
 *      taken over all n_kb key blocks.
 * q, k       : bf16 [B,H,N_pad,d], s.dtype == AB_BF16, d in {64,128}.
 * n_clusters : 1..8 (8 is the method's value; 1 gives mean-pooled block scores).
 * iters      : >= 1 Lloyd iterations (5 in the method's configuration).
 * scores     : out, fp32 [B,H,n_qb,n_kb]; each row sums to 1.
 * kbar, centroids, cweights, assign : optional outputs (NULL to skip): fp32
 *              [B,H,n_kb,d], fp32 [B,H,n_qb,C,d], fp32 [B,H,n_qb,C], uint8 [B,H,N_pad]
 *              (cluster of each query after the last assignment, 255 on padding rows).
 * workspace  : device scratch of at least ab_score_workspace_size() bytes, owned by
 *              the caller, contents need not be initialised, not read after return.
 * dev_flag   : optional (see above).
 * Errors: AB_ERR_NULL, AB_ERR_SHAPE, AB_ERR_DTYPE, AB_ERR_UNSUPPORTED, AB_ERR_RANGE,
 * AB_ERR_ALIGN, AB_ERR_WORKSPACE, AB_ERR_CUDA.
 */
ab_status ab_score(const void *q, const void *k, ab_shape s, int n_clusters, int iters,
                   float *scores, float *kbar, float *centroids, float *cweights,
                   uint8_t *assign, void *workspace, size_t workspace_bytes, int *dev_flag,
                   void *stream);

/*
 * ab_score_noalloc -- ab_score for callers that cannot allocate device memory. The
 * method's pages have no counterpart to this call; it exists for integration only.
 * Some callers cannot call cudaMalloc or hand the library a workspace: a plugin or
 * custom operator running inside a host framework that owns all device memory and
 * forbids allocation on its execution path, or code that has no allocator of its own.
 * This call computes exactly what ab_score computes (scores only; no optional
 * outputs), with its scratch (the regions of ab_score_workspace_size) in a fixed array
 * of AB_NOALLOC_SCRATCH_BYTES bytes in the library's own device memory. That array
 * exists once on every GPU that loads the library and stays allocated until the
 * process exits. The call itself allocates nothing.
 *   - Scratch needed = ab_score_workspace_size(s, n_clusters); larger problems are
 *     rejected with AB_ERR_WORKSPACE (e.g. 12 heads x 32768 tokens, d = 128, C = 8
 *     needs 16.6 MB and fits; 24 heads x 118912 tokens does not).
 *   - The first call on each device looks up the array's device address (with that
 *     device current) and caches it; make that first call before any stream capture.
 *   - Every call uses the same array and leaves its contents behind; every region is
 *     rewritten before it is read, so no clearing is needed. Calls that overlap on the
 *     GPU (different streams, or different host threads) race on the array: serialise
 *     them, e.g. on one stream.
 * Other arguments, conventions and errors as ab_score.
 */
#define AB_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
ab_status ab_score_noalloc(const void *q, const void *k, ab_shape s, int n_clusters, int iters,
                           float *scores, int *dev_flag, void *stream);

/*
 * ab_score_units, ab_score_units_workspace_size -- IBCS scores at key-unit granularity
 * (page section «Три приёма AB-Attention», third technique: key/value selection units
 * of 4 tokens instead of 128, at the same tile budget). Queries stay in 128-token
 * blocks with their k-means clusters; keys are grouped into units of key_unit tokens
 * (AB_BLOCK or AB_UNIT4): kbar_u = mean of the valid keys of unit u, and
 * scores[qb][u] = sum_c w_c softmax_u(cent_c . kbar_u / sqrt(d)) over the units that
 * hold at least one valid token (u < ceil(N / key_unit)); the other units score 0.
 * With key_unit = AB_BLOCK this is ab_score.
 * scores : out, fp32 [B,H,n_qb,n_ku], n_ku = N_pad / key_unit (<= AB_MAX_UNITS).
 * kbar   : optional out, fp32 [B,H,n_ku,d]. Other arguments as ab_score; the workspace
 *          needs ab_score_units_workspace_size() bytes.
 * Errors: as ab_score; AB_ERR_UNSUPPORTED for another key_unit, AB_ERR_RANGE when
 * n_ku > AB_MAX_UNITS.
 */
ab_status ab_score_units_workspace_size(ab_shape s, int n_clusters, int key_unit, size_t *bytes);
ab_status ab_score_units(const void *q, const void *k, ab_shape s, int n_clusters, int iters,
                         int key_unit, float *scores, float *kbar, float *centroids,
                         float *cweights, uint8_t *assign, void *workspace,
                         size_t workspace_bytes, int *dev_flag, void *stream);

/*
 * ab_selftest_bounded_wait -- exercises the failure path every pipeline of the library
 * relies on, without a GPU fault. The method's pages have no counterpart; it exists so
 * that a test can make an in-kernel wait run out. One CTA initialises an mbarrier that
 * expects one arrival and waits on it with the library's bounded wait (limit limit_us
 * microseconds, 1..1e6). With complete = 0 nothing arrives: the wait gives up after the
 * limit, ORs AB_FLAG_TIMEOUT into *dev_flag and the kernel returns normally (*dev_done
 * = 2), leaving the context usable. With complete != 0 the CTA arrives first and the
 * wait succeeds (*dev_done = 1, no flag). dev_flag, dev_done: device ints owned by the
 * caller. Asynchronous on `stream`; read the result with ab_check_flag.
 * Errors: AB_ERR_NULL, AB_ERR_RANGE, AB_ERR_CUDA (launch).
 */
ab_status ab_selftest_bounded_wait(int limit_us, int complete, int *dev_flag, int *dev_done,
                                   void *stream);

/*
 * ab_selftest_attn_wait_limit -- test entry point with no counterpart on the method's
 * pages: ab_attn_units_fwd (w != NULL) or ab_attn_units_topk_fwd (w == NULL) with every
 * bounded wait inside the attention kernel limited to limit_ns nanoseconds (1..1e9)
 * instead of 2 s, so that a test can make the kernel's own waits give up. A wait that
 * gives up ORs AB_FLAG_TIMEOUT into *dev_flag (required here) and every role of the CTA
 * unwinds: the producer and MMA warps let their copies and MMAs in flight land, the
 * softmax warps run out their loops without waiting, and the CTA frees its tensor
 * memory and returns, leaving the context usable. The output of such a call is
 * undefined. Arguments and errors otherwise as ab_attn_units_fwd.
 */
ab_status ab_selftest_attn_wait_limit(const void *q, const void *k, const void *v, ab_shape s,
                                      int key_unit, const int32_t *idx, const int32_t *cnt,
                                      const float *w, void *out, ab_dtype out_dtype, float *lse,
                                      int *dev_flag, int limit_ns, void *stream);

/*
 * ab_selftest_force_counter_slot -- test hook with no counterpart on the method's pages:
 * the next attention call (from any thread) takes claim slot `slot` instead of the next
 * one in turn, so a test can make two concurrently running calls share a slot and
 * check that the sharing is detected (AB_FLAG_SCHED_COLLISION). Errors: AB_ERR_RANGE
 * unless 0 <= slot < 4096.
 */
ab_status ab_selftest_force_counter_slot(int slot);

/*
 * ab_select -- choose key blocks per query block (page section «Три приёма
 * AB-Attention», second technique SIP; section «Где ломаются прежние разреженные
 * схемы» for top-k).
 * AB_MODE_SIP: inclusion probabilities p_j = min(1, c s_j) with sum p_j = K =
 *   min(budget, n_kb), solved exactly in integers on u_j = floor(s_j 2^50): the
 *   saturated set S grows from empty by S <- S + {j : (K-|S|) u_j >= U - sum_S u} until
 *   stable (if at most K blocks have u_j > 0, exactly those are kept with p = 1);
 *   p_j = 1 on S, else (double)((K-|S|) u_j) / (double)(U - sum_S u). Block j is kept
 *   iff (double)R < p_j 2^53, where R = ((x0 << 32) | x1) >> 11 and (x0, x1) are the
 *   first two words of Philox4x32-10 with key (seed & 0xffffffff, seed >> 32) and
 *   counter (j, qb, h, b). Kept blocks carry w = (float)(1 / p_j), so a block drawn
 *   with p = 1/4 counts four times.
 * AB_MODE_TOPK: the K blocks with the largest scores (ties to the lower index),
 *   weights 1.
 * scores : fp32 [B,H,nqb,nkb], every entry finite and in [0, 2]; for SIP the row's
 *          U = sum_j u_j must fit in 64 bits (a row sum below 2^14; IBCS rows sum to 1).
 * idx    : out, int32 [B,H,nqb,nkb]: kept block indices in ascending order in the
 *          first cnt entries of each row, -1 after them.
 * cnt    : out, int32 [B,H,nqb].
 * w      : out, fp32 [B,H,nqb,nkb] aligned with idx (0 after cnt); required for SIP,
 *          optional (NULL) for top-k.
 * p      : optional out, fp64 [B,H,nqb,nkb]: p_j by block index (SIP only).
 * A row with an invalid score sets AB_FLAG_BAD_SCORE and gets cnt = 0, idx = -1.
 * Errors: AB_ERR_NULL, AB_ERR_SHAPE, AB_ERR_RANGE (budget < 1, nkb > AB_MAX_UNITS),
 * AB_ERR_ALIGN, AB_ERR_CUDA.
 */
ab_status ab_select(const float *scores, int B, int H, int nqb, int nkb, int budget,
                    ab_mode mode, uint64_t seed, int32_t *idx, int32_t *cnt, float *w,
                    double *p, int *dev_flag, void *stream);

/*
 * ab_attn_fwd -- block-sparse softmax attention over the selected key blocks with
 * Horvitz-Thompson weights (page section «Три приёма AB-Attention», SIP and the third
 * technique: the kernel gathers the chosen blocks by index, tokens stay in order, the
 * weights enter as a logit shift). For query i of block qb, over the kept blocks j and
 * their valid keys t < N:
 *   O_i = sum_j w_j sum_t e^{q_i.k_t/sqrt(d)} v_t / sum_j w_j sum_t e^{q_i.k_t/sqrt(d)}
 * computed as online softmax of q_i.k_t/sqrt(d) + ln w_j.
 * q, k, v : bf16 [B,H,N_pad,d], d in {64,128}.
 * idx, cnt, w : the plan from ab_select (row stride n_kb); every w_j must be > 0.
 * out     : [B,H,N_pad,d] in `out_dtype` (AB_BF16 or AB_F32); rows t >= N and rows of
 *           an empty selection are 0.
 * lse     : optional fp32 [B,H,N_pad]: ln of the denominator (0 on padding rows,
 *           -inf for an empty selection).
 * Device-side: an idx/cnt outside range sets AB_FLAG_BAD_INDEX (the block is clamped
 * into range), a bad weight sets AB_FLAG_BAD_WEIGHT.
 * Scheduling: the kernel hands the (b, h, query block) items to its persistent CTAs
 * from a claim slot. Each call takes the next of the 4096 library-owned slots in turn
 * (process-wide, on the host), zeroes it with a memset on `stream` just before the
 * kernel, and tags it with its own launch number. Calls on one stream never share a
 * slot at the same time, nor do the replays of one CUDA graph executable (CUDA orders
 * them). Two executions share a slot only if (a) more than 4096 attention calls are
 * in flight at once across streams, or (b) two graph executables instantiated from
 * ONE capture of a call run at the same time: a captured call keeps the slot and tag
 * it took at capture. Case (b) repeats the same call on the same buffers and still
 * writes the right output. In case (a) each CTA checks the slot's tag when it starts,
 * at every claim and when it ends; a call that finds another call's tag raises
 * AB_FLAG_SCHED_COLLISION and marks the slot so that the other call raises it too.
 * Treat the output of a call that raised it as unreliable.
 * Errors: AB_ERR_NULL, AB_ERR_SHAPE, AB_ERR_DTYPE (inputs not bf16, or out_dtype not
 * AB_BF16 / AB_F32), AB_ERR_UNSUPPORTED, AB_ERR_ALIGN, AB_ERR_CUDA.
 */
ab_status ab_attn_fwd(const void *q, const void *k, const void *v, ab_shape s,
                      const int32_t *idx, const int32_t *cnt, const float *w, void *out,
                      ab_dtype out_dtype, float *lse, int *dev_flag, void *stream);

/*
 * ab_attn_topk_fwd -- the same attention with every weight 1 (no logit shift): the
 * top-k baseline, where a dropped block leaves both the numerator and the softmax
 * normaliser (page section «Где ломаются прежние разреженные схемы»). Takes the
 * idx / cnt of ab_select(..., AB_MODE_TOPK, ...). Arguments and errors as ab_attn_fwd.
 */
ab_status ab_attn_topk_fwd(const void *q, const void *k, const void *v, ab_shape s,
                           const int32_t *idx, const int32_t *cnt, void *out, ab_dtype out_dtype,
                           float *lse, int *dev_flag, void *stream);

/*
 * ab_attn_bwd_workspace_size -- bytes of device scratch ab_attn_bwd() needs for shape s:
 * two fp32 values per query row, a uint16 table of n_qb x n_kb entries per head and a
 * uint32 count per key block, each region 256-byte aligned. Errors: AB_ERR_NULL and the
 * shape errors of ab_attn_fwd.
 */
ab_status ab_attn_bwd_workspace_size(ab_shape s, size_t *bytes);

/*
 * ab_attn_bwd -- gradient of ab_attn_fwd (w != NULL) or ab_attn_topk_fwd (w == NULL)
 * with respect to Q, K and V, for an upstream gradient dO of the output. The plan and
 * the weights are constants (the selection is a sample, page section «Три приёма
 * AB-Attention»); the gradient is that of the softmax attention with logits
 * q_i.k_t/sqrt(d) + ln w_j over the kept blocks: with P_it the attention probabilities
 * and D_i = dO_i . O_i,
 *   dV_t = sum_i P_it dO_i,  dS_it = P_it (dO_i . v_t - D_i),
 *   dQ_i = sum_t dS_it k_t / sqrt(d),  dK_t = sum_i dS_it q_i / sqrt(d).
 * q, k, v   : bf16 [B,H,N_pad,d] as given to the forward call; d in {64, 128}.
 * idx, cnt, w : the plan given to the forward call (key blocks of 128 tokens); the
 *             blocks of a row must be distinct (as ab_select makes them).
 * out, out_dtype, lse : the forward call's output (AB_BF16 or AB_F32) and its lse.
 * dout      : bf16 [B,H,N_pad,d], the upstream gradient; rows t >= N are ignored.
 * dq, dk, dv: out, fp32 [B,H,N_pad,d]; rows t >= N, the rows of a query block with an
 *             empty selection (dq) and the rows of a key block no query block kept
 *             (dk, dv) are 0.
 * workspace : device scratch of ab_attn_bwd_workspace_size() bytes, owned by the
 *             caller, contents need not be initialised; the call clears its table and
 *             counts with one memset on `stream`.
 * Every sum runs in a fixed order: the result is the same on every run.
 * Device-side: an idx/cnt outside range or a block twice in one row sets
 * AB_FLAG_BAD_INDEX, a bad weight AB_FLAG_BAD_WEIGHT, a bounded wait that gave up
 * AB_FLAG_TIMEOUT (the output is then undefined).
 * Errors: AB_ERR_NULL, AB_ERR_SHAPE, AB_ERR_DTYPE, AB_ERR_UNSUPPORTED, AB_ERR_RANGE,
 * AB_ERR_ALIGN, AB_ERR_WORKSPACE, AB_ERR_CUDA.
 */
ab_status ab_attn_bwd(const void *q, const void *k, const void *v, ab_shape s, const int32_t *idx,
                      const int32_t *cnt, const float *w, const void *out, ab_dtype out_dtype,
                      const float *lse, const void *dout, float *dq, float *dk, float *dv,
                      void *workspace, size_t workspace_bytes, int *dev_flag, void *stream);

/*
 * ab_selftest_attn_bwd_wait_limit -- test entry point with no counterpart on the method's
 * pages: ab_attn_bwd with every bounded wait inside its two tensor-core kernels limited to
 * limit_ns nanoseconds (1..1e9) instead of 2 s, so that a test can make their own waits
 * give up (below 1 ms the waits poll without blocking and read the clock at every
 * poll). A wait that gives up ORs AB_FLAG_TIMEOUT into *dev_flag (required here); the
 * issuer warp lets its copies and MMAs in flight land, the compute warps leave their
 * loops, and the CTA frees its tensor memory and returns, leaving the context usable.
 * The gradients of such a call are undefined. Arguments and errors otherwise as
 * ab_attn_bwd.
 */
ab_status ab_selftest_attn_bwd_wait_limit(const void *q, const void *k, const void *v, ab_shape s,
                                          const int32_t *idx, const int32_t *cnt, const float *w,
                                          const void *out, ab_dtype out_dtype, const float *lse,
                                          const void *dout, float *dq, float *dk, float *dv,
                                          void *workspace, size_t workspace_bytes, int *dev_flag,
                                          int limit_ns, void *stream);

/*
 * ab_attn_units_fwd, ab_attn_units_topk_fwd -- the attention of ab_attn_fwd /
 * ab_attn_topk_fwd over selected key units of key_unit tokens (AB_BLOCK, or AB_UNIT4:
 * the page's 4-token units, third technique). idx / cnt / w come from ab_select run on
 * ab_score_units' scores (rows of n_ku = N_pad / key_unit entries, kept unit indices
 * ascending). For AB_UNIT4 the kernel gathers the kept units 32 at a time into
 * 128-key tiles (unit s of a tile -> tile rows 4s..4s+3), so a query block costs
 * ceil(cnt / 32) tensor-core tiles; tokens t >= N and empty tile slots take no part.
 * Unit u counts with weight w (HT: logit + ln w), 1 in the top-k call.
 *   O_i = sum_{u in sel} w_u sum_{t in u, t<N} e^{q_i.k_t/sqrt(d)} v_t
 *         / sum_{u in sel} w_u sum_{t in u, t<N} e^{q_i.k_t/sqrt(d)}
 * With key_unit = AB_BLOCK these are ab_attn_fwd / ab_attn_topk_fwd.
 * Errors and device flags: as ab_attn_fwd; AB_ERR_UNSUPPORTED for another key_unit,
 * AB_ERR_RANGE when n_ku > AB_MAX_UNITS.
 */
ab_status ab_attn_units_fwd(const void *q, const void *k, const void *v, ab_shape s, int key_unit,
                            const int32_t *idx, const int32_t *cnt, const float *w, void *out,
                            ab_dtype out_dtype, float *lse, int *dev_flag, void *stream);
ab_status ab_attn_units_topk_fwd(const void *q, const void *k, const void *v, ab_shape s,
                                 int key_unit, const int32_t *idx, const int32_t *cnt, void *out,
                                 ab_dtype out_dtype, float *lse, int *dev_flag, void *stream);

/*
 * ab_forward_host -- the whole path (ab_score, ab_select, then ab_attn_fwd for SIP or
 * ab_attn_topk_fwd for top-k) for Q, K, V in HOST memory, with O written back to host
 * memory: the end-to-end call of an application whose activations live on the host.
 * The B*H (b, h) head pairs go through in chunks of chunk_heads. The copy of chunk c
 * to the device overlaps the computation of chunk c - 1 and the copy back of chunk
 * c - 2's O. Two device slots per tensor are carved from `workspace`, the copies run
 * on two library-owned streams per GPU, and the computation runs on `stream`. The
 * result is bit for bit that of the device calls on the whole tensors with the same
 * seed: every stage works per (b, h), and SIP keys its random numbers by the global
 * (b, h).
 * q_host, k_host, v_host : bf16 [B,H,N_pad,d] in host memory. Page-locked memory
 *          (cudaHostAlloc / cudaHostRegister) lets the copies overlap the computation;
 *          pageable memory gives the same result with the copies serialised.
 * o_host : out, [B,H,N_pad,d] in out_dtype (AB_BF16 or AB_F32), host memory.
 * n_clusters, iters : as ab_score. mode, budget, seed : as ab_select.
 * chunk_heads : head pairs per chunk, 1 .. B*H. Smaller chunks shorten the first
 *          copy-in and the last copy-out that nothing overlaps; a few heads per chunk
 *          keep each attention launch large enough to fill the GPU.
 * workspace : device memory of ab_forward_host_workspace_size() bytes (16-byte
 *          aligned). It holds two slots of Q, K, V and O for chunk_heads head pairs,
 *          plus one chunk's scoring workspace, scores and plan.
 * Returns once everything is enqueued; O is in host memory when `stream` completes.
 * The host buffers and the workspace must stay untouched until then. Library-owned
 * state: two copy streams and seven events per GPU, created on the first call on that
 * GPU and kept until process exit. Concurrent calls from several host threads are
 * safe; their copies queue on the same copy streams.
 * Errors: AB_ERR_NULL, AB_ERR_SHAPE, AB_ERR_DTYPE, AB_ERR_UNSUPPORTED, AB_ERR_RANGE
 * (iters, budget, chunk_heads), AB_ERR_ALIGN, AB_ERR_WORKSPACE, AB_ERR_CUDA; device-side
 * problems as the three calls, in dev_flag.
 */
ab_status ab_forward_host_workspace_size(ab_shape s, int n_clusters, int chunk_heads,
                                         ab_dtype out_dtype, size_t *bytes);
ab_status ab_forward_host(const void *q_host, const void *k_host, const void *v_host, ab_shape s,
                          int n_clusters, int iters, ab_mode mode, int budget, uint64_t seed,
                          void *o_host, ab_dtype out_dtype, int chunk_heads, void *workspace,
                          size_t workspace_bytes, int *dev_flag, void *stream);

/*
 * ab_check_flag -- synchronise `stream`, copy *dev_flag to *host_flag and map it to a
 * status: AB_OK (0), AB_ERR_TIMEOUT (AB_FLAG_TIMEOUT set) or AB_ERR_DEVICE_FLAG.
 */
ab_status ab_check_flag(const int *dev_flag, int *host_flag, void *stream);

/* Human-readable name of a status code (static storage). */
const char *ab_status_str(ab_status s);

/* The CUDA error string behind the calling thread's most recent AB_ERR_CUDA (static
 * storage; "no error" if the thread has seen none). */
const char *ab_last_cuda_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int ab_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AB_ATTN_H */
