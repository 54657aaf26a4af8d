// attn_bwd_kernel.cu -- gradient of the block-sparse HT attention with respect to Q, K
// and V on sm_100a (tcgen05 + TMEM + TMA).
//
// The forward (news page "AB-Attention ускорил генерацию видео до 2,23× и пропускает 92%
// внимания", section «Три приёма AB-Attention») is softmax attention over the kept key
// blocks with the logit of block j shifted by ln w_j. Its gradient, for an upstream
// gradient dO and the forward's O and ln-denominator lse, per query row i and kept key t:
//   P_it = 2^(s_it log2e / sqrt(d) + log2 w_j - lse_i log2e),  D_i = dO_i . O_i
//   dV_t += P_it dO_i,  dS_it = P_it (dO_i . v_t - D_i),
//   dQ_i += dS_it k_t / sqrt(d),  dK_t += dS_it q_i / sqrt(d).
// The selection and the weights are constants of the step.
//
// Four launches on the caller's stream:
//   1. row statistics: D_i and lse_i log2e per query row (+inf on rows that take no part:
//      padding rows and rows of an empty selection, so that their P is 0);
//   2. the plan transposed into a mark table [bh][key block][query block] holding c + 1
//      for the plan entry c that keeps the pair, and a count per key block (zeroed just
//      before; a second mark of the same pair is a duplicate block in a row and raises
//      AB_FLAG_BAD_INDEX);
//   3. dQ: one CTA per (b, h, query block), over its kept key blocks in plan order:
//      S = Q K_j^T and dP = dO V_j^T into TMEM (SS MMAs, both operands K-major), dS packed
//      to bf16 over dP, dQ += dS K_j (TS MMA: dS from TMEM, K_j as an MN-major operand);
//   4. dK, dV: one CTA per (b, h, key block), over the query blocks that kept it in
//      ascending order (read from the mark table): S^T = K Q^T and dP^T = V dO^T, then
//      dV += P^T dO and dK += dS^T Q (TS MMAs, dO and Q as MN-major operands).
// Every sum runs in a fixed order, so the result does not depend on scheduling. The two
// gradient kernels share one structure: warps 0-7 do the elementwise work, warp w on
// TMEM lanes 32 (w mod 4) .. +31 (its rows) and half w / 4 of the columns; warp 8 issues
// every TMA copy and MMA. The two hand over through mbarriers (S read, dS stored), so the
// tensor core runs the next pair's products while the warps work on the current one.
// Tiles arrive by TMA in 64-column boxes with the 128-byte swizzle, as in the forward
// kernel. Every wait is bounded; a wait that gives up raises AB_FLAG_TIMEOUT, and the
// CTA lets its copies and MMAs land and frees its tensor memory before it returns. The C
// entry points ab_attn_bwd, ab_attn_bwd_workspace_size and the wait-limit test entry
// ab_selftest_attn_bwd_wait_limit are at the end of this file.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include <nvtx3/nvToolsExt.h>

#include "ab_device.cuh"
#include "ab_kernels.h"
#include "tmap_host.h"

namespace ab {

namespace {

// Workspace regions, each 256-byte aligned: per query row D_i = dO_i . O_i and
// lse_i log2e (fp32 [BH][N_pad] each), the plan's mark table uint16 [BH][n_kb][n_qb] and
// the number of query blocks keeping each key block, uint32 [BH][n_kb].
struct AttnBwdLayout {
    size_t rowD, rowL2, mark, kcount, total;
};

AttnBwdLayout attn_bwd_layout(size_t BH, size_t N_pad)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t nb = N_pad / 128;
    AttnBwdLayout L;
    L.rowD = 0;
    L.rowL2 = up(BH * N_pad * sizeof(float));
    L.mark = up(L.rowL2 + BH * N_pad * sizeof(float));
    L.kcount = up(L.mark + BH * nb * nb * sizeof(uint16_t));
    L.total = up(L.kcount + BH * nb * sizeof(uint32_t));
    return L;
}

struct AttnBwdLaunch {
    const void *q, *k, *v;
    const void *out;   // the forward's output O
    bool out_f32;      // O is fp32 (else bf16)
    const void *dout;  // upstream gradient dO, bf16
    const float *lse;  // the forward's ln-denominator
    const int32_t *idx, *cnt;
    const float *w;  // nullptr = unweighted (top-k)
    float *dq, *dk, *dv;
    void *workspace;  // attn_bwd_layout(...).total bytes
    int *flag;
    int B, H, N, N_pad, d;
    unsigned long long wait_ns;  // > 0: limit of the kernels' bounded waits (tests); 0: 2 s
};

constexpr int kBwdThreads = 288;  // 8 compute warps + 1 issuer warp
constexpr int kBwdTmemCols = 512;
constexpr int kTileMax = 128 * 128 * 2;  // one 128 x 128 bf16 tile
// dynamic shared memory (+ 1024 bytes of alignment slack), one CTA per SM:
// dQ: Q, dO and rings of 3 (K) and 2 (V) tiles; dK/dV: K, V and two rings of 2 (Q, dO)
constexpr int kDqSmem = 7 * kTileMax + 1024;
constexpr int kDkdvSmem = 6 * kTileMax + 1024;

struct BwdParams {
    const int32_t *idx, *cnt;
    const float *w;  // nullptr: every weight 1 (top-k)
    const float *rowD, *rowL2;
    const uint16_t *mark;
    const uint32_t *kcount;
    float *dq, *dk, *dv;
    int *flag;
    int N, N_pad, nqb, nkb;
    float scale, scale_log2;
    uint64_t wait_ns;  // limit of every bounded wait
};

// S (+)= A B^T over the head dimension: A, B are [128 rows][D] tiles, K-major, two
// 64-column swizzled boxes 16 KB apart for D = 128.
template <int D>
__device__ __forceinline__ void mma_rows(uint32_t d_tmem, uint64_t a0, uint64_t b0)
{
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
        mma_ss(d_tmem, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u);
    }
}

// Acc[128 x D] (+)= A B: A is a 128 x 128 bf16 matrix in TMEM, packed two per column,
// its columns 0-63 in TMEM columns 0-31 and 64-127 in columns 64-95 (each softmax half
// packs into the first half of its own columns); B is a [128 k-rows][D] tile used
// MN-major (16 k-rows = 2048 bytes per step).
template <int D>
__device__ __forceinline__ void mma_packed(uint32_t acc_tmem, uint32_t a_tmem, uint64_t b0,
                                           bool accumulate)
{
    constexpr uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        mma_ts(acc_tmem, a_tmem + kk * 8 + (kk >= 4 ? 32 : 0), b0 + (uint64_t)(kk * (2048 >> 4)),
               idesc, (kk > 0 || accumulate) ? 1u : 0u);
}

template <int D>
__device__ __forceinline__ void tma_tile(uint8_t *dst, const CUtensorMap *tm, uint64_t *bar,
                                         int row_block, int bh)
{
#pragma unroll
    for (int x = 0; x < D / 64; ++x) tma_load_3d(dst + x * 16384, tm, bar, x * 64, row_block * 128, bh);
}

__device__ __forceinline__ float lw2_val(float wj, int *flag, bool report)
{
    if (wj > 0.f && wj < INFINITY) return fast_log2(wj);
    if (report) raise_flag(flag, AB_FLAG_BAD_WEIGHT);
    return 0.f;
}

// 2^x for a pair: on the MUFU unit, or (soft) on the FMA pipe by the forward kernel's
// polynomial (max relative error 7.5e-5); the P step gives every fifth pair to the FMA
// pipe so that the two units share the exponentials.
__device__ __forceinline__ float2 exp2_pair(uint64_t x2, bool soft)
{
    if (soft) return soft_exp2_pair(x2);
    const float2 x = f2_unpack(x2);
    return make_float2(fast_exp2(x.x), fast_exp2(x.y));
}

// Rows [row0, row0 + 128) of a [.., D] fp32 tensor set to 0 by the whole CTA.
template <int D>
__device__ __forceinline__ void zero_rows(float *base, size_t row0)
{
    float4 *p4 = reinterpret_cast<float4 *>(base + row0 * D);
    for (int e = threadIdx.x; e < 128 * D / 4; e += blockDim.x) p4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// This thread's D / 2 accumulator columns of its row, times `mul`, to row `row` of `dst`
// (0 when the row is past the sequence end).
template <int D>
__device__ __forceinline__ void store_acc_row(uint32_t taddr, float *dst_row, float mul, bool valid)
{
#pragma unroll
    for (int ch = 0; ch < D / 64; ++ch) {
        uint32_t r[32];
        tmem_ld32(taddr + ch * 32, r);
        tmem_wait_ld();
        float4 *o4 = reinterpret_cast<float4 *>(dst_row + ch * 32);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            o4[e] = valid ? make_float4(__uint_as_float(r[4 * e]) * mul, __uint_as_float(r[4 * e + 1]) * mul,
                                        __uint_as_float(r[4 * e + 2]) * mul, __uint_as_float(r[4 * e + 3]) * mul)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ---------------------------------------------------------------------------------
// 1. Row statistics: D_i = dO_i . O_i and lse_i log2e (16 threads per row).
// ---------------------------------------------------------------------------------
template <int D, bool kOF32>
__global__ void __launch_bounds__(256) attn_bwd_rowstats_kernel(const void *o, const __nv_bfloat16 *g,
                                                                const float *lse, float *rowD,
                                                                float *rowL2, size_t rows, int N,
                                                                int N_pad)
{
    constexpr int kPer = D / 16;  // elements per thread
    const size_t r = (size_t)blockIdx.x * 16 + (threadIdx.x >> 4);
    const int sub = threadIdx.x & 15;
    if (r >= rows) return;  // whole 16-lane groups leave together
    float acc = 0.f;
    const __nv_bfloat16 *gr = g + r * D + sub * kPer;
    if constexpr (kOF32) {
        const float *orow = static_cast<const float *>(o) + r * D + sub * kPer;
#pragma unroll
        for (int e = 0; e < kPer; e += 4) {
            const float4 ov = *reinterpret_cast<const float4 *>(orow + e);
            const uint2 gv = *reinterpret_cast<const uint2 *>(gr + e);
            const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gv.x));
            const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gv.y));
            acc = fmaf(ov.x, g01.x, acc);
            acc = fmaf(ov.y, g01.y, acc);
            acc = fmaf(ov.z, g23.x, acc);
            acc = fmaf(ov.w, g23.y, acc);
        }
    } else {
        const __nv_bfloat16 *orow = static_cast<const __nv_bfloat16 *>(o) + r * D + sub * kPer;
#pragma unroll
        for (int e = 0; e < kPer; e += 4) {
            const uint2 ov = *reinterpret_cast<const uint2 *>(orow + e);
            const uint2 gv = *reinterpret_cast<const uint2 *>(gr + e);
            const float2 o01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ov.x));
            const float2 o23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ov.y));
            const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gv.x));
            const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gv.y));
            acc = fmaf(o01.x, g01.x, acc);
            acc = fmaf(o01.y, g01.y, acc);
            acc = fmaf(o23.x, g23.x, acc);
            acc = fmaf(o23.y, g23.y, acc);
        }
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (sub == 0) {
        const float l = lse[r];
        const bool on = (int)(r % (size_t)N_pad) < N && l > -INFINITY && l < INFINITY;
        rowD[r] = on ? acc : 0.f;
        rowL2[r] = on ? l * 1.4426950408889634f : INFINITY;
    }
}

// ---------------------------------------------------------------------------------
// 2. Mark table: mark[bh][j][qb] = c + 1 for plan entry c of row (bh, qb) keeping block
//    j, and kcount[bh][j] = the number of query blocks keeping j (one warp per plan row).
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) attn_bwd_mark_kernel(const int32_t *idx, const int32_t *cnt,
                                                            uint16_t *mark, uint32_t *kcount,
                                                            size_t n_rows, int nqb, int nkb, int *flag)
{
    const size_t r = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= n_rows) return;
    int n = cnt[r];
    if (n < 0 || n > nkb) {
        if (lane == 0) raise_flag(flag, AB_FLAG_BAD_INDEX);
        n = n < 0 ? 0 : nkb;
    }
    const size_t bh = r / (size_t)nqb;
    const int qb = (int)(r % (size_t)nqb);
    for (int c = lane; c < n; c += 32) {
        const int j = idx[r * nkb + c];
        if (j < 0 || j >= nkb) {
            raise_flag(flag, AB_FLAG_BAD_INDEX);
            continue;
        }
        unsigned short *m = reinterpret_cast<unsigned short *>(mark + (bh * nkb + j) * nqb + qb);
        if (atomicCAS(m, (unsigned short)0, (unsigned short)(c + 1)) != 0)
            raise_flag(flag, AB_FLAG_BAD_INDEX);  // block j twice in one row
        else
            atomicAdd(kcount + bh * nkb + j, 1u);
    }
}

// ---------------------------------------------------------------------------------
// Shared pieces of the two gradient kernels: warps 0-7 compute (elementwise work on TMEM
// rows), warp 8 issues every TMA copy and MMA. Barrier slots:
//   0: the CTA's fixed tiles   1-3: ring A (3 slots in the dQ kernel, 2 in the dK/dV
//   kernel)   4-5: ring B (2 slots)   6: S (or S^T) done   7: dP (or dP^T) done
//   8: S read (and P^T stored) (256 arrivals)   9: dS stored, dP read (256 arrivals)
//   10: a pair's accumulating MMAs done (dK/dV kernel)   11: all MMAs done
//   12: drain after a failed wait
// ---------------------------------------------------------------------------------
constexpr int kIssuerWarp = 8;
constexpr int kBars = 13;

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16), counted on bar.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// The kernels' bounded wait. With the normal limit it is mbar_wait; with a limit below
// 1 ms (the wait-limit test entry) it polls with the non-blocking test_wait and reads the
// clock at every poll (try_wait may hold the thread until the phase completes), so that
// even a wait of a few microseconds can run past the limit.
// The polling form is a separate instantiation of the kernels (kPoll), launched only by
// the test entry, so that it adds nothing to the normal kernels' code.
template <bool kPoll>
__device__ __forceinline__ bool bwd_wait(uint64_t *bar, uint32_t parity, volatile int *abort, int *flag,
                                         uint64_t limit_ns)
{
    if constexpr (!kPoll) return mbar_wait(bar, parity, abort, flag, limit_ns);
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (done) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > limit_ns) {
            *abort = 1;
            raise_flag(flag, AB_FLAG_TIMEOUT);
            return false;
        }
    }
}

// The issuer warp's bounded wait (all lanes agree).
template <bool kPoll>
__device__ __forceinline__ bool issuer_wait(uint64_t *bar, uint32_t parity, volatile int *abort, int *flag,
                                            uint64_t limit_ns)
{
    return __all_sync(0xffffffffu, bwd_wait<kPoll>(bar, parity, abort, flag, limit_ns));
}

// Copies of the issuer still in flight after a failed wait: let them land before the CTA
// releases its memory. Loads of each ring were issued and waited in order.
struct Inflight {
    int issued[3] = {0, 0, 0}, waited[3] = {0, 0, 0};  // 0: fixed tiles, 1: ring A, 2: ring B
};

__device__ __forceinline__ void drain_issuer(uint64_t *bars, const Inflight &f, int ring_a)
{
    if (elect_one()) mma_commit(&bars[12]);
    __syncwarp();
    drain_wait(&bars[12], 0);
    for (int k = f.waited[0]; k < f.issued[0]; ++k) drain_wait(&bars[0], 0);
    for (int k = f.waited[1]; k < f.issued[1]; ++k) drain_wait(&bars[1 + k % ring_a], (k / ring_a) & 1);
    for (int k = f.waited[2]; k < f.issued[2]; ++k) drain_wait(&bars[4 + (k & 1)], (k >> 1) & 1);
}

// ---------------------------------------------------------------------------------
// 3. dQ: one CTA per (b, h, query block). Pipeline per kept block c (K_c in slot c mod 3
//    of the three-slot ring, V_c in slot c mod 2 of the two-slot ring):
//      issuer: S(0), dP(0); then for each c: [S(c) read] S(c+1); [dS(c) stored]
//              dQ += dS(c) K_c, dP(c+1); loads of K, V for c + 2;
//      compute: [S(c)] P in registers, arrive; [dP(c)] dS packed to bf16 over dP, arrive.
//    dS sits in the dP columns, so S(c+1) overlaps the dS step and dQ(c), dP(c+1) overlap
//    the next P step. (Issuing dP(c+1) ahead of dQ(c), with dS in two buffers of the spare
//    TMEM columns, measured 10% slower.)
// ---------------------------------------------------------------------------------
template <int D, bool kW, bool kPoll>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                       const BwdParams p)
{
    constexpr uint32_t kTileBytes = 128 * D * 2;
    const int item = blockIdx.x;
    const int bh = item / p.nqb, qb = item % p.nqb;
    int n = p.cnt[item];
    if (n < 0 || n > p.nkb) {
        if (threadIdx.x == 0) raise_flag(p.flag, AB_FLAG_BAD_INDEX);
        n = n < 0 ? 0 : p.nkb;
    }
    const size_t row0 = (size_t)bh * p.N_pad + (size_t)qb * 128;
    if (n == 0) {  // no kept block: no gradient reaches these queries
        zero_rows<D>(p.dq, row0);
        return;
    }
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    uint8_t *sQ = smem, *sG = smem + kTileMax;
    auto sK = [&](int slot) { return smem + (2 + slot) * kTileMax; };
    auto sV = [&](int slot) { return smem + (5 + slot) * kTileMax; };
    __shared__ __align__(8) uint64_t bars[kBars];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int b = 0; b < kBars; ++b) mbar_init(&bars[b], (b == 8 || b == 9) ? 256 : 1);
        abort_s = 0;
        fence_barrier_init();
    }
    if (warp == kIssuerWarp) {
        tmem_alloc(&tmem_slot, kBwdTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const uint32_t tS = tmem, tP = tmem + 128, tAcc = tmem + 256;  // S, dP then dS, dQ
    const int32_t *idx = p.idx + (size_t)item * p.nkb;
    const float *wrow = kW ? p.w + (size_t)item * p.nkb : nullptr;
    auto clamp_j = [&](int j) { return j < 0 ? 0 : (j >= p.nkb ? p.nkb - 1 : j); };

    if (warp == kIssuerWarp) {
        // ------------------------------ issuer warp ------------------------------
        Inflight f;
        auto block_of = [&](int c) {
            const int j = __ldg(idx + c);
            if ((j < 0 || j >= p.nkb) && lane == 0) raise_flag(p.flag, AB_FLAG_BAD_INDEX);
            return clamp_j(j);
        };
        auto load_k = [&](int c, int j) {
            const int slot = c % 3;
            if (elect_one()) {
                mbar_arrive_expect_tx(&bars[1 + slot], kTileBytes);
                tma_tile<D>(sK(slot), &tmK, &bars[1 + slot], j, bh);
            }
            __syncwarp();
            ++f.issued[1];
        };
        auto load_v = [&](int c, int j) {
            const int slot = c & 1;
            if (elect_one()) {
                mbar_arrive_expect_tx(&bars[4 + slot], kTileBytes);
                tma_tile<D>(sV(slot), &tmV, &bars[4 + slot], j, bh);
            }
            __syncwarp();
            ++f.issued[2];
        };
        auto kd = [&](int slot) { return smem_desc_sw128(smem_u32(sK(slot)), 16, 1024); };
        auto kd_mn = [&](int slot) { return smem_desc_sw128(smem_u32(sK(slot)), 16384, 1024); };
        auto vd = [&](int slot) { return smem_desc_sw128(smem_u32(sV(slot)), 16, 1024); };
        const uint64_t q_desc = smem_desc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t g_desc = smem_desc_sw128(smem_u32(sG), 16, 1024);
        volatile int *ab = &abort_s;
        if (elect_one()) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmG);
            mbar_arrive_expect_tx(&bars[0], 2 * kTileBytes);
            tma_tile<D>(sQ, &tmQ, &bars[0], qb, bh);
            tma_tile<D>(sG, &tmG, &bars[0], qb, bh);
        }
        __syncwarp();
        f.issued[0] = 1;
        {
            const int j0 = block_of(0);
            load_k(0, j0);
            load_v(0, j0);
        }
        if (n > 1) {
            const int j1 = block_of(1);
            load_k(1, j1);
            load_v(1, j1);
        }
        // the block index of the next pair to load, read one iteration ahead of its use
        int j_pre = n > 2 ? __ldg(idx + 2) : 0;
        bool ok = issuer_wait<kPoll>(&bars[0], 0, ab, p.flag, p.wait_ns);
        if (ok) f.waited[0] = 1;
        ok = ok && issuer_wait<kPoll>(&bars[1], 0, ab, p.flag, p.wait_ns);
        if (ok) ++f.waited[1];
        ok = ok && issuer_wait<kPoll>(&bars[4], 0, ab, p.flag, p.wait_ns);
        if (ok) {
            ++f.waited[2];
            tc_fence_after();
            if (elect_one()) {
                mma_rows<D>(tS, q_desc, kd(0));
                mma_commit(&bars[6]);
                mma_rows<D>(tP, g_desc, vd(0));
                mma_commit(&bars[7]);
            }
            __syncwarp();
        }
        for (int c = 0; ok && c < n; ++c) {
            // S(c) has been read: S(c + 1) may overwrite it
            if (!issuer_wait<kPoll>(&bars[8], c & 1, ab, p.flag, p.wait_ns)) { ok = false; break; }
            if (c + 1 < n) {
                const int ks = (c + 1) % 3;
                if (!issuer_wait<kPoll>(&bars[1 + ks], ((c + 1) / 3) & 1, ab, p.flag, p.wait_ns)) { ok = false; break; }
                ++f.waited[1];
                tc_fence_after();
                if (elect_one()) {
                    mma_rows<D>(tS, q_desc, kd(ks));
                    mma_commit(&bars[6]);
                }
                __syncwarp();
            }
            // dS(c) stored and dP(c) read: dQ += dS(c) K_c, then dP(c + 1) over it
            if (!issuer_wait<kPoll>(&bars[9], c & 1, ab, p.flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
                mma_packed<D>(tAcc, tP, kd_mn(c % 3), c > 0);
                if (c == n - 1) mma_commit(&bars[11]);
            }
            __syncwarp();
            if (c + 1 < n) {
                const int vs = (c + 1) & 1;
                if (!issuer_wait<kPoll>(&bars[4 + vs], ((c + 1) >> 1) & 1, ab, p.flag, p.wait_ns)) { ok = false; break; }
                ++f.waited[2];
                tc_fence_after();
                if (elect_one()) {
                    mma_rows<D>(tP, g_desc, vd(vs));
                    mma_commit(&bars[7]);
                }
                __syncwarp();
            }
            // K_{c-1} (read by dQ(c-1)) and V_c (read by dP(c)) are free: the compute warps
            // saw dP(c) done, which the pipe ran after dQ(c-1)
            if (c + 2 < n) {
                if ((j_pre < 0 || j_pre >= p.nkb) && lane == 0) raise_flag(p.flag, AB_FLAG_BAD_INDEX);
                const int j2 = clamp_j(j_pre);
                j_pre = c + 3 < n ? __ldg(idx + c + 3) : 0;
                load_k(c + 2, j2);
                load_v(c + 2, j2);
            }
        }
        // the CTA frees its tensor memory only after every MMA is done: on a failed wait the
        // drain, else the final commit (also when only the compute warps gave up)
        if (!ok)
            drain_issuer(bars, f, 3);
        else
            drain_wait(&bars[11], 0);
    } else {
        // ------------------------------ compute warps ------------------------------
        const int grp = warp & 3, half = warp >> 2;
        const uint32_t lane_off = (uint32_t)(32 * grp) << 16;
        const int row = 32 * grp + lane;  // query row of the block (TMEM lane)
        const float L2r = p.rowL2[row0 + row];
        const float Dr = p.rowD[row0 + row];
        volatile int *ab = &abort_s;
        int j_cur = clamp_j(__ldg(idx));
        float lw_cur = kW ? lw2_val(__ldg(wrow), p.flag, threadIdx.x == 0) : 0.f;
        bool ok = true;
        for (int c = 0; c < n; ++c) {
            // the next plan entry: loaded here, used only after this pair's work
            int j_raw = 0;
            float w_raw = 1.f;
            if (c + 1 < n) {
                j_raw = __ldg(idx + c + 1);
                if (kW) w_raw = __ldg(wrow + c + 1);
            }
            if (!__all_sync(0xffffffffu, bwd_wait<kPoll>(&bars[6], c & 1, ab, p.flag, p.wait_ns))) { ok = false; break; }
            tc_fence_after();
            // P = 2^(s scale_log2 + log2 w - L2) on the valid keys of block j
            const int nvalid = p.N - j_cur * 128;
            const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
            const uint64_t b2 = f2_pack(lw_cur - L2r, lw_cur - L2r);
            float pv[64];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t sv[32];
                tmem_ld32(tS + lane_off + half * 64 + ch * 32, sv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int key = half * 64 + ch * 32 + e;
                    const float2 r = exp2_pair(
                        f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2, b2),
                        (ch * 16 + e / 2) % 5 == 4);
                    pv[ch * 32 + e] = key < nvalid ? r.x : 0.f;
                    pv[ch * 32 + e + 1] = key + 1 < nvalid ? r.y : 0.f;
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[8]);
            if (!__all_sync(0xffffffffu, bwd_wait<kPoll>(&bars[7], c & 1, ab, p.flag, p.wait_ns))) { ok = false; break; }
            tc_fence_after();
            // dS = P (dP - D), packed to bf16 over the first 32 of this half's dP columns
            uint32_t pk[32];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t dv[32];
                tmem_ld32(tP + lane_off + half * 64 + ch * 32, dv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    pk[ch * 16 + e / 2] = pack_bf16x2(pv[ch * 32 + e] * (__uint_as_float(dv[e]) - Dr),
                                                      pv[ch * 32 + e + 1] * (__uint_as_float(dv[e + 1]) - Dr));
            }
            tmem_st32(tP + lane_off + half * 64, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[9]);
            j_cur = clamp_j(j_raw);
            lw_cur = kW ? lw2_val(w_raw, p.flag, threadIdx.x == 0) : 0.f;
        }
        if (ok) ok = __all_sync(0xffffffffu, bwd_wait<kPoll>(&bars[11], 0, ab, p.flag, p.wait_ns));
        if (ok) {
            tc_fence_after();
            store_acc_row<D>(tAcc + lane_off + half * (D / 2), p.dq + (row0 + row) * D + half * (D / 2),
                             p.scale, qb * 128 + row < p.N);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kIssuerWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kBwdTmemCols);
    }
}

// ---------------------------------------------------------------------------------
// 4. dK, dV: one CTA per (b, h, key block), over the kcount[bh][kb] query blocks that
//    kept it, ascending, read from the mark column. Pipeline per pair c (Q_c with its
//    rows' L2 and D, and dO_c, in slot c mod 2 of their rings):
//      issuer: S^T(0), dP^T(0); then for each c: [P^T(c) stored] dV += P^T dO_c,
//              S^T(c+1); [dS^T(c) stored] dK += dS^T Q_c, dP^T(c+1); [pair c done]
//              loads for c + 2 into its slots;
//      compute: [S^T(c)] P^T packed over S^T, arrive; [dP^T(c)] dS^T packed over dP^T,
//               arrive.
//    dV(c) and S^T(c+1) run while the warps form dS^T(c); dK(c) and dP^T(c+1) while they
//    form P^T(c+1).
// ---------------------------------------------------------------------------------
// Every warp walks the mark column in chunks of 32 (one ballot per chunk, the next
// chunk's entries already loaded), so all warps see the same sequence without talking
// to each other.
struct MarkWalk {
    const uint16_t *col;
    int nqb, base;
    uint32_t mask, mv, mv_next;
    __device__ uint32_t raw(int b) const
    {
        const int q = b + (int)(threadIdx.x & 31);
        return q < nqb ? (uint32_t)col[q] : 0u;
    }
    __device__ void start()
    {
        base = 0;
        mv = raw(0);
        mv_next = raw(32);
        mask = __ballot_sync(0xffffffffu, mv != 0);
    }
    __device__ bool next(int &qb, int &c)
    {
        while (mask == 0) {
            if (base + 32 >= nqb) return false;
            base += 32;
            mv = mv_next;
            mv_next = raw(base + 32);
            mask = __ballot_sync(0xffffffffu, mv != 0);
        }
        const int l = __ffs(mask) - 1;
        mask &= mask - 1;
        qb = base + l;
        c = (int)__shfl_sync(0xffffffffu, mv, l) - 1;
        return true;
    }
};

template <int D, bool kW, bool kPoll>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                         const BwdParams p)
{
    constexpr uint32_t kTileBytes = 128 * D * 2;
    const int item = blockIdx.x;
    const int bh = item / p.nkb, kb = item % p.nkb;
    const size_t row0 = (size_t)bh * p.N_pad + (size_t)kb * 128;
    const int n = (int)min(p.kcount[item], (uint32_t)p.nqb);
    if (n == 0) {  // no query block kept this key block
        zero_rows<D>(p.dk, row0);
        zero_rows<D>(p.dv, row0);
        return;
    }
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    uint8_t *sK = smem, *sV = smem + kTileMax;
    auto sQ = [&](int slot) { return smem + (2 + slot) * kTileMax; };
    auto sG = [&](int slot) { return smem + (4 + slot) * kTileMax; };
    __shared__ __align__(8) uint64_t bars[kBars];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_s;
    __shared__ __align__(16) float sLD[2][256];  // per slot: L2 of the 128 queries, then D
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int b = 0; b < kBars; ++b) mbar_init(&bars[b], (b == 8 || b == 9) ? 256 : 1);
        abort_s = 0;
        fence_barrier_init();
    }
    if (warp == kIssuerWarp) {
        tmem_alloc(&tmem_slot, kBwdTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    // S^T then P^T, dP^T then dS^T, dV, dK
    const uint32_t tS = tmem, tP = tmem + 128, tV = tmem + 256, tK = tmem + 256 + D;
    MarkWalk walk{p.mark + (size_t)item * p.nqb, p.nqb, 0, 0u, 0u, 0u};
    walk.start();
    volatile int *ab = &abort_s;

    if (warp == kIssuerWarp) {
        // ------------------------------ issuer warp ------------------------------
        Inflight f;
        auto next_qb = [&]() {
            int q = 0, c = 0;
            if (!walk.next(q, c) && lane == 0) raise_flag(p.flag, AB_FLAG_BAD_INDEX);
            return q;
        };
        auto load_q = [&](int c, int q) {
            const int slot = c & 1;
            if (elect_one()) {
                mbar_arrive_expect_tx(&bars[1 + slot], kTileBytes + 1024);
                tma_tile<D>(sQ(slot), &tmQ, &bars[1 + slot], q, bh);
                const size_t r = (size_t)bh * p.N_pad + (size_t)q * 128;
                bulk_load(&sLD[slot][0], p.rowL2 + r, 512, &bars[1 + slot]);
                bulk_load(&sLD[slot][128], p.rowD + r, 512, &bars[1 + slot]);
            }
            __syncwarp();
            ++f.issued[1];
        };
        auto load_g = [&](int c, int q) {
            const int slot = c & 1;
            if (elect_one()) {
                mbar_arrive_expect_tx(&bars[4 + slot], kTileBytes);
                tma_tile<D>(sG(slot), &tmG, &bars[4 + slot], q, bh);
            }
            __syncwarp();
            ++f.issued[2];
        };
        auto qd = [&](int slot) { return smem_desc_sw128(smem_u32(sQ(slot)), 16, 1024); };
        auto qd_mn = [&](int slot) { return smem_desc_sw128(smem_u32(sQ(slot)), 16384, 1024); };
        auto gd = [&](int slot) { return smem_desc_sw128(smem_u32(sG(slot)), 16, 1024); };
        auto gd_mn = [&](int slot) { return smem_desc_sw128(smem_u32(sG(slot)), 16384, 1024); };
        const uint64_t k_desc = smem_desc_sw128(smem_u32(sK), 16, 1024);
        const uint64_t v_desc = smem_desc_sw128(smem_u32(sV), 16, 1024);
        if (elect_one()) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmG);
            mbar_arrive_expect_tx(&bars[0], 2 * kTileBytes);
            tma_tile<D>(sK, &tmK, &bars[0], kb, bh);
            tma_tile<D>(sV, &tmV, &bars[0], kb, bh);
        }
        __syncwarp();
        f.issued[0] = 1;
        {
            const int q0 = next_qb();
            load_q(0, q0);
            load_g(0, q0);
        }
        if (n > 1) {
            const int q1 = next_qb();
            load_q(1, q1);
            load_g(1, q1);
        }
        bool ok = issuer_wait<kPoll>(&bars[0], 0, ab, p.flag, p.wait_ns);
        if (ok) f.waited[0] = 1;
        ok = ok && issuer_wait<kPoll>(&bars[1], 0, ab, p.flag, p.wait_ns);
        if (ok) ++f.waited[1];
        ok = ok && issuer_wait<kPoll>(&bars[4], 0, ab, p.flag, p.wait_ns);
        if (ok) {
            ++f.waited[2];
            tc_fence_after();
            if (elect_one()) {
                mma_rows<D>(tS, k_desc, qd(0));
                mma_commit(&bars[6]);
                mma_rows<D>(tP, v_desc, gd(0));
                mma_commit(&bars[7]);
            }
            __syncwarp();
        }
        for (int c = 0; ok && c < n; ++c) {
            const int s = c & 1, s1 = s ^ 1;
            // P^T(c) stored and S^T(c) read: dV += P^T dO_c, then S^T(c + 1) over it (the
            // pipe runs them in order; Q_{c+1} is the other slot of the ring)
            if (!issuer_wait<kPoll>(&bars[8], c & 1, ab, p.flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) mma_packed<D>(tV, tS, gd_mn(s), c > 0);
            __syncwarp();
            if (c + 1 < n) {
                if (!issuer_wait<kPoll>(&bars[1 + s1], ((c + 1) >> 1) & 1, ab, p.flag, p.wait_ns)) { ok = false; break; }
                ++f.waited[1];
                tc_fence_after();
                if (elect_one()) {
                    mma_rows<D>(tS, k_desc, qd(s1));
                    mma_commit(&bars[6]);
                }
                __syncwarp();
            }
            // dS^T(c) stored and dP^T(c) read: dK += dS^T Q_c, then dP^T(c + 1) over it
            if (!issuer_wait<kPoll>(&bars[9], c & 1, ab, p.flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
                mma_packed<D>(tK, tP, qd_mn(s), c > 0);
                mma_commit(&bars[10]);
                if (c == n - 1) mma_commit(&bars[11]);
            }
            __syncwarp();
            if (c + 1 < n) {
                if (!issuer_wait<kPoll>(&bars[4 + s1], ((c + 1) >> 1) & 1, ab, p.flag, p.wait_ns)) { ok = false; break; }
                ++f.waited[2];
                tc_fence_after();
                if (elect_one()) {
                    mma_rows<D>(tP, v_desc, gd(s1));
                    mma_commit(&bars[7]);
                }
                __syncwarp();
            }
            // pair c accumulated (dV(c), dK(c) and every earlier MMA done): its Q, rows and
            // dO slots take pair c + 2
            if (!issuer_wait<kPoll>(&bars[10], c & 1, ab, p.flag, p.wait_ns)) { ok = false; break; }
            if (c + 2 < n) {
                const int q2 = next_qb();
                load_q(c + 2, q2);
                load_g(c + 2, q2);
            }
        }
        if (!ok)
            drain_issuer(bars, f, 2);
        else
            drain_wait(&bars[11], 0);
    } else {
        // ------------------------------ compute warps ------------------------------
        const int grp = warp & 3, half = warp >> 2;
        const uint32_t lane_off = (uint32_t)(32 * grp) << 16;
        const int key = 32 * grp + lane;  // key row of the block (TMEM lane)
        const bool key_ok = kb * 128 + key < p.N;
        auto weight_ptr = [&](int q, int ce) { return p.w + ((size_t)bh * p.nqb + q) * p.nkb + ce; };
        int q_cur = 0, ce_cur = 0;
        walk.next(q_cur, ce_cur);
        float lw_cur = kW ? lw2_val(__ldg(weight_ptr(q_cur, ce_cur)), p.flag, threadIdx.x == 0) : 0.f;
        bool ok = true;
        for (int c = 0; c < n; ++c) {
            // the next pair's weight: loaded here, used only after this pair's work
            float w_raw = 1.f;
            if (c + 1 < n) {
                int q_nx = 0, ce_nx = 0;
                walk.next(q_nx, ce_nx);
                if (kW) w_raw = __ldg(weight_ptr(q_nx, ce_nx));
            }
            const int slot = c & 1;
            // the L2 and D rows arrive with Q_c
            if (!__all_sync(0xffffffffu, bwd_wait<kPoll>(&bars[1 + slot], (c >> 1) & 1, ab, p.flag, p.wait_ns))) { ok = false; break; }
            if (!__all_sync(0xffffffffu, bwd_wait<kPoll>(&bars[6], c & 1, ab, p.flag, p.wait_ns))) { ok = false; break; }
            tc_fence_after();
            // P^T = 2^(s scale_log2 + log2 w - L2_i) for this key over the half's queries
            float pv[64];
            uint32_t pk[32];
            const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
            uint32_t sv2[2][32];  // both 32-column halves of this warp's S^T columns, one wait
            tmem_ld32(tS + lane_off + half * 64, sv2[0]);
            tmem_ld32(tS + lane_off + half * 64 + 32, sv2[1]);
            tmem_wait_ld();
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                const uint32_t (&sv)[32] = sv2[ch];
                const float4 *l4 = reinterpret_cast<const float4 *>(&sLD[slot][half * 64 + ch * 32]);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 lq = l4[e4];
                    const int e = e4 * 4;
                    const float2 r0 = exp2_pair(
                        f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2,
                               f2_pack(lw_cur - lq.x, lw_cur - lq.y)),
                        (ch * 16 + e4 * 2) % 5 == 4);
                    const float2 r1 = exp2_pair(
                        f2_fma(f2_pack(__uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3])), sc2,
                               f2_pack(lw_cur - lq.z, lw_cur - lq.w)),
                        (ch * 16 + e4 * 2 + 1) % 5 == 4);
                    pv[ch * 32 + e] = key_ok ? r0.x : 0.f;
                    pv[ch * 32 + e + 1] = key_ok ? r0.y : 0.f;
                    pv[ch * 32 + e + 2] = key_ok ? r1.x : 0.f;
                    pv[ch * 32 + e + 3] = key_ok ? r1.y : 0.f;
                    pk[ch * 16 + e4 * 2] = pack_bf16x2(pv[ch * 32 + e], pv[ch * 32 + e + 1]);
                    pk[ch * 16 + e4 * 2 + 1] = pack_bf16x2(pv[ch * 32 + e + 2], pv[ch * 32 + e + 3]);
                }
            }
            tmem_st32(tS + lane_off + half * 64, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[8]);
            if (!__all_sync(0xffffffffu, bwd_wait<kPoll>(&bars[7], c & 1, ab, p.flag, p.wait_ns))) { ok = false; break; }
            tc_fence_after();
            // dS^T = P^T (dP^T - D_i)
            uint32_t dv2[2][32];
            tmem_ld32(tP + lane_off + half * 64, dv2[0]);
            tmem_ld32(tP + lane_off + half * 64 + 32, dv2[1]);
            tmem_wait_ld();
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                const uint32_t (&dv)[32] = dv2[ch];
                const float4 *d4 = reinterpret_cast<const float4 *>(&sLD[slot][128 + half * 64 + ch * 32]);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 dq = d4[e4];
                    const int e = ch * 32 + e4 * 4;
                    pk[ch * 16 + e4 * 2] = pack_bf16x2(pv[e] * (__uint_as_float(dv[e4 * 4]) - dq.x),
                                                       pv[e + 1] * (__uint_as_float(dv[e4 * 4 + 1]) - dq.y));
                    pk[ch * 16 + e4 * 2 + 1] = pack_bf16x2(pv[e + 2] * (__uint_as_float(dv[e4 * 4 + 2]) - dq.z),
                                                           pv[e + 3] * (__uint_as_float(dv[e4 * 4 + 3]) - dq.w));
                }
            }
            tmem_st32(tP + lane_off + half * 64, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[9]);
            lw_cur = kW ? lw2_val(w_raw, p.flag, threadIdx.x == 0) : 0.f;
        }
        if (ok) ok = __all_sync(0xffffffffu, bwd_wait<kPoll>(&bars[11], 0, ab, p.flag, p.wait_ns));
        if (ok) {
            tc_fence_after();
            store_acc_row<D>(tV + lane_off + half * (D / 2), p.dv + (row0 + key) * D + half * (D / 2), 1.f,
                             key_ok);
            store_acc_row<D>(tK + lane_off + half * (D / 2), p.dk + (row0 + key) * D + half * (D / 2),
                             p.scale, key_ok);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kIssuerWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kBwdTmemCols);
    }
}

// 3-D map over a [B*H, N_pad, d] bf16 tensor with row extent N (rows >= N read as 0),
// box 64 columns x 128 rows, 128-byte swizzle.
bool bwd_tmap(CUtensorMap *tm, const void *base, int BH, int N, int N_pad, int d)
{
    return make_tmap_bf16_3d(tm, base, (uint64_t)d, (uint64_t)N, (uint64_t)BH, (uint64_t)d * 2,
                             (uint64_t)N_pad * d * 2, 64, 128);
}

template <int D, bool kW, bool kPoll>
cudaError_t launch_bwd_t(const AttnBwdLaunch &a, cudaStream_t st)
{
    const int BH = a.B * a.H, nb = a.N_pad / 128;
    const AttnBwdLayout L = attn_bwd_layout((size_t)BH, (size_t)a.N_pad);
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    float *rowD = reinterpret_cast<float *>(ws + L.rowD);
    float *rowL2 = reinterpret_cast<float *>(ws + L.rowL2);
    uint16_t *mark = reinterpret_cast<uint16_t *>(ws + L.mark);
    uint32_t *kcount = reinterpret_cast<uint32_t *>(ws + L.kcount);
    CUtensorMap tq, tk, tv, tg;
    if (!bwd_tmap(&tq, a.q, BH, a.N, a.N_pad, D) || !bwd_tmap(&tk, a.k, BH, a.N, a.N_pad, D) ||
        !bwd_tmap(&tv, a.v, BH, a.N, a.N_pad, D) || !bwd_tmap(&tg, a.dout, BH, a.N, a.N_pad, D))
        return cudaErrorInvalidValue;
    const size_t rows = (size_t)BH * a.N_pad;
    // the mark table and the per-key-block counts, one contiguous region
    cudaError_t e = cudaMemsetAsync(mark, 0, L.total - L.mark, st);
    if (e != cudaSuccess) return e;
    const unsigned rs_grid = (unsigned)((rows + 15) / 16);
    if (a.out_f32)
        attn_bwd_rowstats_kernel<D, true><<<rs_grid, 256, 0, st>>>(
            a.out, static_cast<const __nv_bfloat16 *>(a.dout), a.lse, rowD, rowL2, rows, a.N, a.N_pad);
    else
        attn_bwd_rowstats_kernel<D, false><<<rs_grid, 256, 0, st>>>(
            a.out, static_cast<const __nv_bfloat16 *>(a.dout), a.lse, rowD, rowL2, rows, a.N, a.N_pad);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t plan_rows = (size_t)BH * nb;
    attn_bwd_mark_kernel<<<(unsigned)((plan_rows + 7) / 8), 256, 0, st>>>(a.idx, a.cnt, mark, kcount,
                                                                           plan_rows, nb, nb, a.flag);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    BwdParams p;
    p.idx = a.idx;
    p.cnt = a.cnt;
    p.w = a.w;
    p.rowD = rowD;
    p.rowL2 = rowL2;
    p.mark = mark;
    p.kcount = kcount;
    p.dq = a.dq;
    p.dk = a.dk;
    p.dv = a.dv;
    p.flag = a.flag;
    p.N = a.N;
    p.N_pad = a.N_pad;
    p.nqb = nb;
    p.nkb = nb;
    p.scale = (float)(1.0 / std::sqrt((double)D));
    p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    p.wait_ns = a.wait_ns > 0 ? a.wait_ns : kWaitLimitNs;
    e = cudaFuncSetAttribute(attn_bwd_dq_kernel<D, kW, kPoll>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kDqSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D, kW, kPoll>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kDkdvSmem);
    if (e != cudaSuccess) return e;
    attn_bwd_dq_kernel<D, kW, kPoll><<<(unsigned)plan_rows, kBwdThreads, kDqSmem, st>>>(tq, tk, tv, tg, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    attn_bwd_dkdv_kernel<D, kW, kPoll><<<(unsigned)plan_rows, kBwdThreads, kDkdvSmem, st>>>(tq, tk, tv, tg, p);
    return cudaGetLastError();
}

template <bool kPoll>
cudaError_t launch_attn_bwd_p(const AttnBwdLaunch &a, cudaStream_t st)
{
    const bool weighted = a.w != nullptr;
    if (a.d == 128)
        return weighted ? launch_bwd_t<128, true, kPoll>(a, st) : launch_bwd_t<128, false, kPoll>(a, st);
    return weighted ? launch_bwd_t<64, true, kPoll>(a, st) : launch_bwd_t<64, false, kPoll>(a, st);
}

// A wait limit below 1 ms (the test entry) takes the polling instantiation.
cudaError_t launch_attn_bwd(const AttnBwdLaunch &a, cudaStream_t st)
{
    if (a.wait_ns > 0 && a.wait_ns < 1000000ull) return launch_attn_bwd_p<true>(a, st);
    return launch_attn_bwd_p<false>(a, st);
}

// The shape rules of the forward calls (include/ab_attn.h): 128-token blocks, d in
// {64, 128}, bf16 tokens, at most AB_MAX_BLOCKS blocks and 65535 head pairs.
ab_status bwd_check_shape(const ab_shape &s)
{
    if (s.B <= 0 || s.H <= 0 || s.N <= 0 || s.N_pad <= 0 || s.d <= 0) return AB_ERR_SHAPE;
    if (s.N_pad % AB_BLOCK != 0 || s.N > s.N_pad || s.N_pad - s.N >= AB_BLOCK) return AB_ERR_SHAPE;
    if (s.dtype != AB_BF16) return AB_ERR_DTYPE;
    if (s.d != 64 && s.d != 128) return AB_ERR_UNSUPPORTED;
    if (s.N_pad / AB_BLOCK > AB_MAX_BLOCKS) return AB_ERR_RANGE;
    if ((long long)s.B * s.H > 65535LL) return AB_ERR_RANGE;
    return AB_OK;
}

bool bwd_aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Argument checks and launch shared by ab_attn_bwd and its wait-limit test entry.
ab_status attn_bwd_common(const void *q, const void *k, const void *v, ab_shape s, const int32_t *idx,
                          const int32_t *cnt, const float *w, const void *out, ab_dtype out_dtype,
                          const float *lse, const void *dout, float *dq, float *dk, float *dv,
                          void *workspace, size_t workspace_bytes, int *dev_flag, void *stream,
                          unsigned long long wait_ns)
{
    if (!q || !k || !v || !idx || !cnt || !out || !lse || !dout || !dq || !dk || !dv)
        return AB_ERR_NULL;
    const ab_status st = bwd_check_shape(s);
    if (st != AB_OK) return st;
    if (out_dtype != AB_BF16 && out_dtype != AB_F32) return AB_ERR_DTYPE;
    if (!bwd_aligned16(q) || !bwd_aligned16(k) || !bwd_aligned16(v) || !bwd_aligned16(idx) ||
        !bwd_aligned16(cnt) || (w && !bwd_aligned16(w)) || !bwd_aligned16(out) ||
        !bwd_aligned16(lse) || !bwd_aligned16(dout) || !bwd_aligned16(dq) || !bwd_aligned16(dk) ||
        !bwd_aligned16(dv) || (workspace && !bwd_aligned16(workspace)))
        return AB_ERR_ALIGN;
    const AttnBwdLayout L = attn_bwd_layout((size_t)s.B * s.H, (size_t)s.N_pad);
    if (!workspace || workspace_bytes < L.total) return AB_ERR_WORKSPACE;
    AttnBwdLaunch a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.out = out;
    a.out_f32 = out_dtype == AB_F32;
    a.dout = dout;
    a.lse = lse;
    a.idx = idx;
    a.cnt = cnt;
    a.w = w;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.workspace = workspace;
    a.flag = dev_flag;
    a.B = s.B;
    a.H = s.H;
    a.N = s.N;
    a.N_pad = s.N_pad;
    a.d = s.d;
    a.wait_ns = wait_ns;
    return status_of(launch_attn_bwd(a, (cudaStream_t)stream));
}

}  // namespace

}  // namespace ab

extern "C" {

ab_status ab_attn_bwd_workspace_size(ab_shape s, size_t *bytes)
{
    if (!bytes) return AB_ERR_NULL;
    *bytes = 0;
    const ab_status st = ab::bwd_check_shape(s);
    if (st != AB_OK) return st;
    *bytes = ab::attn_bwd_layout((size_t)s.B * s.H, (size_t)s.N_pad).total;
    return AB_OK;
}

ab_status ab_attn_bwd(const void *q, const void *k, const void *v, ab_shape s, const int32_t *idx,
                      const int32_t *cnt, const float *w, const void *out, ab_dtype out_dtype,
                      const float *lse, const void *dout, float *dq, float *dk, float *dv,
                      void *workspace, size_t workspace_bytes, int *dev_flag, void *stream)
{
    nvtxRangePushA("ab_attn_bwd");
    struct Pop {
        ~Pop() { nvtxRangePop(); }
    } pop;
    return ab::attn_bwd_common(q, k, v, s, idx, cnt, w, out, out_dtype, lse, dout, dq, dk, dv, workspace,
                               workspace_bytes, dev_flag, stream, 0);
}

ab_status ab_selftest_attn_bwd_wait_limit(const void *q, const void *k, const void *v, ab_shape s,
                                          const int32_t *idx, const int32_t *cnt, const float *w,
                                          const void *out, ab_dtype out_dtype, const float *lse,
                                          const void *dout, float *dq, float *dk, float *dv,
                                          void *workspace, size_t workspace_bytes, int *dev_flag,
                                          int limit_ns, void *stream)
{
    nvtxRangePushA("ab_selftest_attn_bwd_wait_limit");
    struct Pop {
        ~Pop() { nvtxRangePop(); }
    } pop;
    if (!dev_flag) return AB_ERR_NULL;
    if (limit_ns < 1 || limit_ns > 1000000000) return AB_ERR_RANGE;
    return ab::attn_bwd_common(q, k, v, s, idx, cnt, w, out, out_dtype, lse, dout, dq, dk, dv, workspace,
                               workspace_bytes, dev_flag, stream, (unsigned long long)limit_ns);
}

}  // extern "C"
