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
//      for the plan entry c that keeps the pair (zeroed just before; a second mark of the
//      same pair is a duplicate block in a row and raises AB_FLAG_BAD_INDEX);
//   3. dQ: one CTA per (b, h, query block), over its kept key blocks in plan order:
//      S = Q K_j^T and dP = dO V_j^T into TMEM (SS MMAs, both operands K-major), dS packed
//      to bf16 over S, dQ += dS K_j (TS MMA: dS from TMEM, K_j as an MN-major operand);
//   4. dK, dV: one CTA per (b, h, key block), over the query blocks that kept it in
//      ascending order (read from the mark table): S^T = K Q^T and dP^T = V dO^T, then
//      dV += P^T dO and dK += dS^T Q (TS MMAs, dO and Q as MN-major operands).
// Every sum runs in a fixed order, so the result does not depend on scheduling. The two
// gradient kernels share one structure: 8 warps; warp w reads TMEM lanes 32 (w mod 4) ..
// +31 (its rows) and half w / 4 of the columns; thread 0 issues the TMA copies and the
// MMAs; the K/V (dQ kernel) or Q/dO (dK/dV kernel) tiles of the next pair load while the
// current one is computed (two stages). Tiles arrive by TMA in 64-column boxes with the
// 128-byte swizzle, as in the forward kernel. Every wait is bounded; a wait that gives up
// raises AB_FLAG_TIMEOUT, and the CTA lets its copies and MMAs land and frees its tensor
// memory before it returns. The C entry points ab_attn_bwd and ab_attn_bwd_workspace_size
// are at the end of this file.
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
// lse_i log2e (fp32 [BH][N_pad] each), and the plan's mark table uint16 [BH][n_kb][n_qb].
struct AttnBwdLayout {
    size_t rowD, rowL2, mark, total;
};

AttnBwdLayout attn_bwd_layout(size_t BH, size_t N_pad)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t nb = N_pad / 128;
    AttnBwdLayout L;
    L.rowD = 0;
    L.rowL2 = up(BH * N_pad * sizeof(float));
    L.mark = up(L.rowL2 + BH * N_pad * sizeof(float));
    L.total = up(L.mark + BH * nb * nb * sizeof(uint16_t));
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
};

constexpr int kBwdThreads = 256;
constexpr int kBwdTmemCols = 512;
constexpr int kTileMax = 128 * 128 * 2;     // one 128 x 128 bf16 tile
constexpr int kBwdSmem = 6 * kTileMax + 1024;  // six tile slots + alignment slack: 1 CTA / SM

struct BwdParams {
    const int32_t *idx, *cnt;
    const float *w;  // nullptr: every weight 1 (top-k)
    const float *rowD, *rowL2;
    const uint16_t *mark;
    float *dq, *dk, *dv;
    int *flag;
    int N, N_pad, nqb, nkb;
    float scale, scale_log2;
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

__device__ __forceinline__ float lw2_of(const float *w, int *flag, bool report)
{
    if (!w) return 0.f;
    const float wj = __ldg(w);
    if (wj > 0.f && wj < INFINITY) return fast_log2(wj);
    if (report) raise_flag(flag, AB_FLAG_BAD_WEIGHT);
    return 0.f;
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
//    j (one warp per plan row).
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) attn_bwd_mark_kernel(const int32_t *idx, const int32_t *cnt,
                                                            uint16_t *mark, size_t n_rows, int nqb,
                                                            int nkb, int *flag)
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
    }
}

// ---------------------------------------------------------------------------------
// Shared pieces of the two gradient kernels.
// ---------------------------------------------------------------------------------
struct BwdCta {
    uint64_t *bars;  // 0: first tiles, 1-2: stage tiles, 3: S/dP done, 4: accumulate done, 5: drain
    volatile int *abort;
    int *flag;
};

// Thread 0's bounded wait.
__device__ __forceinline__ bool bwd_wait(const BwdCta &c, uint64_t *bar, uint32_t parity)
{
    return mbar_wait(bar, parity, c.abort, c.flag);
}

// ---------------------------------------------------------------------------------
// 3. dQ: one CTA per (b, h, query block).
// ---------------------------------------------------------------------------------
template <int D, bool kW>
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
    __shared__ __align__(8) uint64_t bars[6];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int b = 0; b < 6; ++b) mbar_init(&bars[b], 1);
        abort_s = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, kBwdTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const uint32_t tS = tmem, tP = tmem + 128, tAcc = tmem + 256;  // S then dS, dP, dQ
    const BwdCta cta{bars, &abort_s, p.flag};
    const int grp = warp & 3, half = warp >> 2;
    const uint32_t lane_off = (uint32_t)(32 * grp) << 16;
    const int row = 32 * grp + lane;  // query row of the block (TMEM lane)
    const float L2r = p.rowL2[row0 + row];
    const float Dr = p.rowD[row0 + row];
    const int32_t *idx = p.idx + (size_t)item * p.nkb;
    const float *wrow = kW ? p.w + (size_t)item * p.nkb : nullptr;
    auto block_of = [&](int c) {
        const int j = __ldg(idx + c);
        if (j >= 0 && j < p.nkb) return j;
        if (threadIdx.x == 0) raise_flag(p.flag, AB_FLAG_BAD_INDEX);
        return j < 0 ? 0 : p.nkb - 1;
    };
    auto sK = [&](int s) { return smem + (2 + 2 * s) * kTileMax; };
    auto sV = [&](int s) { return smem + (3 + 2 * s) * kTileMax; };
    const uint64_t q_desc = smem_desc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t g_desc = smem_desc_sw128(smem_u32(sG), 16, 1024);

    // thread 0's bookkeeping of copies in flight (for the drain after a failed wait)
    bool first_done = false;
    int kv_issued = 0, kv_done = 0;
    auto issue_kv = [&](int c) {
        const int j = block_of(c);
        const int s = c & 1;
        mbar_arrive_expect_tx(&bars[1 + s], 2 * kTileBytes);
        tma_tile<D>(sK(s), &tmK, &bars[1 + s], j, bh);
        tma_tile<D>(sV(s), &tmV, &bars[1 + s], j, bh);
        ++kv_issued;
    };
    bool ok0 = true;  // thread 0: every wait so far succeeded
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmG);
        mbar_arrive_expect_tx(&bars[0], 2 * kTileBytes);
        tma_tile<D>(sQ, &tmQ, &bars[0], qb, bh);
        tma_tile<D>(sG, &tmG, &bars[0], qb, bh);
        issue_kv(0);
    }
    bool failed = false;
    for (int c = 0; c < n; ++c) {
        const int s = c & 1;
        const int j = block_of(c);
        const float lw2 = kW ? lw2_of(wrow + c, p.flag, threadIdx.x == 0) : 0.f;
        if (warp == 0) {
            if (lane == 0) {
                if (c == 0) ok0 = first_done = bwd_wait(cta, &bars[0], 0);
                if (ok0) ok0 = bwd_wait(cta, &bars[1 + s], (c >> 1) & 1);
                if (ok0) {
                    ++kv_done;
                    tc_fence_after();
                    mma_rows<D>(tS, q_desc, smem_desc_sw128(smem_u32(sK(s)), 16, 1024));
                    mma_rows<D>(tP, g_desc, smem_desc_sw128(smem_u32(sV(s)), 16, 1024));
                    mma_commit(&bars[3]);
                }
                // the other stage is free once dQ of pair c - 1 is done: load pair c + 1
                if (ok0 && c >= 1) ok0 = bwd_wait(cta, &bars[4], (c - 1) & 1);
                if (ok0 && c + 1 < n) issue_kv(c + 1);
            }
            __syncwarp();
        }
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[3], c & 1, &abort_s, p.flag));
        if (ok) {
            tc_fence_after();
            // P = 2^(s scale_log2 + log2 w - L2) on the valid keys; dS = P (dP - D)
            const int nvalid = p.N - j * 128;
            const float bias = lw2 - L2r;
            uint32_t pk[32];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t sv[32], dv[32];
                tmem_ld32(tS + lane_off + half * 64 + ch * 32, sv);
                tmem_ld32(tP + lane_off + half * 64 + ch * 32, dv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int key = half * 64 + ch * 32 + e;
                    const float p0 = key < nvalid ? fast_exp2(fmaf(__uint_as_float(sv[e]), p.scale_log2, bias)) : 0.f;
                    const float p1 = key + 1 < nvalid ? fast_exp2(fmaf(__uint_as_float(sv[e + 1]), p.scale_log2, bias)) : 0.f;
                    pk[ch * 16 + e / 2] = pack_bf16x2(p0 * (__uint_as_float(dv[e]) - Dr),
                                                      p1 * (__uint_as_float(dv[e + 1]) - Dr));
                }
            }
            tmem_st32(tS + lane_off + half * 64, pk);
            tmem_wait_st();
        }
        tc_fence_before();
        if (__syncthreads_or(!ok || (threadIdx.x == 0 && !ok0))) {
            failed = true;
            break;
        }
        if (warp == 0) {
            if (lane == 0) {
                tc_fence_after();
                mma_packed<D>(tAcc, tS, smem_desc_sw128(smem_u32(sK(s)), 16384, 1024), c > 0);
                mma_commit(&bars[4]);
            }
            __syncwarp();
        }
    }
    bool ok_end = !failed;
    if (ok_end) ok_end = __all_sync(0xffffffffu, mbar_wait(&bars[4], (n - 1) & 1, &abort_s, p.flag));
    if (ok_end) {
        tc_fence_after();
        store_acc_row<D>(tAcc + lane_off + half * (D / 2), p.dq + (row0 + row) * D + half * (D / 2),
                         p.scale, qb * 128 + row < p.N);
    }
    if (threadIdx.x == 0 && (failed || !ok_end)) {
        // let the copies and MMAs in flight land before the memory is released
        mma_commit(&bars[5]);
        drain_wait(&bars[5], 0);
        if (!first_done) drain_wait(&bars[0], 0);
        for (int k = kv_done; k < kv_issued; ++k) drain_wait(&bars[1 + (k & 1)], (k >> 1) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kBwdTmemCols);
    }
}

// ---------------------------------------------------------------------------------
// 4. dK, dV: one CTA per (b, h, key block).
// ---------------------------------------------------------------------------------
// The query blocks that kept this key block, in ascending order, from its mark column:
// every warp walks the column in chunks of 32 (one ballot per chunk), so all warps see
// the same sequence without talking to each other.
struct MarkWalk {
    const uint16_t *col;
    int nqb, base;
    uint32_t mask, mv;
    __device__ void load(int b)
    {
        base = b;
        const int q = b + (int)(threadIdx.x & 31);
        mv = q < nqb ? col[q] : 0u;
        mask = __ballot_sync(0xffffffffu, mv != 0);
    }
    __device__ bool next(int &qb, int &c)
    {
        while (mask == 0) {
            if (base + 32 >= nqb) return false;
            load(base + 32);
        }
        const int l = __ffs(mask) - 1;
        mask &= mask - 1;
        qb = base + l;
        c = (int)__shfl_sync(0xffffffffu, mv, l) - 1;
        return true;
    }
};

template <int D, bool kW>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                         const BwdParams p)
{
    constexpr uint32_t kTileBytes = 128 * D * 2;
    const int item = blockIdx.x;
    const int bh = item / p.nkb, kb = item % p.nkb;
    const size_t row0 = (size_t)bh * p.N_pad + (size_t)kb * 128;
    MarkWalk walk{p.mark + (size_t)item * p.nqb, p.nqb, 0, 0u, 0u};
    walk.load(0);
    int cur_qb = 0, cur_c = 0, nxt_qb = 0, nxt_c = 0;
    bool have_cur = walk.next(cur_qb, cur_c);
    if (!have_cur) {  // no query block kept this key block
        zero_rows<D>(p.dk, row0);
        zero_rows<D>(p.dv, row0);
        return;
    }
    bool have_nxt = walk.next(nxt_qb, nxt_c);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    uint8_t *sK = smem, *sV = smem + kTileMax;
    __shared__ __align__(8) uint64_t bars[6];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_s;
    __shared__ __align__(16) float sL2[2][128];
    __shared__ __align__(16) float sD[2][128];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int b = 0; b < 6; ++b) mbar_init(&bars[b], 1);
        abort_s = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, kBwdTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x < 128) {
        const size_t r = (size_t)bh * p.N_pad + (size_t)cur_qb * 128 + threadIdx.x;
        sL2[0][threadIdx.x] = p.rowL2[r];
        sD[0][threadIdx.x] = p.rowD[r];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    // S^T then P^T, dP^T then dS^T, dV, dK
    const uint32_t tS = tmem, tP = tmem + 128, tV = tmem + 256, tK = tmem + 256 + D;
    const BwdCta cta{bars, &abort_s, p.flag};
    const int grp = warp & 3, half = warp >> 2;
    const uint32_t lane_off = (uint32_t)(32 * grp) << 16;
    const int key = 32 * grp + lane;  // key row of the block (TMEM lane)
    const bool key_ok = kb * 128 + key < p.N;
    auto sQ = [&](int s) { return smem + (2 + 2 * s) * kTileMax; };
    auto sG = [&](int s) { return smem + (3 + 2 * s) * kTileMax; };
    const uint64_t k_desc = smem_desc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t v_desc = smem_desc_sw128(smem_u32(sV), 16, 1024);

    bool first_done = false;
    int qg_issued = 0, qg_done = 0;
    auto issue_qg = [&](int it, int qbl) {
        const int s = it & 1;
        mbar_arrive_expect_tx(&bars[1 + s], 2 * kTileBytes);
        tma_tile<D>(sQ(s), &tmQ, &bars[1 + s], qbl, bh);
        tma_tile<D>(sG(s), &tmG, &bars[1 + s], qbl, bh);
        ++qg_issued;
    };
    bool ok0 = true;
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmG);
        mbar_arrive_expect_tx(&bars[0], 2 * kTileBytes);
        tma_tile<D>(sK, &tmK, &bars[0], kb, bh);
        tma_tile<D>(sV, &tmV, &bars[0], kb, bh);
        issue_qg(0, cur_qb);
    }
    bool failed = false;
    int it = 0;
    for (; have_cur; ++it) {
        const int s = it & 1;
        const float lw2 = kW ? lw2_of(p.w + ((size_t)bh * p.nqb + cur_qb) * p.nkb + cur_c, p.flag,
                                      threadIdx.x == 0)
                             : 0.f;
        if (warp == 0) {
            if (lane == 0) {
                if (it == 0) ok0 = first_done = bwd_wait(cta, &bars[0], 0);
                if (ok0) ok0 = bwd_wait(cta, &bars[1 + s], (it >> 1) & 1);
                if (ok0) {
                    ++qg_done;
                    tc_fence_after();
                    mma_rows<D>(tS, k_desc, smem_desc_sw128(smem_u32(sQ(s)), 16, 1024));
                    mma_rows<D>(tP, v_desc, smem_desc_sw128(smem_u32(sG(s)), 16, 1024));
                    mma_commit(&bars[3]);
                }
                // the other stage is free once dV, dK of pair it - 1 are done
                if (ok0 && it >= 1) ok0 = bwd_wait(cta, &bars[4], (it - 1) & 1);
                if (ok0 && have_nxt) issue_qg(it + 1, nxt_qb);
            }
            __syncwarp();
        }
        // the next pair's row statistics (stage s^1 was last read before the previous
        // iteration's barrier)
        if (have_nxt && threadIdx.x < 128) {
            const size_t r = (size_t)bh * p.N_pad + (size_t)nxt_qb * 128 + threadIdx.x;
            sL2[s ^ 1][threadIdx.x] = p.rowL2[r];
            sD[s ^ 1][threadIdx.x] = p.rowD[r];
        }
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[3], it & 1, &abort_s, p.flag));
        if (ok) {
            tc_fence_after();
            // P^T and dS^T for this thread's key over the half's 64 queries
            uint32_t pp[32], pd[32];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t sv[32], dv[32];
                tmem_ld32(tS + lane_off + half * 64 + ch * 32, sv);
                tmem_ld32(tP + lane_off + half * 64 + ch * 32, dv);
                tmem_wait_ld();
                const float4 *l4 = reinterpret_cast<const float4 *>(&sL2[s][half * 64 + ch * 32]);
                const float4 *d4 = reinterpret_cast<const float4 *>(&sD[s][half * 64 + ch * 32]);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 lq = l4[e4], dq = d4[e4];
                    const float lv[4] = {lq.x, lq.y, lq.z, lq.w};
                    const float dd[4] = {dq.x, dq.y, dq.z, dq.w};
                    float pv[4], ds[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int e = e4 * 4 + u;
                        pv[u] = key_ok ? fast_exp2(fmaf(__uint_as_float(sv[e]), p.scale_log2, lw2 - lv[u])) : 0.f;
                        ds[u] = pv[u] * (__uint_as_float(dv[e]) - dd[u]);
                    }
                    pp[ch * 16 + e4 * 2] = pack_bf16x2(pv[0], pv[1]);
                    pp[ch * 16 + e4 * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
                    pd[ch * 16 + e4 * 2] = pack_bf16x2(ds[0], ds[1]);
                    pd[ch * 16 + e4 * 2 + 1] = pack_bf16x2(ds[2], ds[3]);
                }
            }
            tmem_st32(tS + lane_off + half * 64, pp);
            tmem_st32(tP + lane_off + half * 64, pd);
            tmem_wait_st();
        }
        tc_fence_before();
        if (__syncthreads_or(!ok || (threadIdx.x == 0 && !ok0))) {
            failed = true;
            break;
        }
        if (warp == 0) {
            if (lane == 0) {
                tc_fence_after();
                mma_packed<D>(tV, tS, smem_desc_sw128(smem_u32(sG(s)), 16384, 1024), it > 0);
                mma_packed<D>(tK, tP, smem_desc_sw128(smem_u32(sQ(s)), 16384, 1024), it > 0);
                mma_commit(&bars[4]);
            }
            __syncwarp();
        }
        cur_qb = nxt_qb;
        cur_c = nxt_c;
        have_cur = have_nxt;
        if (have_cur) have_nxt = walk.next(nxt_qb, nxt_c);
    }
    bool ok_end = !failed;
    if (ok_end) ok_end = __all_sync(0xffffffffu, mbar_wait(&bars[4], (it - 1) & 1, &abort_s, p.flag));
    if (ok_end) {
        tc_fence_after();
        store_acc_row<D>(tV + lane_off + half * (D / 2), p.dv + (row0 + key) * D + half * (D / 2), 1.f,
                         key_ok);
        store_acc_row<D>(tK + lane_off + half * (D / 2), p.dk + (row0 + key) * D + half * (D / 2),
                         p.scale, key_ok);
    }
    if (threadIdx.x == 0 && (failed || !ok_end)) {
        mma_commit(&bars[5]);
        drain_wait(&bars[5], 0);
        if (!first_done) drain_wait(&bars[0], 0);
        for (int k = qg_done; k < qg_issued; ++k) drain_wait(&bars[1 + (k & 1)], (k >> 1) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
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

template <int D, bool kW>
cudaError_t launch_bwd_t(const AttnBwdLaunch &a, cudaStream_t st)
{
    const int BH = a.B * a.H, nb = a.N_pad / 128;
    const AttnBwdLayout L = attn_bwd_layout((size_t)BH, (size_t)a.N_pad);
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    float *rowD = reinterpret_cast<float *>(ws + L.rowD);
    float *rowL2 = reinterpret_cast<float *>(ws + L.rowL2);
    uint16_t *mark = reinterpret_cast<uint16_t *>(ws + L.mark);
    CUtensorMap tq, tk, tv, tg;
    if (!bwd_tmap(&tq, a.q, BH, a.N, a.N_pad, D) || !bwd_tmap(&tk, a.k, BH, a.N, a.N_pad, D) ||
        !bwd_tmap(&tv, a.v, BH, a.N, a.N_pad, D) || !bwd_tmap(&tg, a.dout, BH, a.N, a.N_pad, D))
        return cudaErrorInvalidValue;
    const size_t rows = (size_t)BH * a.N_pad;
    cudaError_t e = cudaMemsetAsync(mark, 0, (size_t)BH * nb * nb * sizeof(uint16_t), st);
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
    attn_bwd_mark_kernel<<<(unsigned)((plan_rows + 7) / 8), 256, 0, st>>>(a.idx, a.cnt, mark, plan_rows,
                                                                           nb, nb, a.flag);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    BwdParams p;
    p.idx = a.idx;
    p.cnt = a.cnt;
    p.w = a.w;
    p.rowD = rowD;
    p.rowL2 = rowL2;
    p.mark = mark;
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
    e = cudaFuncSetAttribute(attn_bwd_dq_kernel<D, kW>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D, kW>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdSmem);
    if (e != cudaSuccess) return e;
    attn_bwd_dq_kernel<D, kW><<<(unsigned)plan_rows, kBwdThreads, kBwdSmem, st>>>(tq, tk, tv, tg, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    attn_bwd_dkdv_kernel<D, kW><<<(unsigned)plan_rows, kBwdThreads, kBwdSmem, st>>>(tq, tk, tv, tg, p);
    return cudaGetLastError();
}

cudaError_t launch_attn_bwd(const AttnBwdLaunch &a, cudaStream_t st)
{
    const bool weighted = a.w != nullptr;
    if (a.d == 128) return weighted ? launch_bwd_t<128, true>(a, st) : launch_bwd_t<128, false>(a, st);
    return weighted ? launch_bwd_t<64, true>(a, st) : launch_bwd_t<64, false>(a, st);
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
    using ab::bwd_aligned16;
    if (!q || !k || !v || !idx || !cnt || !out || !lse || !dout || !dq || !dk || !dv)
        return AB_ERR_NULL;
    const ab_status st = ab::bwd_check_shape(s);
    if (st != AB_OK) return st;
    if (out_dtype != AB_BF16 && out_dtype != AB_F32) return AB_ERR_DTYPE;
    if (!bwd_aligned16(q) || !bwd_aligned16(k) || !bwd_aligned16(v) || !bwd_aligned16(idx) ||
        !bwd_aligned16(cnt) || (w && !bwd_aligned16(w)) || !bwd_aligned16(out) ||
        !bwd_aligned16(lse) || !bwd_aligned16(dout) || !bwd_aligned16(dq) || !bwd_aligned16(dk) ||
        !bwd_aligned16(dv) || (workspace && !bwd_aligned16(workspace)))
        return AB_ERR_ALIGN;
    const ab::AttnBwdLayout L = ab::attn_bwd_layout((size_t)s.B * s.H, (size_t)s.N_pad);
    if (!workspace || workspace_bytes < L.total) return AB_ERR_WORKSPACE;
    ab::AttnBwdLaunch a;
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
    return ab::status_of(ab::launch_attn_bwd(a, (cudaStream_t)stream));
}

}  // extern "C"
