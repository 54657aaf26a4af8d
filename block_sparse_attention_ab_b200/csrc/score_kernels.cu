// score_kernels.cu -- IBCS block scoring on sm_100a (AB-Attention news page, section
// «Три приёма AB-Attention», first technique): mean key per 128-token key block,
// per-query-block k-means into C <= 8 weighted clusters, and the block score
// s_j = sum_c w_c softmax_j(cent_c . kbar_j / sqrt(d)).
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ab_device.cuh"
#include "ab_kernels.h"

namespace ab {

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// ---------------------------------------------------------------------------------
// Mean key: one CTA of 256 threads per (b, h, key block); 16-byte coalesced loads,
// fp32 sums in a fixed order, divided by the block's valid-key count.
// ---------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) meankey_kernel(const __nv_bfloat16 *__restrict__ k,
                                                      float *__restrict__ kbar, int N, int N_pad,
                                                      int nkb)
{
    constexpr int VEC = D / 8;         // 16-byte vectors per row
    constexpr int GROUPS = 256 / VEC;  // row groups
    constexpr int RPT = 128 / GROUPS;  // rows per thread
    __shared__ __align__(16) float part[GROUPS][D];

    const int blk = blockIdx.x;
    const int bh = blk / nkb, j = blk % nkb;
    const int t0 = j * 128;
    const int nv = min(128, N - t0);
    const int tid = threadIdx.x, cv = tid % VEC, rg = tid / VEC;
    const uint4 *base = reinterpret_cast<const uint4 *>(k + ((size_t)bh * N_pad + t0) * D);

    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int it = 0; it < RPT; ++it) {
        const int r = rg + it * GROUPS;
        if (r < nv) {
            const uint4 v = __ldg(base + (size_t)r * VEC + cv);
            acc[0] += bf16_lo(v.x); acc[1] += bf16_hi(v.x);
            acc[2] += bf16_lo(v.y); acc[3] += bf16_hi(v.y);
            acc[4] += bf16_lo(v.z); acc[5] += bf16_hi(v.z);
            acc[6] += bf16_lo(v.w); acc[7] += bf16_hi(v.w);
        }
    }
    float4 *dst = reinterpret_cast<float4 *>(&part[rg][cv * 8]);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    __syncthreads();
    const float inv = 1.0f / (float)nv;
    for (int col = tid; col < D; col += 256) {
        float s = 0.f;
#pragma unroll 8
        for (int g = 0; g < GROUPS; ++g) s += part[g][col];
        kbar[(size_t)blk * D + col] = s * inv;
    }
}

// ---------------------------------------------------------------------------------
// Per-block k-means on the tensor cores (warp-level mma.sync m16n8k16, bf16 inputs,
// fp32 accumulation). One CTA of 128 threads (4 warps) per (b, h, query block); the
// block's queries stay in shared memory for all T iterations.
//   assign: q.c for every (query, centroid) as one small GEMM; each fp32 centroid is
//           split exactly into three bf16 terms (hi + mid + lo), so the products are
//           those of fp32 centroids with the bf16 queries, accumulated in fp32;
//           distance |c|^2 - 2 q.c (|q|^2 is common); argmin with ties to the lowest
//           cluster (compared as (distance, index) pairs across the 4 lanes that hold
//           a row's 8 centroids);
//   update: member sums as onehot[c][t] x Q[t][d] (exact 0/1 and bf16 operands, fp32
//           accumulation), divided by the member counts; an empty cluster keeps its
//           centroid.
// The GEMMs are 128 x 24 x d and 16 x d x 128: far below one tcgen05 tile, and each
// iteration needs the previous one's result, so warp-level MMAs in registers are used.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t &r0, uint32_t &r1)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int D>
struct KmSmem {
    static constexpr int kStride = D + 8;                      // bf16 row stride (ldmatrix conflict-free)
    static constexpr int kQ = 0;                               // Q     [128][kStride] bf16
    static constexpr int kCB = kQ + 128 * kStride * 2;         // splits [24][kStride] bf16
    static constexpr int kOH = kCB + 24 * kStride * 2;         // onehot [16][136] bf16
    static constexpr int kCS = kOH + 16 * 136 * 2;             // fp32 centroids [8][D]
    static constexpr int kBytes = kCS + 8 * D * 4;
};

template <int D>
__global__ void __launch_bounds__(128) kmeans_kernel(const __nv_bfloat16 *__restrict__ q, int N,
                                                     int N_pad, int nqb, int C, int T,
                                                     float *__restrict__ cent_out,
                                                     float *__restrict__ w_out,
                                                     uint8_t *__restrict__ assign_out)
{
    using L = KmSmem<D>;
    constexpr int CMAX = 8, S = L::kStride;
    extern __shared__ __align__(16) uint8_t km_smem[];
    __nv_bfloat16 *qs = reinterpret_cast<__nv_bfloat16 *>(km_smem + L::kQ);
    __nv_bfloat16 *cb = reinterpret_cast<__nv_bfloat16 *>(km_smem + L::kCB);
    __nv_bfloat16 *oh = reinterpret_cast<__nv_bfloat16 *>(km_smem + L::kOH);
    float *cs = reinterpret_cast<float *>(km_smem + L::kCS);
    __shared__ float cn[CMAX];
    __shared__ int wcount[4][CMAX];
    __shared__ int ccount[CMAX];
    __shared__ uint8_t lab[128];

    const int blk = blockIdx.x;
    const int bh = blk / nqb, qb = blk % nqb;
    const int t0 = qb * 128;
    const int nv = min(128, N - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = lane >> 2, tig = lane & 3;

    // Stage the block's queries (padding rows as zero) with 16-byte loads; clear the
    // one-hot matrix (its rows 8..15 stay zero).
    {
        constexpr int VEC = D / 8;
        const uint4 *src = reinterpret_cast<const uint4 *>(q + ((size_t)bh * N_pad + t0) * D);
        for (int v = tid; v < 128 * VEC; v += 128) {
            const int r = v / VEC, c8 = v % VEC;
            *reinterpret_cast<uint4 *>(qs + r * S + c8 * 8) =
                r < nv ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
        }
        for (int v = tid; v < 16 * 136 / 8; v += 128)
            reinterpret_cast<uint4 *>(oh)[v] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    for (int e = tid; e < CMAX * D; e += 128) {
        const int c = e / D, i = e % D;
        float v = 0.f;
        if (c < C) {
            const int src = nv >= C ? c * (nv / C) : min(c, nv - 1);
            v = __bfloat162float(qs[src * S + i]);
        }
        cs[c * D + i] = v;
    }
    __syncthreads();

    const uint32_t qs_a = smem_u32(qs), cb_a = smem_u32(cb), oh_a = smem_u32(oh);
    for (int it = 0; it < T; ++it) {
        // fp32 centroids -> exact three-term bf16 split; squared norms
        for (int e = tid; e < CMAX * D; e += 128) {
            const int c = e / D, i = e % D;
            const float x = cs[c * D + i];
            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
            const float r1 = x - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
            cb[c * S + i] = hi;
            cb[(8 + c) * S + i] = mid;
            cb[(16 + c) * S + i] = lo;
        }
        for (int c = warp; c < CMAX; c += 4) {
            float sq = 0.f;
            for (int i = lane; i < D; i += 32) sq = fmaf(cs[c * D + i], cs[c * D + i], sq);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
            if (lane == 0) cn[c] = sq;
        }
        __syncthreads();

        // assignment: warp w owns queries 32w..32w+31 (two 16-row tiles)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const int r_base = warp * 32 + mt * 16;
            float acc[3][4];
#pragma unroll
            for (int nt = 0; nt < 3; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(qs_a + ((r_base + (lane & 15)) * S + kk * 16 + (lane >> 4) * 8) * 2, a0, a1,
                        a2, a3);
#pragma unroll
                for (int nt = 0; nt < 3; ++nt) {
                    uint32_t b0, b1;
                    ldsm_x2(cb_a + ((nt * 8 + (lane & 7)) * S + kk * 16 + ((lane >> 3) & 1) * 8) * 2,
                            b0, b1);
                    mma_16816(acc[nt], a0, a1, a2, a3, b0, b1);
                }
            }
            // rows r_base+grp (acc[.][0..1]) and r_base+grp+8 (acc[.][2..3]);
            // columns (centroids) 2*tig and 2*tig+1
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float best = INFINITY;
                int arg = CMAX;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int c = 2 * tig + e;
                    const float dot = acc[0][2 * h + e] + acc[1][2 * h + e] + acc[2][2 * h + e];
                    const float dist = c < C ? fmaf(-2.f, dot, cn[c]) : INFINITY;
                    if (dist < best) {
                        best = dist;
                        arg = c;
                    }
                }
#pragma unroll
                for (int o = 1; o <= 2; o <<= 1) {
                    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
                    const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
                    if (ob < best || (ob == best && oa < arg)) {
                        best = ob;
                        arg = oa;
                    }
                }
                const int r = r_base + grp + 8 * h;
                if (tig == 0) lab[r] = r < nv ? (uint8_t)arg : (uint8_t)255;
            }
        }
        __syncthreads();

        // one-hot matrix [c][t] and member counts
        {
            const int a = lab[tid];
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
                oh[c * 136 + tid] = __float2bfloat16_rn(a == c ? 1.f : 0.f);
                const unsigned m = __ballot_sync(0xffffffffu, a == c);
                if (lane == 0) wcount[warp][c] = __popc(m);
            }
        }
        __syncthreads();
        if (tid < CMAX) ccount[tid] = wcount[0][tid] + wcount[1][tid] + wcount[2][tid] + wcount[3][tid];

        // update: sums[c][d] = onehot[c][.] x Q[.][d]; warp w owns columns w*D/4..
        constexpr int NT = D / 32;  // n-tiles of 8 columns per warp
        float sacc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(oh_a + ((lane & 15) * 136 + kk * 16 + (lane >> 4) * 8) * 2, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int n0 = warp * (D / 4) + nt * 8;
                uint32_t b0, b1;
                ldsm_x2_trans(qs_a + ((kk * 16 + (lane & 15)) * S + n0) * 2, b0, b1);
                mma_16816(sacc[nt], a0, a1, a2, a3, b0, b1);
            }
        }
        __syncthreads();  // ccount visible; all reads of cs done
        // rows 0..7 of the product are the clusters: this thread holds cluster grp,
        // columns n0 + 2*tig + {0, 1}
        {
            const int c = grp;
            const int n = ccount[c];
            if (c < C && n > 0) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int col = warp * (D / 4) + nt * 8 + 2 * tig;
                    cs[c * D + col] = sacc[nt][0] / (float)n;
                    cs[c * D + col + 1] = sacc[nt][1] / (float)n;
                }
            }
        }
        __syncthreads();
    }

    const size_t rowc = (size_t)blk * C;
    for (int e = tid; e < C * D; e += 128) cent_out[rowc * D + e] = cs[(e / D) * D + (e % D)];
    if (tid < C) w_out[rowc + tid] = (float)ccount[tid] / (float)nv;
    if (assign_out) assign_out[(size_t)bh * N_pad + t0 + tid] = lab[tid];
}

// ---------------------------------------------------------------------------------
// Block score: one CTA of 8 warps per (b, h, 8 query blocks); warp w owns query block
// qb0 + w and its C <= 8 centroids; lane l owns key-block columns 2l, 2l+1 of each
// 64-wide tile of mean keys. Pass 1 accumulates each centroid's softmax max and sum
// over all key blocks (online, merged across lanes); pass 2 recomputes the logits and
// writes s_j = sum_c (w_c / Z_c) exp(L_cj - m_c).
// ---------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) score_kernel(const float *__restrict__ cent,
                                                    const float *__restrict__ cw,
                                                    const float *__restrict__ kbar, int nqb,
                                                    int nkb, int C, float scale,
                                                    float *__restrict__ scores)
{
    constexpr int CMAX = 8, TJ = 64, BS = TJ + 2;
    extern __shared__ __align__(16) float smem_f[];
    float *As = smem_f;                 // [8 warps][D][CMAX]
    float *Bt = smem_f + 8 * D * CMAX;  // [D][BS]

    const int bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qb = blockIdx.x * 8 + warp;
    const bool row_ok = qb < nqb;

    // centroids of this warp's query block, transposed to [i][c]; absent ones are 0
    for (int e = lane; e < D * CMAX; e += 32) {
        const int i = e / CMAX, c = e % CMAX;
        float v = 0.f;
        if (row_ok && c < C) v = cent[(((size_t)bh * nqb + qb) * C + c) * D + i];
        As[(warp * D + i) * CMAX + c] = v;
    }
    float wc[CMAX];
#pragma unroll
    for (int c = 0; c < CMAX; ++c)
        wc[c] = (row_ok && c < C) ? cw[((size_t)bh * nqb + qb) * C + c] : 0.f;

    const float *kb = kbar + (size_t)bh * nkb * D;
    const int ntiles = (nkb + TJ - 1) / TJ;
    float m[CMAX], z[CMAX];
#pragma unroll
    for (int c = 0; c < CMAX; ++c) {
        m[c] = -INFINITY;
        z[c] = 0.f;
    }

    for (int pass = 0; pass < 2; ++pass) {
        float coef[CMAX];
        if (pass == 1) {
#pragma unroll
            for (int c = 0; c < CMAX; ++c) coef[c] = (c < C && z[c] > 0.f) ? wc[c] / z[c] : 0.f;
        }
        for (int tj = 0; tj < ntiles; ++tj) {
            const int j0 = tj * TJ;
            __syncthreads();
            for (int e = tid; e < TJ * D; e += 256) {
                const int jj = e / D, i = e % D;
                Bt[i * BS + jj] = (j0 + jj < nkb) ? kb[(size_t)(j0 + jj) * D + i] : 0.f;
            }
            __syncthreads();
            float L0[CMAX], L1[CMAX];
#pragma unroll
            for (int c = 0; c < CMAX; ++c) L0[c] = L1[c] = 0.f;
            const float *a = As + warp * D * CMAX;
#pragma unroll 4
            for (int i = 0; i < D; ++i) {
                const float4 a0 = *reinterpret_cast<const float4 *>(a + i * CMAX);
                const float4 a1 = *reinterpret_cast<const float4 *>(a + i * CMAX + 4);
                const float2 b = *reinterpret_cast<const float2 *>(Bt + i * BS + 2 * lane);
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                for (int c = 0; c < CMAX; ++c) {
                    L0[c] = fmaf(av[c], b.x, L0[c]);
                    L1[c] = fmaf(av[c], b.y, L1[c]);
                }
            }
            const int ja = j0 + 2 * lane, jb = ja + 1;
            if (pass == 0) {
#pragma unroll
                for (int c = 0; c < CMAX; ++c) {
                    const float x0 = L0[c] * scale, x1 = L1[c] * scale;
                    float mx = m[c];
                    if (ja < nkb) mx = fmaxf(mx, x0);
                    if (jb < nkb) mx = fmaxf(mx, x1);
                    float zz = (m[c] == -INFINITY) ? 0.f : z[c] * expf(m[c] - mx);
                    if (ja < nkb) zz += expf(x0 - mx);
                    if (jb < nkb) zz += expf(x1 - mx);
                    m[c] = mx;
                    z[c] = zz;
                }
            } else if (row_ok) {
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int c = 0; c < CMAX; ++c) {
                    if (c < C) {
                        s0 = fmaf(coef[c], expf(L0[c] * scale - m[c]), s0);
                        s1 = fmaf(coef[c], expf(L1[c] * scale - m[c]), s1);
                    }
                }
                float *dst = scores + ((size_t)bh * nqb + qb) * nkb;
                if (jb < nkb) {
                    if ((nkb & 1) == 0) {
                        *reinterpret_cast<float2 *>(dst + ja) = make_float2(s0, s1);
                    } else {
                        dst[ja] = s0;
                        dst[jb] = s1;
                    }
                } else if (ja < nkb) {
                    dst[ja] = s0;
                }
            }
        }
        if (pass == 0) {
            // merge (max, sum) across the 32 lanes of the warp
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float mo = __shfl_xor_sync(0xffffffffu, m[c], o);
                    const float zo = __shfl_xor_sync(0xffffffffu, z[c], o);
                    const float mx = fmaxf(m[c], mo);
                    float zz = 0.f;
                    if (m[c] != -INFINITY) zz += z[c] * expf(m[c] - mx);
                    if (mo != -INFINITY) zz += zo * expf(mo - mx);
                    m[c] = mx;
                    z[c] = zz;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------------
cudaError_t launch_meankey(const void *k, float *kbar, int BH, int N, int N_pad, int d,
                           cudaStream_t st)
{
    const int nkb = N_pad / 128;
    const dim3 grid((unsigned)(BH * nkb));
    if (d == 128)
        meankey_kernel<128><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)k, kbar, N, N_pad, nkb);
    else
        meankey_kernel<64><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)k, kbar, N, N_pad, nkb);
    return cudaGetLastError();
}

cudaError_t launch_kmeans(const void *q, float *cent, float *cw, uint8_t *assign, int BH, int N,
                          int N_pad, int d, int C, int T, cudaStream_t st)
{
    const int nqb = N_pad / 128;
    const dim3 grid((unsigned)(BH * nqb));
    if (d == 128) {
        const int smem = KmSmem<128>::kBytes;
        cudaError_t e = cudaFuncSetAttribute(kmeans_kernel<128>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kmeans_kernel<128><<<grid, 128, smem, st>>>((const __nv_bfloat16 *)q, N, N_pad, nqb, C, T,
                                                    cent, cw, assign);
    } else {
        const int smem = KmSmem<64>::kBytes;
        cudaError_t e = cudaFuncSetAttribute(kmeans_kernel<64>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kmeans_kernel<64><<<grid, 128, smem, st>>>((const __nv_bfloat16 *)q, N, N_pad, nqb, C, T,
                                                   cent, cw, assign);
    }
    return cudaGetLastError();
}

cudaError_t launch_score(const float *cent, const float *cw, const float *kbar, float *scores,
                         int BH, int nqb, int nkb, int d, int C, cudaStream_t st)
{
    const dim3 grid((unsigned)((nqb + 7) / 8), (unsigned)BH);
    const float scale = (float)(1.0 / sqrt((double)d));
    const size_t smem = sizeof(float) * (8 * d * 8 + d * 66);
    if (d == 128) {
        cudaError_t e = cudaFuncSetAttribute(score_kernel<128>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        score_kernel<128><<<grid, 256, smem, st>>>(cent, cw, kbar, nqb, nkb, C, scale, scores);
    } else {
        cudaError_t e = cudaFuncSetAttribute(score_kernel<64>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        score_kernel<64><<<grid, 256, smem, st>>>(cent, cw, kbar, nqb, nkb, C, scale, scores);
    }
    return cudaGetLastError();
}

}  // namespace ab
