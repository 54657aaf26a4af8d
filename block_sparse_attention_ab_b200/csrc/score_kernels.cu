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
// Per-block k-means: one CTA of 128 threads per (b, h, query block), thread t owns
// query t (kept in fp32 registers); centroids live in shared memory.
//   assign: argmin_c |c|^2 - 2 q.c (the |q|^2 term is common), strict < so ties go
//           to the lowest cluster;
//   update: members gathered per cluster in index order (warp ballots), summed in
//           that order by one thread per dimension; an empty cluster keeps its centroid.
// ---------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) kmeans_kernel(const __nv_bfloat16 *__restrict__ q, int N,
                                                     int N_pad, int nqb, int C, int T,
                                                     float *__restrict__ cent_out,
                                                     float *__restrict__ w_out,
                                                     uint8_t *__restrict__ assign_out)
{
    constexpr int CMAX = 8;
    __shared__ __align__(16) __nv_bfloat16 qs[128][D];
    __shared__ __align__(16) float cs[CMAX][D];
    __shared__ float cn[CMAX];
    __shared__ int wcount[4][CMAX];
    __shared__ int cstart[CMAX + 1];
    __shared__ int ccount[CMAX];
    __shared__ uint8_t order[128];
    __shared__ uint8_t lab[128];

    const int blk = blockIdx.x;
    const int bh = blk / nqb, qb = blk % nqb;
    const int t0 = qb * 128;
    const int nv = min(128, N - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // Stage the block's queries (padding rows as zero) with 16-byte loads.
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(q + ((size_t)bh * N_pad + t0) * D);
        uint4 *dst = reinterpret_cast<uint4 *>(&qs[0][0]);
        constexpr int VEC = D / 8;
        for (int v = tid; v < 128 * VEC; v += 128) {
            const int r = v / VEC;
            dst[v] = r < nv ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();

    float qr[D];
#pragma unroll
    for (int i = 0; i < D; i += 2) {
        const uint32_t x = *reinterpret_cast<const uint32_t *>(&qs[tid][i]);
        qr[i] = bf16_lo(x);
        qr[i + 1] = bf16_hi(x);
    }
    for (int e = tid; e < C * D; e += 128) {
        const int c = e / D, i = e % D;
        const int src = nv >= C ? c * (nv / C) : min(c, nv - 1);
        cs[c][i] = __bfloat162float(qs[src][i]);
    }
    __syncthreads();

    for (int it = 0; it < T; ++it) {
        // squared norms of the centroids
        for (int c = warp; c < C; c += 4) {
            float s = 0.f;
            for (int i = lane; i < D; i += 32) s = fmaf(cs[c][i], cs[c][i], s);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) cn[c] = s;
        }
        __syncthreads();
        // assignment
        int a = CMAX;  // padding rows belong to no cluster
        if (tid < nv) {
            float best = 0.f;
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
                if (c < C) {
                    const float4 *cv = reinterpret_cast<const float4 *>(&cs[c][0]);
                    float dot = 0.f;
#pragma unroll
                    for (int i4 = 0; i4 < D / 4; ++i4) {
                        const float4 cc = cv[i4];
                        dot = fmaf(qr[4 * i4 + 0], cc.x, dot);
                        dot = fmaf(qr[4 * i4 + 1], cc.y, dot);
                        dot = fmaf(qr[4 * i4 + 2], cc.z, dot);
                        dot = fmaf(qr[4 * i4 + 3], cc.w, dot);
                    }
                    const float dist = fmaf(-2.f, dot, cn[c]);
                    if (c == 0 || dist < best) {
                        best = dist;
                        a = c;
                    }
                }
            }
        }
        lab[tid] = (uint8_t)a;
        // stable counting sort of the members by cluster (warp ballots)
        int rank = 0;
#pragma unroll
        for (int c = 0; c < CMAX; ++c) {
            const unsigned m = __ballot_sync(0xffffffffu, a == c);
            if (a == c) rank = __popc(m & ((1u << lane) - 1u));
            if (lane == 0) wcount[warp][c] = __popc(m);
        }
        __syncthreads();
        if (tid == 0) {
            int s = 0;
            for (int c = 0; c < CMAX; ++c) {
                cstart[c] = s;
                int n = 0;
                for (int w = 0; w < 4; ++w) n += wcount[w][c];
                ccount[c] = n;
                s += n;
            }
            cstart[CMAX] = s;
        }
        __syncthreads();
        if (a < CMAX) {
            int pos = cstart[a] + rank;
            for (int w = 0; w < warp; ++w) pos += wcount[w][a];
            order[pos] = (uint8_t)tid;
        }
        __syncthreads();
        // update: thread i sums dimension i of each cluster's members in index order
        for (int i = tid; i < D; i += 128) {
            for (int c = 0; c < C; ++c) {
                const int n = ccount[c];
                if (n == 0) continue;
                float s = 0.f;
                const int st = cstart[c];
                for (int m = 0; m < n; ++m) s += __bfloat162float(qs[order[st + m]][i]);
                cs[c][i] = s / (float)n;
            }
        }
        __syncthreads();
    }

    const size_t rowc = (size_t)blk * C;
    for (int e = tid; e < C * D; e += 128) cent_out[rowc * D + e] = cs[e / D][e % D];
    if (tid < C) w_out[rowc + tid] = (float)ccount[tid] / (float)nv;
    if (assign_out) assign_out[(size_t)bh * N_pad + t0 + tid] = tid < nv ? lab[tid] : (uint8_t)255;
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
    if (d == 128)
        kmeans_kernel<128><<<grid, 128, 0, st>>>((const __nv_bfloat16 *)q, N, N_pad, nqb, C, T,
                                                 cent, cw, assign);
    else
        kmeans_kernel<64><<<grid, 128, 0, st>>>((const __nv_bfloat16 *)q, N, N_pad, nqb, C, T,
                                                cent, cw, assign);
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
