// ab_kernels.h -- internal launchers of the sm_100a kernels (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace ab {

// IBCS scoring (score_kernels.cu)
cudaError_t launch_meankey(const void *k, float *kbar, int BH, int N, int N_pad, int d,
                           cudaStream_t st);
cudaError_t launch_kmeans(const void *q, float *cent, float *cw, uint8_t *assign, int BH, int N,
                          int N_pad, int d, int C, int T, cudaStream_t st);
cudaError_t launch_score(const float *cent, const float *cw, const float *kbar, float *scores,
                         int BH, int nqb, int nkb, int d, int C, cudaStream_t st);

// SIP / top-k selection (select_kernels.cu)
cudaError_t launch_sip(const float *scores, int B, int H, int nqb, int nkb, int K, uint64_t seed,
                       int32_t *idx, int32_t *cnt, float *w, double *p, int *flag,
                       cudaStream_t st);
cudaError_t launch_topk(const float *scores, int B, int H, int nqb, int nkb, int K, int32_t *idx,
                        int32_t *cnt, float *w, int *flag, cudaStream_t st);

// Block-sparse attention (attn_kernel.cu)
struct AttnLaunch {
    const void *q, *k, *v;
    const int32_t *idx, *cnt;
    const float *w;  // nullptr = unweighted (top-k)
    void *out;
    bool out_f32;  // output fp32 instead of bf16
    float *lse;
    int *flag;
    int B, H, N, N_pad, d;
    int grid_override;  // > 0: number of CTAs (tests); 0: one per SM
};
cudaError_t launch_attn(const AttnLaunch &a, cudaStream_t st);

}  // namespace ab
