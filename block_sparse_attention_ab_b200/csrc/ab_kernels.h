// ab_kernels.h -- internal launchers of the sm_100a kernels (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/ab_attn.h"

namespace ab {

// AB_OK, or AB_ERR_CUDA with the error kept for ab_last_cuda_error (ab_api.cu).
ab_status status_of(cudaError_t e);

// IBCS scoring (score_kernels.cu)
// Device scratch of the scoring pass, each region 256-byte aligned: mean keys fp32
// [BH][n_ku][d], centroids fp32 [BH][n_qb][C][d], cluster weights fp32 [BH][n_qb][C],
// the two fp16 terms of the scaled mean keys [2][BH][n_ku][d], and each mean key's
// unscale factor fp32 [BH][n_ku_pad] (n_ku_pad = n_ku rounded up to 256); n_ku = key
// units per head (n_qb for 128-token key blocks).
struct ScoreLayout {
    size_t kbar, cent, cw, kbar_terms, kscale, total;
};

inline size_t kscale_stride(size_t nku) { return (nku + 255) / 256 * 256; }

inline ScoreLayout score_layout(size_t BH, size_t nqb, size_t nku, size_t d, size_t C)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    ScoreLayout L;
    L.kbar = 0;
    L.cent = up(L.kbar + BH * nku * d * sizeof(float));
    L.cw = up(L.cent + BH * nqb * C * d * sizeof(float));
    L.kbar_terms = up(L.cw + BH * nqb * C * sizeof(float));
    L.kscale = up(L.kbar_terms + 2 * BH * nku * d * 2);
    L.total = up(L.kscale + BH * kscale_stride(nku) * sizeof(float));
    return L;
}

cudaError_t launch_meankey(const void *k, float *kbar, void *kbar_terms, float *kscale, int BH,
                           int N, int N_pad, int d, cudaStream_t st);
cudaError_t launch_meankey_units(const void *k, float *kbar, void *kbar_terms, float *kscale,
                                 int BH, int N, int N_pad, int d, int unit, cudaStream_t st);
cudaError_t launch_kmeans(const void *q, float *cent, float *cw, uint8_t *assign, int BH, int N,
                          int N_pad, int d, int C, int T, int *flag, cudaStream_t st);
cudaError_t launch_score(const float *cent, const float *cw, const void *kbar_terms,
                         const float *kscale, float *scores, int BH, int nqb, int nkb,
                         int nkb_valid, int d, int C, int *flag, cudaStream_t st);

// SIP / top-k selection (select_kernels.cu)
// SIP over n_bh head pairs starting at global pair bh0 (b = pair / H, h = pair % H key
// the random numbers)
cudaError_t launch_sip(const float *scores, int n_bh, int H, int bh0, int nqb, int nkb, int K,
                       uint64_t seed, int32_t *idx, int32_t *cnt, float *w, double *p, int *flag,
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
    int unit;           // key unit of idx entries: 128 (key blocks) or 4 (gathered 4-token units)
    int grid_override;  // > 0: number of CTAs (tests); 0: one per SM
    unsigned long long wait_ns;  // > 0: limit of the kernel's bounded waits (tests); 0: 2 s
};
cudaError_t launch_attn(const AttnLaunch &a, cudaStream_t st);
// Tests: the next attention launch uses claim slot `slot` (0..4095) instead of the next
// slot in turn.
void force_next_counter_slot(int slot);

}  // namespace ab
