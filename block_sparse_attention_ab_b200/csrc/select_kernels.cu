// select_kernels.cu -- key-block selection per query block on sm_100a.
//
// SIP (AB-Attention news page, section «Три приёма AB-Attention», second technique):
// inclusion probability p_j = min(1, c s_j) with sum p_j = K, the top blocks always
// kept, each kept block weighted by 1/p_j. Solved exactly in integers on the fixed
// point u_j = floor(s_j 2^50) so every implementation reproduces the same bits (a row
// whose exact sum U = sum u_j needs more than 64 bits is rejected as invalid); draws
// from Philox4x32-10 (Salmon et al., SC'11) keyed by the seed, counter (j, qb, h, b).
// Top-k (section «Где ломаются прежние разреженные схемы»): the K largest scores, ties
// to the lower index, found by an MSB-first radix select on the score bits.
// One CTA of 256 threads per (b, h, qb) row (rows of up to 65536 entries: key blocks or
// 4-token key units); kept entries are compacted in ascending order: each warp owns a
// contiguous slab of the row and uses ballots, and one block-wide prefix over the eight
// warps' counts places the slabs.
#include <cstdint>
#include <cuda_runtime.h>

#include "ab_device.cuh"
#include "ab_kernels.h"

namespace ab {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

// Philox4x32-10: ten rounds of the 4x32 S-box, key bumped by the Weyl constants
// 0x9E3779B9 / 0xBB67AE85 between rounds, round multipliers 0xD2511F53 / 0xCD9E8D57.
__device__ __forceinline__ uint4 philox_4x32_10(uint4 c, uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

__device__ __forceinline__ bool score_ok(float v) { return v >= 0.f && v <= 2.f; }

// exact: v in [0, 2] -> floor(v * 2^50) < 2^52 (the product is exact in double)
__device__ __forceinline__ uint64_t fixed50(float v)
{
    return __double2ull_rz((double)v * 1125899906842624.0);
}

// k * u >= R with a 128-bit product
__device__ __forceinline__ bool mul_ge(uint64_t k, uint64_t u, uint64_t R)
{
    return __umul64hi(k, u) != 0ull || k * u >= R;
}

// The least u with k u >= R (k >= 1), so that the test k u_j >= R of a pass becomes
// u_j >= thr: a double quotient (within a few units of the exact one: R / k < 2^64
// carries a relative error near 2^-52) corrected by the exact 128-bit test. k = 0: 0
// when R = 0, else no u qualifies.
__device__ __forceinline__ uint64_t ceil_div_threshold(uint64_t R, uint64_t k)
{
    if (k == 0) return R == 0 ? 0ull : ~0ull;
    const double qd = __ull2double_rn(R) / __ull2double_rn(k);
    uint64_t q = qd >= 18446744073709549568.0 ? ~0ull : __double2ull_rz(qd);
    while (q > 0 && mul_ge(k, q - 1, R)) --q;
    while (!mul_ge(k, q, R)) ++q;
    return q;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Block-wide sums of (a, b, c); every thread gets the totals.
struct Sum3 {
    unsigned long long a, b, c;
};

__device__ Sum3 block_sum3(unsigned long long a, unsigned long long b, unsigned long long c,
                           unsigned long long (*red)[3])
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    a = warp_sum(a);
    b = warp_sum(b);
    c = warp_sum(c);
    __syncthreads();
    if (lane == 0) {
        red[warp][0] = a;
        red[warp][1] = b;
        red[warp][2] = c;
    }
    __syncthreads();
    Sum3 s{0, 0, 0};
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
        s.a += red[w][0];
        s.b += red[w][1];
        s.c += red[w][2];
    }
    return s;
}

// kCacheU: the row's u_j stay in shared memory after pass 0 (rows of up to
// kSipCacheMax entries); otherwise each pass recomputes them from the scores.
constexpr int kSipCacheMax = 8192;

template <bool kCacheU>
__global__ void __launch_bounds__(kSelThreads) sip_kernel(const float *__restrict__ scores,
                                                         int H, int bh0, int nqb, int nkb, int K,
                                                         uint32_t key0, uint32_t key1,
                                                         int32_t *__restrict__ idx,
                                                         int32_t *__restrict__ cnt,
                                                         float *__restrict__ w,
                                                         double *__restrict__ p_out, int *flag)
{
    // kCacheU: u_j as uint64 [nkb]; then nkb bytes (0 = out, 1 = saturated, 2 = joining),
    // then the keep bits of the draws
    extern __shared__ __align__(16) uint8_t sip_sh[];
    uint64_t *u_sh = reinterpret_cast<uint64_t *>(sip_sh);
    uint8_t *inS = sip_sh + (kCacheU ? (size_t)nkb * 8 : 0);
    __shared__ unsigned long long red[kSelWarps][3];
    __shared__ int wtot[kSelWarps];

    // row of this call; its (b, h) counts from the call's first head pair bh0 (a call on
    // a range of head pairs draws the same numbers as one on the whole tensor)
    const size_t row = blockIdx.x;
    const int bh = bh0 + (int)(row / nqb);
    const int b = bh / H, h = bh % H;
    const int qb = (int)(row % nqb);
    const float *s = scores + row * nkb;
    const int tid = threadIdx.x;
    auto u_of = [&](int j) -> uint64_t { return kCacheU ? u_sh[j] : fixed50(s[j]); };

    // pass 0: validate, U = sum u_j, number of positive u_j. U is summed exactly as
    // U_hi = sum (u_j >> 12) and U_lo = sum (u_j & 0xfff) (neither can overflow), and a row
    // whose U needs more than 64 bits is rejected like a bad score.
    unsigned long long u_hi = 0, u_lo = 0, counts = 0;  // counts: positive | bad << 32
    for (int j = tid; j < nkb; j += kSelThreads) {
        const float v = s[j];
        inS[j] = 0;
        if (!score_ok(v)) {
            counts += 1ull << 32;
            continue;
        }
        const uint64_t u = fixed50(v);
        if (kCacheU) u_sh[j] = u;
        u_hi += u >> 12;
        u_lo += u & 0xfffull;
        counts += u > 0;
    }
    Sum3 t = block_sum3(u_hi, u_lo, counts, red);
    const unsigned long long top = t.a + (t.b >> 12);  // U = top * 2^12 + (U_lo mod 2^12)
    unsigned long long U = (top << 12) | (t.b & 0xfffull);
    unsigned long long npos = t.c & 0xffffffffull;
    if ((t.c >> 32) != 0 || top >= (1ull << 52)) {
        for (int j = tid; j < nkb; j += kSelThreads) {
            idx[row * nkb + j] = -1;
            w[row * nkb + j] = 0.f;
            if (p_out) p_out[row * nkb + j] = 0.0;
        }
        if (tid == 0) {
            cnt[row] = 0;
            raise_flag(flag, AB_FLAG_BAD_SCORE);
        }
        return;
    }

    // saturated set S by the fixed point S <- S + {j : (K-|S|) u_j >= U - sum_S u}
    const bool all_positive_kept = npos <= (unsigned long long)K;
    uint64_t k_rest = 0, R = 0;
    if (all_positive_kept) {
        for (int j = tid; j < nkb; j += kSelThreads) inS[j] = u_of(j) > 0 ? 1 : 0;
        __syncthreads();
    } else {
        unsigned long long sizeS = 0, sumS = 0;
        for (;;) {
            k_rest = (uint64_t)K - sizeS;
            R = U - sumS;
            // (K - |S|) u_j >= R  <=>  u_j >= ceil(R / (K - |S|))
            const uint64_t thr = ceil_div_threshold(R, k_rest);
            unsigned long long add_n = 0, add_u = 0;
            for (int j = tid; j < nkb; j += kSelThreads) {
                if (inS[j]) continue;
                const uint64_t u = u_of(j);
                if (u >= thr) {
                    inS[j] = 2;
                    ++add_n;
                    add_u += u;
                }
            }
            t = block_sum3(add_n, add_u, 0, red);
            if (t.a == 0) break;
            sizeS += t.a;
            sumS += t.b;
            for (int j = tid; j < nkb; j += kSelThreads)
                if (inS[j] == 2) inS[j] = 1;
            __syncthreads();
        }
    }

    // probabilities and draws, then ordered compaction. Warp w owns the contiguous slab
    // [w L, (w + 1) L) of the row (L a multiple of 32): it draws its entries 32 at a time,
    // keeps the keep-bits of each 32-entry chunk in shared memory and counts its kept
    // entries; one block barrier gives each warp its output offset (the kept entries of
    // the slabs before it), and a second walk over the slab writes the kept indices and
    // weights in ascending order. Two block barriers per row instead of two per 256
    // entries.
    const double Rd = __ull2double_rn(R);
    const int lane = tid & 31, warp = tid >> 5;
    const int slab = (((nkb + kSelWarps - 1) / kSelWarps) + 31) & ~31;
    const int j_begin = min(nkb, warp * slab), j_end = min(nkb, j_begin + slab);
    uint32_t *keep_bits = reinterpret_cast<uint32_t *>(inS + ((nkb + 15) & ~15));  // [nkb / 32]
    auto prob = [&](int j) -> double {  // p_j of entry j
        if (inS[j] == 1) return 1.0;
        if (all_positive_kept) return 0.0;
        const uint64_t u = u_of(j);
        return u > 0 ? __ull2double_rn(k_rest * u) / Rd : 0.0;
    };
    int kept_here = 0;
    for (int j0 = j_begin; j0 < j_end; j0 += 32) {
        const int j = j0 + lane;
        bool keep = false;
        if (j < j_end) {
            const double pj = prob(j);
            if (p_out) p_out[row * nkb + j] = pj;
            const uint4 x = philox_4x32_10(make_uint4((uint32_t)j, (uint32_t)qb, (uint32_t)h,
                                                      (uint32_t)b),
                                           key0, key1);
            const uint64_t r53 = ((((uint64_t)x.x) << 32) | x.y) >> 11;
            keep = __ull2double_rn(r53) < pj * 9007199254740992.0;
        }
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) keep_bits[j0 >> 5] = m;
        kept_here += __popc(m);
    }
    if (lane == 0) wtot[warp] = kept_here;
    __syncthreads();
    int base = 0, total = 0;
#pragma unroll
    for (int v = 0; v < kSelWarps; ++v) {
        const int t = wtot[v];
        base += v < warp ? t : 0;
        total += t;
    }
    __syncwarp();
    for (int j0 = j_begin; j0 < j_end; j0 += 32) {
        const unsigned m = keep_bits[j0 >> 5];
        const int j = j0 + lane;
        if ((m >> lane) & 1u) {
            const int pos = base + __popc(m & ((1u << lane) - 1u));
            idx[row * nkb + pos] = j;
            w[row * nkb + pos] = __double2float_rn(1.0 / prob(j));
        }
        base += __popc(m);
    }
    for (int c = total + tid; c < nkb; c += kSelThreads) {
        idx[row * nkb + c] = -1;
        w[row * nkb + c] = 0.f;
    }
    if (tid == 0) cnt[row] = total;
}

// Score bit patterns (order-preserving for s >= 0, -0 taken as +0): staged in shared
// memory (kSmemKeys) or, for rows too long for it, read from the scores in global memory.
template <bool kSmemKeys>
struct TopkKeys {
    uint32_t *sh;
    const float *s;
    __device__ __forceinline__ uint32_t operator[](int j) const
    {
        return kSmemKeys ? sh[j] : __float_as_uint(__ldg(s + j) + 0.0f);
    }
};

template <bool kSmemKeys>
__global__ void __launch_bounds__(kSelThreads) topk_kernel(const float *__restrict__ scores,
                                                          int nkb, int K,
                                                          int32_t *__restrict__ idx,
                                                          int32_t *__restrict__ cnt,
                                                          float *__restrict__ w, int *flag)
{
    extern __shared__ uint32_t keys_sh[];  // kSmemKeys: nkb score bit patterns; then keep bits
    __shared__ unsigned long long red[kSelWarps][3];
    __shared__ int hist[256];
    __shared__ int wtot[kSelWarps];
    __shared__ uint32_t sel_digit;
    __shared__ int sel_rem;

    const size_t row = blockIdx.x;
    const float *s = scores + row * nkb;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const TopkKeys<kSmemKeys> keys{keys_sh, s};
    unsigned long long nbad = 0;
    for (int j = tid; j < nkb; j += kSelThreads) {
        const float v = s[j];
        if (!score_ok(v)) ++nbad;
        if (kSmemKeys) keys_sh[j] = __float_as_uint(v + 0.0f);  // -0 -> +0
    }
    const Sum3 t = block_sum3(nbad, 0, 0, red);
    if (t.a != 0) {
        for (int j = tid; j < nkb; j += kSelThreads) {
            idx[row * nkb + j] = -1;
            if (w) w[row * nkb + j] = 0.f;
        }
        if (tid == 0) {
            cnt[row] = 0;
            raise_flag(flag, AB_FLAG_BAD_SCORE);
        }
        return;
    }

    // K-th largest key by MSB-first radix select, 8-bit digits
    uint32_t prefix = 0, mask = 0;
    int rem = K;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int e = tid; e < 256; e += kSelThreads) hist[e] = 0;
        __syncthreads();
        for (int j = tid; j < nkb; j += kSelThreads) {
            const uint32_t key = keys[j];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns digits 255-8l .. 248-8l (descending)
            int local = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) local += hist[255 - 8 * lane - e];
            int incl = local;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const int excl = incl - local;
            if (excl < rem && incl >= rem) {
                int acc = excl;
                for (int e = 0; e < 8; ++e) {
                    const int dgt = 255 - 8 * lane - e;
                    if (acc + hist[dgt] >= rem) {
                        sel_digit = (uint32_t)dgt;
                        sel_rem = rem - acc;
                        break;
                    }
                    acc += hist[dgt];
                }
            }
        }
        __syncthreads();
        prefix |= sel_digit << shift;
        mask |= 255u << shift;
        rem = sel_rem;
        __syncthreads();
    }
    // keep key > T, plus the first `rem` keys equal to T in index order. Warp w owns the
    // slab [w L, (w + 1) L) (L a multiple of 32): it counts its keys equal to T; a block
    // barrier gives each warp the number of equal keys before its slab; it decides its
    // keeps (keep-bits per 32-entry chunk in shared memory) and counts them; a second
    // barrier gives its output offset; a last walk writes the kept indices in order.
    const uint32_t T = prefix;
    const int slab = (((nkb + kSelWarps - 1) / kSelWarps) + 31) & ~31;
    const int j_begin = min(nkb, warp * slab), j_end = min(nkb, j_begin + slab);
    uint32_t *keep_bits = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(keys_sh) +
                                                       (kSmemKeys ? (size_t)nkb * 4 : 0));
    const unsigned lt = (1u << lane) - 1u;
    int eq_here = 0;
    for (int j0 = j_begin; j0 < j_end; j0 += 32) {
        const int j = j0 + lane;
        eq_here += __popc(__ballot_sync(0xffffffffu, j < j_end && keys[j] == T));
    }
    if (lane == 0) wtot[warp] = eq_here;
    __syncthreads();
    int eq_run = 0;
#pragma unroll
    for (int v = 0; v < kSelWarps; ++v) eq_run += v < warp ? wtot[v] : 0;
    __syncthreads();
    int kept_here = 0;
    for (int j0 = j_begin; j0 < j_end; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t key = j < j_end ? keys[j] : 0u;
        const bool eq = j < j_end && key == T;
        const unsigned meq = __ballot_sync(0xffffffffu, eq);
        const bool keep = j < j_end && (key > T || (eq && eq_run + __popc(meq & lt) < rem));
        const unsigned mk = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) keep_bits[j0 >> 5] = mk;
        kept_here += __popc(mk);
        eq_run += __popc(meq);
    }
    if (lane == 0) wtot[warp] = kept_here;
    __syncthreads();
    int base = 0, total = 0;
#pragma unroll
    for (int v = 0; v < kSelWarps; ++v) {
        const int t = wtot[v];
        base += v < warp ? t : 0;
        total += t;
    }
    for (int j0 = j_begin; j0 < j_end; j0 += 32) {
        const unsigned m = keep_bits[j0 >> 5];
        if ((m >> lane) & 1u) {
            const int pos = base + __popc(m & lt);
            idx[row * nkb + pos] = j0 + lane;
            if (w) w[row * nkb + pos] = 1.0f;
        }
        base += __popc(m);
    }
    for (int c = total + tid; c < nkb; c += kSelThreads) {
        idx[row * nkb + c] = -1;
        if (w) w[row * nkb + c] = 0.f;
    }
    if (tid == 0) cnt[row] = total;
}

// Rows of more than 48 KB of per-row shared memory need the opt-in limit.
constexpr size_t kTopkSmemKeysMax = 160 * 1024;

template <typename Kern>
static cudaError_t allow_smem(Kern kern, size_t bytes)
{
    if (bytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t launch_sip(const float *scores, int n_bh, int H, int bh0, int nqb, int nkb, int K,
                       uint64_t seed, int32_t *idx, int32_t *cnt, float *w, double *p, int *flag,
                       cudaStream_t st)
{
    const unsigned rows = (unsigned)((size_t)n_bh * nqb);
    const size_t flags = (size_t)((nkb + 15) & ~15) + (size_t)(nkb + 255) / 256 * 32 + 32;
    const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
    cudaError_t e;
    if (nkb <= kSipCacheMax) {
        const size_t smem = (size_t)nkb * 8 + flags;
        e = allow_smem(sip_kernel<true>, smem);
        if (e != cudaSuccess) return e;
        sip_kernel<true><<<rows, kSelThreads, smem, st>>>(scores, H, bh0, nqb, nkb, K, k0, k1, idx,
                                                          cnt, w, p, flag);
    } else {
        e = allow_smem(sip_kernel<false>, flags);
        if (e != cudaSuccess) return e;
        sip_kernel<false><<<rows, kSelThreads, flags, st>>>(scores, H, bh0, nqb, nkb, K, k0, k1, idx,
                                                            cnt, w, p, flag);
    }
    return cudaGetLastError();
}

cudaError_t launch_topk(const float *scores, int B, int H, int nqb, int nkb, int K, int32_t *idx,
                        int32_t *cnt, float *w, int *flag, cudaStream_t st)
{
    const unsigned rows = (unsigned)((size_t)B * H * nqb);
    const size_t bits = (size_t)(nkb + 255) / 256 * 32 + 32;  // keep bits of the compaction
    const size_t smem = (size_t)nkb * sizeof(uint32_t);
    if (smem <= kTopkSmemKeysMax) {
        cudaError_t e = allow_smem(topk_kernel<true>, smem + bits);
        if (e != cudaSuccess) return e;
        topk_kernel<true><<<rows, kSelThreads, smem + bits, st>>>(scores, nkb, K, idx, cnt, w, flag);
    } else {
        topk_kernel<false><<<rows, kSelThreads, bits, st>>>(scores, nkb, K, idx, cnt, w, flag);
    }
    return cudaGetLastError();
}

}  // namespace ab
