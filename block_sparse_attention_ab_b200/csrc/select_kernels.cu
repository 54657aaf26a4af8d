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
// SIP runs one warp per (b, h, qb) row and top-k one CTA of 256 threads per row (rows of
// up to 65536 entries: key blocks or 4-token key units); kept entries are compacted in
// ascending order with warp ballots (top-k: each warp owns a contiguous slab of the row,
// and one block-wide prefix over the eight warps' counts places the slabs).
#include <cstdint>
#include <cuda_runtime.h>

#include "ab_device.cuh"
#include "ab_kernels.h"

namespace ab {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

// Philox4x32-10: ten rounds of the 4x32 S-box with round multipliers 0xD2511F53 /
// 0xCD9E8D57 (each a 32 x 32 -> 64-bit product); round r uses the key bumped r times by
// the Weyl constants 0x9E3779B9 / 0xBB67AE85, precomputed per thread in rk0 / rk1.
__device__ __forceinline__ uint4 philox_4x32_10(uint4 c, const uint32_t (&rk0)[10],
                                                const uint32_t (&rk1)[10])
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c.x;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c.z;
        c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ rk0[r], (uint32_t)p1,
                       (uint32_t)(p0 >> 32) ^ c.w ^ rk1[r], (uint32_t)p0);
    }
    return c;
}

__device__ __forceinline__ bool score_ok(float v) { return v >= 0.f && v <= 2.f; }

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

// u = floor(v 2^50) from the bit pattern b of a score v in [0, 2] (+0 for zero): the
// significand shifted by the exponent, exactly the truncated product (v 2^50 is exact).
// Monotone in b, so a threshold on u is a threshold on the bit pattern.
__device__ __forceinline__ uint64_t fixed50_bits(uint32_t b)
{
    const uint32_t E = b >> 23;
    const uint64_t m = E ? (uint64_t)((b & 0x7FFFFFu) | 0x800000u) : (uint64_t)(b & 0x7FFFFFu);
    const int sh = (E ? (int)E : 1) - 100;  // exponent - 23 + 50
    return sh >= 0 ? m << sh : (sh > -25 ? m >> -sh : 0ull);
}

// Canonical bit pattern of a valid score (-0 becomes +0)
__device__ __forceinline__ uint32_t score_bits(float v) { return __float_as_uint(v + 0.0f); }

constexpr uint32_t kBitsTwo = 0x40000000u;  // 2.0f: u(2) = 2^51, the largest u

// The least bit pattern b (of a score in [0, 2]) with fixed50_bits(b) >= thr, or
// 0xFFFFFFFF when no score reaches thr. thr >= 1. The float nearest above thr 2^-50 is the
// candidate; the exact test moves it by the few steps the double rounding can leave.
__device__ __forceinline__ uint32_t bits_threshold(uint64_t thr)
{
    if (thr > (1ull << 51)) return 0xFFFFFFFFu;
    uint32_t b = __float_as_uint(__double2float_ru(__ull2double_rn(thr) * 0x1p-50));
    b = min(b, kBitsTwo);
    while (b > 0 && fixed50_bits(b - 1) >= thr) --b;
    while (fixed50_bits(b) < thr) ++b;
    return b;
}

// One warp per row, eight rows per CTA: the row's sums are warp shuffles and its
// compaction runs in the same ascending walk as its draws, so nothing waits on a block
// barrier. Rows of up to kSipCacheMax entries keep their score bit patterns in the warp's
// slice of shared memory after pass 0; longer rows re-read the scores (L2) in each pass.
// Every walk loads four 32-entry chunks ahead of their use.
constexpr int kSipCacheMax = 2048;
constexpr int kSipUnroll = 4;

// SIP per row. The saturated set S of the fixed point S <- S + {j : (K-|S|) u_j >= R_S}
// (R_S = U - sum_S u) is always {j : u_j >= theta} for the last threshold theta =
// ceil(R_S / (K-|S|)) of the iteration: a pass either lowers theta, adding the entries
// between the new and the old threshold, or adds nothing and ends. So S is held as one
// bit-pattern threshold, and every pass is a compare on the bit patterns.
// Draws: keep j iff R53_j < p_j 2^53 with p_j = fl64(fl64((K-|S|) u_j) / fl64(R_S)) and
// R53_j the top 53 bits of Philox(j, qb, h, b). The test is first taken in fp32 on
// a = top 32 bits of the draw as a fraction (within 2^-23 below R53 2^-53) and
// p' = u_j c (c = fl32((K-|S|) / R_S), within 2^-22 of p_j relative): a' < p'(1 - 2^-19)
// - 2^-22 proves keep, a' >= p'(1 + 2^-19) proves drop (margins above every rounding of
// both sides); the rest (about 2^-18 p + 2^-22 of the draws) takes the exact fp64 test.
// Entries in S (p = 1) and with u_j = 0 (p = 0) need no draw. The weight of a kept entry
// is fl32(1 / p_j) from the exact quotient.
template <bool kCacheBits>
__global__ void __launch_bounds__(kSelThreads) sip_kernel(const float *__restrict__ scores,
                                                         int H, int bh0, int nqb, int nkb, int K,
                                                         uint32_t key0, uint32_t key1,
                                                         int32_t *__restrict__ idx,
                                                         int32_t *__restrict__ cnt,
                                                         float *__restrict__ w,
                                                         double *__restrict__ p_out, int *flag,
                                                         size_t rows)
{
    extern __shared__ __align__(16) uint32_t sip_sh[];  // kCacheBits: [8 warps][nkb]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // row of this call; its (b, h) counts from the call's first head pair bh0 (a call on
    // a range of head pairs draws the same numbers as one on the whole tensor)
    const size_t row = (size_t)blockIdx.x * kSelWarps + warp;
    if (row >= rows) return;  // no block barrier below: the warp may leave alone
    const int bh = bh0 + (int)(row / nqb);
    const int b = bh / H, h = bh % H;
    const int qb = (int)(row % nqb);
    const float *s = scores + row * nkb;
    uint32_t *bits_sh = sip_sh + (kCacheBits ? (size_t)warp * nkb : 0);
    int32_t *idx_row = idx + row * nkb;
    float *w_row = w + row * nkb;
    auto bits_of = [&](int j) -> uint32_t {
        return j >= nkb ? 0u : kCacheBits ? bits_sh[j] : score_bits(__ldg(s + j));
    };

    // pass 0: validate, U = sum u_j, number of positive u_j. U is summed exactly as
    // U_hi = sum (u_j >> 12) and U_lo = sum (u_j & 0xfff) (neither can overflow), and a row
    // whose U needs more than 64 bits is rejected like a bad score.
    unsigned long long u_hi = 0, u_lo = 0, npos = 0, nbad = 0;
    for (int j0 = 0; j0 < nkb; j0 += 32 * kSipUnroll) {
        float v[kSipUnroll];
#pragma unroll
        for (int c = 0; c < kSipUnroll; ++c) {
            const int j = j0 + 32 * c + lane;
            v[c] = j < nkb ? __ldg(s + j) : 0.f;
        }
#pragma unroll
        for (int c = 0; c < kSipUnroll; ++c) {
            const int j = j0 + 32 * c + lane;
            if (j >= nkb) continue;
            if (!score_ok(v[c])) {
                ++nbad;
                continue;
            }
            const uint32_t bj = score_bits(v[c]);
            if (kCacheBits) bits_sh[j] = bj;
            const uint64_t u = fixed50_bits(bj);
            u_hi += u >> 12;
            u_lo += u & 0xfffull;
            npos += u > 0;
        }
    }
    u_hi = warp_sum(u_hi);
    u_lo = warp_sum(u_lo);
    npos = warp_sum(npos);
    nbad = warp_sum(nbad);
    const unsigned long long top = u_hi + (u_lo >> 12);  // U = top * 2^12 + (U_lo mod 2^12)
    const unsigned long long U = (top << 12) | (u_lo & 0xfffull);
    if (nbad != 0 || top >= (1ull << 52)) {
        for (int j = lane; j < nkb; j += 32) {
            idx_row[j] = -1;
            w_row[j] = 0.f;
            if (p_out) p_out[row * nkb + j] = 0.0;
        }
        if (lane == 0) {
            cnt[row] = 0;
            raise_flag(flag, AB_FLAG_BAD_SCORE);
        }
        return;
    }
    __syncwarp();

    // saturated set S = {u_j >= theta}: at most K positive entries keep exactly those
    // (p = 1 on them, 0 elsewhere); otherwise the fixed point above
    const uint32_t b_one = bits_threshold(1);  // u_j >= 1
    const bool all_positive_kept = npos <= (unsigned long long)K;
    uint32_t theta_b = b_one;
    uint64_t k_rest = 0, R = 0;
    if (!all_positive_kept) {
        uint64_t theta = ~0ull;  // S empty
        theta_b = 0xFFFFFFFFu;
        unsigned long long sizeS = 0, sumS = 0;
        for (;;) {
            k_rest = (uint64_t)K - sizeS;
            R = U - sumS;
            const uint64_t thr = ceil_div_threshold(R, k_rest);
            if (thr >= theta) break;  // every u_j >= thr is in S already
            const uint32_t thr_b = bits_threshold(thr);
            unsigned long long add_n = 0, add_u = 0;
            for (int j0 = 0; j0 < nkb; j0 += 32 * kSipUnroll) {
                uint32_t bv[kSipUnroll];
#pragma unroll
                for (int c = 0; c < kSipUnroll; ++c) bv[c] = bits_of(j0 + 32 * c + lane);
#pragma unroll
                for (int c = 0; c < kSipUnroll; ++c) {
                    if (bv[c] >= thr_b && bv[c] < theta_b) {  // out-of-row entries read 0
                        ++add_n;
                        add_u += fixed50_bits(bv[c]);
                    }
                }
            }
            add_n = warp_sum(add_n);
            add_u = warp_sum(add_u);
            theta = thr;
            theta_b = thr_b;
            if (add_n == 0) break;
            sizeS += add_n;
            sumS += add_u;
        }
    }

    // draws and ordered compaction in one ascending walk: each 32-entry chunk's keep
    // ballot places its kept entries after those of the chunks before it. The four chunks
    // of a step draw their Philox numbers first, unconditionally (independent chains the
    // scheduler interleaves); the weights follow in a second walk over the kept entries
    // only, one per lane, so the fp64 quotients never wait on a divergent branch.
    const double Rd = __ull2double_rn(R);
    const float c_f = all_positive_kept ? 0.f : __double2float_rn(__ull2double_rn(k_rest) / Rd);
    // exact p_j from the bit pattern (1 in S, 0 for u = 0 or when only S is kept)
    auto prob = [&](uint32_t bj) -> double {
        if (bj >= theta_b) return 1.0;
        if (all_positive_kept || bj < b_one) return 0.0;
        return __ull2double_rn(k_rest * fixed50_bits(bj)) / Rd;
    };
    uint32_t rk0[10], rk1[10];  // Philox round keys
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        rk0[r] = key0 + (uint32_t)r * 0x9E3779B9u;
        rk1[r] = key1 + (uint32_t)r * 0xBB67AE85u;
    }
    const unsigned lt = (1u << lane) - 1u;
    int base = 0;
    for (int j0 = 0; j0 < nkb; j0 += 32 * kSipUnroll) {
        uint32_t bv[kSipUnroll];
        uint4 x[kSipUnroll];
#pragma unroll
        for (int c = 0; c < kSipUnroll; ++c) bv[c] = bits_of(j0 + 32 * c + lane);
#pragma unroll
        for (int c = 0; c < kSipUnroll; ++c)
            x[c] = philox_4x32_10(
                make_uint4((uint32_t)(j0 + 32 * c + lane), (uint32_t)qb, (uint32_t)h, (uint32_t)b),
                rk0, rk1);
#pragma unroll
        for (int c = 0; c < kSipUnroll; ++c) {
            const int j = j0 + 32 * c + lane;
            const uint32_t bj = bv[c];
            bool keep = false;
            if (j < nkb) {
                if (p_out) p_out[row * nkb + j] = prob(bj);
                if (bj >= theta_b) {
                    keep = true;
                } else if (!all_positive_kept && bj >= b_one) {
                    // u_j as a float is exact: floor of the exactly scaled score
                    const float pf = floorf(__uint_as_float(bj) * 0x1p50f) * c_f;
                    const float af = __uint_as_float((x[c].x >> 9) | 0x3F800000u) - 1.0f;  // top 23 bits
                    if (af < fmaf(pf, 1.0f - 0x1p-19f, -0x1p-22f)) {
                        keep = true;
                    } else if (af < pf * (1.0f + 0x1p-19f)) {
                        const uint64_t r53 = ((((uint64_t)x[c].x) << 32) | x[c].y) >> 11;
                        keep = __ull2double_rn(r53) < prob(bj) * 9007199254740992.0;
                    }
                }
            }
            const unsigned m = __ballot_sync(0xffffffffu, keep);
            if (keep) idx_row[base + __popc(m & lt)] = j;
            base += __popc(m);
        }
    }
    __syncwarp();  // the kept indices written above are read back by other lanes
    for (int c = lane; c < base; c += 32) {
        const uint32_t bj = bits_of(idx_row[c]);
        w_row[c] = bj >= theta_b ? 1.0f : __double2float_rn(1.0 / prob(bj));
    }
    for (int c = base + lane; c < nkb; c += 32) {
        idx_row[c] = -1;
        w_row[c] = 0.f;
    }
    if (lane == 0) cnt[row] = base;
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
    const size_t rows = (size_t)n_bh * nqb;
    const unsigned grid = (unsigned)((rows + kSelWarps - 1) / kSelWarps);
    const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
    if (nkb <= kSipCacheMax) {
        const size_t smem = (size_t)kSelWarps * nkb * 4;
        cudaError_t e = allow_smem(sip_kernel<true>, smem);
        if (e != cudaSuccess) return e;
        sip_kernel<true><<<grid, kSelThreads, smem, st>>>(scores, H, bh0, nqb, nkb, K, k0, k1, idx,
                                                          cnt, w, p, flag, rows);
    } else {
        sip_kernel<false><<<grid, kSelThreads, 0, st>>>(scores, H, bh0, nqb, nkb, K, k0, k1, idx,
                                                        cnt, w, p, flag, rows);
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
