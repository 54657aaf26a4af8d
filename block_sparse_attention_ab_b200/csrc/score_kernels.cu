// score_kernels.cu -- IBCS block scoring on sm_100a (AB-Attention news page, section
// «Три приёма AB-Attention», first technique): mean key per 128-token key block,
// per-query-block k-means into C <= 8 weighted clusters, and the block score
// s_j = sum_c w_c softmax_j(cent_c . kbar_j / sqrt(d)).
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ab_device.cuh"
#include "ab_kernels.h"
#include "tmap_host.h"

namespace ab {

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// Round-to-nearest-even of a finite fp32 value to bf16 precision on its bit pattern:
// add 0x7FFF plus the lowest kept bit, then clear the 16 dropped bits (integer pipe,
// no conversion unit). The result is an fp32 bit pattern whose upper half is the bf16.
__device__ __forceinline__ uint32_t rne_bf16_bits(float x)
{
    const uint32_t u = __float_as_uint(x);
    return (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
}

// Exact three-term bf16 split of an fp32 value on the integer pipe, x = hi + mid + lo
// with every term a bf16 (each subtraction is exact: the remainder of rounding to 8
// significant bits has at most 16, then at most 8); the terms come back as fp32 bit
// patterns (bf16 in the upper half). Products of two such splits with the terms of total
// order <= 4 reproduce an fp32 product to about 2^-24 relative.
__device__ __forceinline__ void split3_bits(float x, uint32_t &a, uint32_t &b, uint32_t &c)
{
    a = rne_bf16_bits(x);
    const float r = x - __uint_as_float(a);
    b = rne_bf16_bits(r);
    c = rne_bf16_bits(r - __uint_as_float(b));
}

// x / n for a member count n >= 1: hardware reciprocal estimate, quotient, and one
// Newton residual correction q + (x - q n) r (Markstein's method), within about one ulp
// of the rounded quotient.
__device__ __forceinline__ float div_by_count(float x, float n, float r)
{
    const float q = x * r;
    return fmaf(fmaf(-q, n, x), r, q);
}

__device__ __forceinline__ float rcp_approx(float n)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(n));
    return r;
}

// Power-of-two scaling for the two-term fp16 split of the block-score operands: the
// exponent e with amax * 2^e in [2^14, 2^15) for a vector whose largest magnitude is amax
// (0 for a zero vector; clamped to [-126, 126]). The scaled components stay below the
// fp16 maximum, and the low term of a component within 2^10 of amax is a normal fp16.
__device__ __forceinline__ int scale_exponent(float amax)
{
    if (!(amax > 0.f)) return 0;
    const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127;  // floor(log2 amax)
    return min(126, max(-126, 14 - ex));
}

// 2^e as a float, e in [-126, 127]
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// Two-term fp16 split of y (|y| < 2^15): y = hi + lo + r with hi, lo fp16 and |r| at most
// half an fp16 ulp of lo; y - hi is exact in fp32 (hi keeps the leading 11 bits of y).
__device__ __forceinline__ uint32_t half2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

__device__ __forceinline__ void split2h_x8(const float (&y)[8], uint4 (&t)[2])
{
    uint32_t a[4], b[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __half2 h = __floats2half2_rn(y[2 * e], y[2 * e + 1]);
        const float2 hf = __half22float2(h);
        a[e] = half2_bits(h);
        b[e] = half2_bits(__floats2half2_rn(y[2 * e] - hf.x, y[2 * e + 1] - hf.y));
    }
    t[0] = make_uint4(a[0], a[1], a[2], a[3]);
    t[1] = make_uint4(b[0], b[1], b[2], b[3]);
}

// Byte offset of the 16-byte chunk holding element (row, col) of a K-major tile stored
// as 64-column (128-byte) panels of `panel_bytes` each, with the 128-byte swizzle that
// TMA and the tcgen05 descriptors use (chunk index XOR row mod 8; tiles 1024-aligned).
__device__ __forceinline__ int sw128_chunk(int row, int col, int panel_bytes)
{
    return (col >> 6) * panel_bytes + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4);
}

// ---------------------------------------------------------------------------------
// Mean key: one CTA of 256 threads per (b, h, key block); 16-byte coalesced loads,
// fp32 sums in a fixed order, divided by the block's valid-key count. Also writes the
// mean key for the tensor-core block score: scaled by 2^e (scale_exponent of its largest
// component) and split into two fp16 terms, kbs[t][bh][j][i] (t = 0 high, 1 low), with
// the unscale factor 2^-e in kscale[bh][j] (row stride ks_stride).
// ---------------------------------------------------------------------------------
// At most 32 registers per thread (8 CTAs' worth of the register file): a CTA then fits
// beside four k-means CTAs, so the mean keys can start on SMs that still run the last
// k-means wave (ab_score launches them on a side stream).
template <int D>
__global__ void __launch_bounds__(256, 8) meankey_kernel(const __nv_bfloat16 *__restrict__ k,
                                                      float *__restrict__ kbar,
                                                      __half *__restrict__ kbs,
                                                      float *__restrict__ kscale, int N,
                                                      int N_pad, int nkb, int ks_stride)
{
    constexpr int VEC = D / 8;         // 16-byte vectors per row
    constexpr int GROUPS = 256 / VEC;  // row groups
    constexpr int RPT = 128 / GROUPS;  // rows per thread
    __shared__ __align__(16) float part[GROUPS][D];
    __shared__ float wmax[D / 32];

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
    // thread col < D owns column col (D <= 128 < 256 threads)
    const float inv = 1.0f / (float)nv;
    float m = 0.f;
    if (tid < D) {
        float sum = 0.f;
#pragma unroll 8
        for (int g = 0; g < GROUPS; ++g) sum += part[g][tid];
        m = sum * inv;
        kbar[(size_t)blk * D + tid] = m;
    }
    // the mean key's largest |component|: warp maxima, then over the D / 32 warps
    float amax = fabsf(m);
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (tid < D && (tid & 31) == 0) wmax[tid >> 5] = amax;
    __syncthreads();
    if (tid < D) {
        amax = wmax[0];
#pragma unroll
        for (int w = 1; w < D / 32; ++w) amax = fmaxf(amax, wmax[w]);
        const int e = scale_exponent(amax);
        const float y = m * pow2f(e);
        const __half hi = __float2half_rn(y);
        const size_t term = (size_t)gridDim.x * D;
        kbs[(size_t)blk * D + tid] = hi;
        kbs[term + (size_t)blk * D + tid] = __float2half_rn(y - __half2float(hi));
        if (tid == 0) kscale[(size_t)bh * ks_stride + j] = pow2f(-e);
    }
}

// ---------------------------------------------------------------------------------
// Mean key of 4-token key units (the page's fine-grained selection unit): one CTA of
// 256 threads per (b, h, 128-token span) = 32 units; thread (unit, 16-byte column chunk)
// sums the unit's valid rows (fixed order) and writes the fp32 mean, its two scaled fp16
// terms and (for chunk 0) the unit's unscale factor, as meankey_kernel. The D / 8 threads
// of a unit are adjacent lanes of one warp and share its largest |component| by shuffles.
// A unit with no valid token gets 0 (factor 1).
// ---------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) meankey4_kernel(const __nv_bfloat16 *__restrict__ k,
                                                       float *__restrict__ kbar,
                                                       __half *__restrict__ kbs,
                                                       float *__restrict__ kscale, int N,
                                                       int N_pad, int nspan, int ks_stride)
{
    constexpr int CH = D / 8;                // 16-byte chunks per row
    constexpr int PER = 32 * CH / 256;       // (unit, chunk) pairs per thread
    const int span = blockIdx.x;
    const int bh = span / nspan, sp = span % nspan;
    const int nku = N_pad / 4;
    const size_t term = (size_t)gridDim.x * 32 * D;  // one term of all units
#pragma unroll
    for (int it = 0; it < PER; ++it) {
        const int e = threadIdx.x + it * 256;
        const int ul = e / CH, ch = e % CH;        // unit within the span, chunk
        const int u = sp * 32 + ul;                // unit within the head
        const int t0 = u * 4;
        const int nv = max(0, min(4, N - t0));
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = 0.f;
        const uint4 *base = reinterpret_cast<const uint4 *>(k + ((size_t)bh * N_pad + t0) * D) + ch;
        for (int r = 0; r < nv; ++r) {
            const uint4 v = __ldg(base + (size_t)r * CH);
            acc[0] += bf16_lo(v.x); acc[1] += bf16_hi(v.x);
            acc[2] += bf16_lo(v.y); acc[3] += bf16_hi(v.y);
            acc[4] += bf16_lo(v.z); acc[5] += bf16_hi(v.z);
            acc[6] += bf16_lo(v.w); acc[7] += bf16_hi(v.w);
        }
        const float inv = nv > 0 ? 1.0f / (float)nv : 0.f;
        float m[8];
        float amax = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            m[c] = acc[c] * inv;
            amax = fmaxf(amax, fabsf(m[c]));
        }
#pragma unroll
        for (int o = CH / 2; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const int ex = scale_exponent(amax);
        const float sc = pow2f(ex);
        const size_t o = ((size_t)bh * nku + u) * D + ch * 8;
        float4 *dst = reinterpret_cast<float4 *>(kbar + o);
        dst[0] = make_float4(m[0], m[1], m[2], m[3]);
        dst[1] = make_float4(m[4], m[5], m[6], m[7]);
#pragma unroll
        for (int c = 0; c < 8; ++c) m[c] *= sc;
        uint4 t[2];
        split2h_x8(m, t);
        *reinterpret_cast<uint4 *>(kbs + o) = t[0];
        *reinterpret_cast<uint4 *>(kbs + term + o) = t[1];
        if (ch == 0) kscale[(size_t)bh * ks_stride + u] = pow2f(-ex);
    }
}

// ---------------------------------------------------------------------------------
// Per-block k-means on the 5th-generation tensor cores. One CTA of 128 threads per
// (b, h, query block). The block's queries arrive by TMA (128-byte swizzle; rows past
// N read as zero) and stay in shared memory for all T iterations. Each iteration runs
// two single-CTA tcgen05 GEMMs with fp32 accumulators in TMEM:
//   assign: G = Q B^T (M = 128 queries, N = 32, K = d): columns 8t + c of B hold term
//           t (split3_bits) of fp32 centroid c, columns 24..31 are zero (B is stored
//           MN-major, so each thread writes its feature's 24 terms as three 16-byte
//           chunks), so q . c =
//           G[q][c] + G[q][8 + c] + G[q][16 + c] is the bf16 query times the fp32
//           centroid; distance |c|^2 - 2 q.c (|q|^2 is common), argmin with ties to
//           the lowest cluster; thread t reads TMEM lane t = query t;
//   update: S = Q^T H (M = 128 features, Q read feature-major from the same tile;
//           N = 16 clusters, one-hot rows 8..15 zero; K = 128 queries): member sums,
//           exact 0/1 and bf16 operands with fp32 accumulation, divided by the member
//           counts; thread i reads TMEM lane i = feature i; an empty cluster keeps its
//           centroid.
// Thread i keeps feature i of the 8 centroids in registers: after each update it
// writes column i of the next assignment's B operand and its share of the squared
// norms (reduced across the warp, then across the 4 warps through shared memory).
// A round whose assignments equal the previous round's ends the iteration there: the
// update would give the same centroids bit for bit, so the remaining rounds change
// nothing (the outputs equal those of all T rounds).
// One elected thread of warp 0 issues the MMAs. Every wait is bounded; a timed-out
// CTA drains its in-flight work and exits.
// ---------------------------------------------------------------------------------
template <int D>
struct KmSmem {
    static constexpr int kQ = 0;                        // queries: 2 panels [128][64] bf16
    static constexpr int kBA = kQ + 2 * 16384;          // centroid terms: [D][64], MN-major
    static constexpr int kBU = kBA + D * 128;           // one-hot: [128 queries][16], MN-major
    static constexpr int kBar = kBU + 2 * 2048;         // q_full, mma_done, drain
    static constexpr int kMisc = kBar + 3 * 8;          // TMEM base, abort flag
    static constexpr int kBytes = kMisc + 8;
    static constexpr int kAlloc = kBytes + 1024;        // slack to align the base to 1024 B
};

constexpr int kKmTmemCols = 64;  // G in columns 0..31, S in columns 32..47

// Write feature k of the 8 centroids as column k of the assignment GEMM's B operand
// (three bf16 terms each) and the warp's partial squared norms to normw[c][warp].
// kFirst: the initial centroids are bf16 queries, whose middle and low terms are exactly
// zero; those rows were zeroed at the start, so only the high terms are written.
template <int D, bool kFirst = false>
__device__ __forceinline__ void km_publish(uint8_t *smem, const float (&cur)[8], int k,
                                           bool has_k, int warp, int lane, float (*normw)[4])
{
    // The assignment GEMM's B operand is stored MN-major (the 8 clusters of a term are
    // contiguous): row k of the 128-byte-swizzled tile holds feature k, its 16-byte chunk
    // t the bf16 term t of the 8 centroids (chunk 3, the zero rows 24..31, stays zero).
    float sq[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) sq[c] = cur[c] * cur[c];
    if (has_k) {
        uint32_t t[3][8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            if (kFirst) {
                t[0][c] = __float_as_uint(cur[c]);
                t[1][c] = t[2][c] = 0u;
            } else {
                split3_bits(cur[c], t[0][c], t[1][c], t[2][c]);
            }
        }
        uint8_t *row = smem + KmSmem<D>::kBA + k * 128;
#pragma unroll
        for (int tt = 0; tt < 3; ++tt) {
            // two bf16 per 32-bit word: the upper halves of the fp32 patterns of c, c + 1
            const uint4 v = make_uint4(__byte_perm(t[tt][0], t[tt][1], 0x7632),
                                       __byte_perm(t[tt][2], t[tt][3], 0x7632),
                                       __byte_perm(t[tt][4], t[tt][5], 0x7632),
                                       __byte_perm(t[tt][6], t[tt][7], 0x7632));
            *reinterpret_cast<uint4 *>(row + ((tt ^ (k & 7)) << 4)) = v;
        }
    }
    // reduce-scatter across the warp: lane L ends with cluster (L >> 2) & 7
    const bool b16 = (lane & 16) != 0, b8 = (lane & 8) != 0, b4 = (lane & 4) != 0;
    float u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b16 ? sq[i] : sq[i + 4], keep = b16 ? sq[i + 4] : sq[i];
        u[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    float w2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b8 ? u[i] : u[i + 2], keep = b8 ? u[i + 2] : u[i];
        w2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float v = (b4 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, b4 ? w2[0] : w2[1], 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    if ((lane & 3) == 0) normw[(lane >> 2) & 7][warp] = v;
}

template <int D>
__global__ void __launch_bounds__(128, 4) kmeans_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                     int N, int N_pad, int nqb, int C, int T,
                                                     float *__restrict__ cent_out,
                                                     float *__restrict__ w_out,
                                                     uint8_t *__restrict__ assign_out, int *flag)
{
    using L = KmSmem<D>;
    constexpr int CMAX = 8;
    extern __shared__ uint8_t km_raw[];
    uint8_t *smem = align_smem_1024(km_raw);
    __shared__ __align__(16) float normw[CMAX][4];  // squared-norm partials per warp
    __shared__ __align__(16) int wcount[CMAX][4];   // member counts per warp
    __shared__ uint8_t lab[128];
    __shared__ int wchanged[4];                     // per warp: an assignment changed
    uint64_t *q_full = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint64_t *mma_done = q_full + 1;
    uint64_t *drain = q_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);

    const int blk = blockIdx.x;
    const int bh = blk / nqb, qb = blk % nqb;
    const int t0 = qb * 128;
    const int nv = min(128, N - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool has_k = tid < D;  // this thread owns feature tid

    if (tid == 0) {
        mbar_init(q_full, 1);
        mbar_init(mma_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        // the query tile's load goes out first and overlaps the rest of the set-up
        prefetch_tmap(&tmQ);
        mbar_arrive_expect_tx(q_full, (D / 64) * 16384);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
            tma_load_3d(smem + L::kQ + h * 16384, &tmQ, q_full, h * 64, t0, bh);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kKmTmemCols);
        tmem_relinquish();
    }
    // zero: the constant padding clusters 24..31 of the centroid terms (chunk 3 of every
    // feature row), one-hot rows 8..15
    if (tid < D)
        *reinterpret_cast<uint4 *>(smem + L::kBA + tid * 128 + ((3 ^ (tid & 7)) << 4)) =
            make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(smem + L::kBU + tid * 32 + ((1 ^ ((tid >> 2) & 1)) << 4)) =
        make_uint4(0, 0, 0, 0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool ok = mbar_wait(q_full, 0, abort_flag, flag);

    // initial centroid c: the query at block-local index c*floor(nv/C) (min(c, nv-1)
    // when nv < C); this thread holds feature tid of every centroid
    float cur[CMAX];
    {
        const __nv_bfloat16 *qs = reinterpret_cast<const __nv_bfloat16 *>(smem + L::kQ);
        const int stride = nv / C;
#pragma unroll
        for (int c = 0; c < CMAX; ++c) {
            const int src = nv >= C ? c * stride : min(c, nv - 1);
            cur[c] = (ok && has_k && c < C)
                         ? __bfloat162float(qs[(sw128_chunk(src, tid, 16384) >> 1) + (tid & 7)])
                         : 0.f;
        }
    }
    km_publish<D, true>(smem, cur, tid, has_k, warp, lane, normw);
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);

    const uint32_t q_addr = smem_u32(smem + L::kQ);
    const uint64_t a_asg = smem_desc_sw128(q_addr, 16, 1024);
    const uint64_t b_asg = smem_desc_sw128(smem_u32(smem + L::kBA), 16384, 1024);  // MN-major
    const uint64_t a_upd = smem_desc_sw128(q_addr, 16384, 1024);  // feature-major view of Q
    // MN-major, 32-byte swizzle: 8-row groups of 256 bytes
    const uint64_t b_upd = (smem_desc_sw128(smem_u32(smem + L::kBU), 16, 256) & ~(7ull << 61)) |
                           (6ull << 61);
    constexpr uint32_t idesc_asg = idesc_bf16_f32(128, 32, 0, 1);
    constexpr uint32_t idesc_upd = idesc_bf16_f32(128, 16, 1, 1);
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
    uint32_t phase = 0;

    for (int it = 0; it < T && ok; ++it) {
        tc_fence_after();
        // (1) assignment GEMM
        if (warp == 0) {
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem, a_asg + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                           b_asg + (uint64_t)((kk * 2048) >> 4), idesc_asg,
                           kk > 0 ? 1u : 0u);
                mma_commit(mma_done);
            }
            __syncwarp();
        }
        float cn[CMAX];
#pragma unroll
        for (int c = 0; c < CMAX; ++c) {
            const float4 p = *reinterpret_cast<const float4 *>(normw[c]);
            cn[c] = (p.x + p.y) + (p.z + p.w);
        }
        bool good = __all_sync(0xffffffffu, mbar_wait(mma_done, phase, abort_flag, flag));
        phase ^= 1;
        tc_fence_after();
        {
            uint32_t g[32];
            if (good) {
                tmem_ld32(t_lane, g);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) g[e] = 0u;
            }
            float best = INFINITY;
            int arg = 0;
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
                const float dot = (__uint_as_float(g[c]) + __uint_as_float(g[8 + c])) +
                                  __uint_as_float(g[16 + c]);
                const float dist = fmaf(-2.f, dot, cn[c]);
                if (c < C && dist < best) {
                    best = dist;
                    arg = c;
                }
            }
            const int a = tid < nv ? arg : 255;
            const bool changed = it == 0 || lab[tid] != (uint8_t)a;  // lab: previous round
            lab[tid] = (uint8_t)a;
            const unsigned chg = __ballot_sync(0xffffffffu, changed);
            if (lane == 0) wchanged[warp] = chg != 0u;
            // (2) one-hot row of this query (B of the update GEMM, MN-major with the 32-byte
            // swizzle: row tid holds clusters 0..7 in its first 16-byte chunk, 8..15 zero in
            // the other) and member counts
            {
                const uint32_t one = a < 8 ? 0x3F80u << (16 * (a & 1)) : 0u;
                const int wsel = a >> 1;
                *reinterpret_cast<uint4 *>(smem + L::kBU + tid * 32 + (((tid >> 2) & 1) << 4)) =
                    make_uint4(wsel == 0 ? one : 0u, wsel == 1 ? one : 0u, wsel == 2 ? one : 0u,
                               wsel == 3 ? one : 0u);
            }
#pragma unroll
            for (int c = 0; c < CMAX; ++c) {
                const unsigned m = __ballot_sync(0xffffffffu, a == c);
                if (lane == 0) wcount[c][warp] = __popc(m);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(good);
        if (!ok) break;
        // Converged: this round reproduced the previous assignments, so the update would
        // reproduce the current centroids bit for bit (same members, same sums) and every
        // later round this one. The outputs of all T rounds are the current ones.
        if (it > 0 && (wchanged[0] | wchanged[1] | wchanged[2] | wchanged[3]) == 0) break;
        tc_fence_after();

        // (3) update GEMM
        if (warp == 0) {
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tmem + 32, a_upd + (uint64_t)((kk * 2048) >> 4),
                           b_upd + (uint64_t)((kk * 512) >> 4), idesc_upd,
                           kk > 0 ? 1u : 0u);
                mma_commit(mma_done);
            }
            __syncwarp();
        }
        int cnt[CMAX];
#pragma unroll
        for (int c = 0; c < CMAX; ++c) {
            const int4 w4 = *reinterpret_cast<const int4 *>(wcount[c]);
            cnt[c] = (w4.x + w4.y) + (w4.z + w4.w);
        }
        good = __all_sync(0xffffffffu, mbar_wait(mma_done, phase, abort_flag, flag));
        phase ^= 1;
        tc_fence_after();
        if (good) {
            uint32_t sv[16];
            tmem_ld16(t_lane + 32, sv);
            tmem_wait_ld();
            // lanes >= d (d = 64) hold rows of an unused panel: ignored
            if (has_k) {
#pragma unroll
                for (int c = 0; c < CMAX; ++c) {
                    if (c < C && cnt[c] > 0) {
                        const float n = (float)cnt[c];
                        cur[c] = div_by_count(__uint_as_float(sv[c]), n, rcp_approx(n));
                    }
                }
            }
        }
        // (4) next assignment's B operand and squared norms
        km_publish<D>(smem, cur, tid, has_k, warp, lane, normw);
        fence_proxy_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(good);
    }

    if (ok) {
        if (has_k) {
#pragma unroll
            for (int c = 0; c < CMAX; ++c)
                if (c < C) cent_out[((size_t)blk * C + c) * D + tid] = cur[c];
        }
        if (tid < C) {
            const int4 w4 = *reinterpret_cast<const int4 *>(wcount[tid]);
            w_out[(size_t)blk * C + tid] = (float)((w4.x + w4.y) + (w4.z + w4.w)) / (float)nv;
        }
        if (assign_out) assign_out[(size_t)bh * N_pad + t0 + tid] = lab[tid];
    } else if (warp == 0) {
        // unwind: let the query copy and the last MMAs land before releasing memory
        if (elect_one()) {
            mma_commit(drain);
            drain_wait(drain, 0);
            drain_wait(q_full, 0);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kKmTmemCols);
    }
}

// ---------------------------------------------------------------------------------
// Block score on the 5th-generation tensor cores. One CTA per (b, h, 16 query
// blocks); its 128 TMEM lanes are the centroid rows r = 8 * (query block) + c
// (clusters c >= C and query blocks past the end are zero rows with weight 0).
// Logits L[r][j] = cent_r . kbar_j are computed as 128 x 64 x d tcgen05 GEMMs over
// tiles of 64 key blocks. Both fp32 operands are scaled by powers of two (each centroid
// row and each mean key so that its largest component lies in [2^14, 2^15)) and split
// into two fp16 terms, hi + lo, which hold 22 significant bits; the three products
// hi.hi + hi.lo + lo.hi accumulate in fp32, the omitted lo.lo and the split's remainder
// lie near 2^-22 of each product, and the exact power-of-two unscaling enters the
// epilogue's per-row and per-column factors. The centroid terms are built once in shared
// memory by all threads; the key terms and factors are written by the mean-key kernel,
// the terms arrive by TMA.
// Key blocks are processed in chunks of 256 (one TMEM buffer of 256 columns; two
// buffers). With n_kb <= 256 one pass suffices: each row's softmax max and sum and
// then the scores come from the logits held in TMEM. With more chunks, a first pass
// accumulates each row's max and sum online and a second pass recomputes the logits
// and writes s_j = sum_c (w_c / Z_c) 2^(L'_cj - m_c) (L' in log2 units), the sum over
// a query block's 8 centroid rows taken across 8 lanes (butterfly reduce-scatter).
// Warp 0: TMA producer; warp 1: TMEM owner and MMA issuer; warps 2..9: epilogue, two
// per TMEM lane group (warp w reads lanes 32 (w mod 4) .. +31 and takes every other 32-
// column slice of a chunk, starting at slice (w - 2) / 4). Each keeps its own row max and
// sum over its slices through the statistics pass; the two of a lane group merge them
// once, where the output pass begins.
// ---------------------------------------------------------------------------------
constexpr int kScThreads = 320;
constexpr int kScChunk = 256;
constexpr int kScTmemCols = 512;

template <int D>
struct ScSmem {
    static constexpr int kPanels = D / 64;
    static constexpr int kATerm = kPanels * 16384;           // one term of the 128 centroid rows
    static constexpr int kBTerm = kPanels * 8192;            // one term of 64 mean keys
    static constexpr int kStageBytes = 2 * kBTerm;
    static constexpr int kStages = D == 128 ? 4 : 8;
    static constexpr int kA = 0;
    static constexpr int kB = kA + 2 * kATerm;
    static constexpr int kBar = kB + kStages * kStageBytes;
    // barriers: full[S], empty[S], tfull[2], tempty[2], drain, a_ready
    static constexpr int kNumBars = 2 * kStages + 6;
    static constexpr int kRows = kBar + kNumBars * 8;  // float [128]: 2^-e per centroid row
    // float [8 warps][2 jobs][256]: column factors, read as float4 (16-byte aligned)
    static constexpr int kFac = (kRows + 128 * 4 + 15) & ~15;
    static constexpr int kXch = kFac + 8 * 2 * 256 * 4;  // float [2][2][128]: (m, z) per half
    static constexpr int kMisc = kXch + 2 * 2 * 128 * 4;  // TMEM base, abort flag
    static_assert(kFac % 16 == 0 && kB % 1024 == 0, "shared-memory layout alignment");
    static constexpr int kBytes = kMisc + 8;
    static constexpr int kAlloc = kBytes + 1024;
};

// the three term products (a, b), terms numbered 0 (hi), 1 (lo): (0,0) (0,1) (1,0)
__host__ __device__ constexpr int prod_term_a(int pr) { return pr == 2 ? 1 : 0; }
__host__ __device__ constexpr int prod_term_b(int pr) { return pr == 1 ? 1 : 0; }

template <int D>
__global__ void __launch_bounds__(kScThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap tmKB, const float *__restrict__ cent,
                 const float *__restrict__ cw, const float *__restrict__ kscale, int ks_stride,
                 int BH, int nqb, int nkb, int nkb_valid, int C, float scale_log2,
                 float *__restrict__ scores, int *flag)
{
    using L = ScSmem<D>;
    extern __shared__ uint8_t sc_raw[];
    uint8_t *smem = align_smem_1024(sc_raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint64_t *empty = full + L::kStages;
    uint64_t *tfull = empty + L::kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);

    const int g = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    uint64_t *a_ready = drain + 1;  // the centroid terms and row factors are in place
    float *row_unscale = reinterpret_cast<float *>(smem + L::kRows);  // 2^-e per centroid row
    if (tid == 0) {
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 256);
        }
        mbar_init(drain, 1);
        mbar_init(a_ready, 8);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kScTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 2) {
        // Centroid terms (A operand), built by the eight epilogue warps while the producer
        // already streams mean-key tiles: warp w takes rows 16 (w - 2) .. + 15, each row
        // read once (a row spans 128 / D warp passes' lanes: D / 4 lanes of one float4
        // each), its scale exponent from a shuffle max, then scaled, split and stored.
        constexpr int LPR = D / 4;        // lanes per row
        constexpr int RPP = 32 / LPR;     // rows per warp pass
        constexpr int PASSES = 16 / RPP;  // passes for the warp's 16 rows
        const int sub = lane / LPR, li = lane % LPR;
        float4 u[PASSES];
#pragma unroll
        for (int ps = 0; ps < PASSES; ++ps) {
            const int row = (warp - 2) * 16 + ps * RPP + sub;
            const int qb = g * 16 + (row >> 3), c = row & 7;
            u[ps] = (qb < nqb && c < C)
                        ? __ldg(reinterpret_cast<const float4 *>(cent + (((size_t)bh * nqb + qb) * C + c) * D) + li)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int ps = 0; ps < PASSES; ++ps) {
            const int row = (warp - 2) * 16 + ps * RPP + sub;
            float amax = fmaxf(fmaxf(fabsf(u[ps].x), fabsf(u[ps].y)), fmaxf(fabsf(u[ps].z), fabsf(u[ps].w)));
#pragma unroll
            for (int o = LPR / 2; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const int e = scale_exponent(amax);
            const float sc = pow2f(e);
            if (li == 0) row_unscale[row] = pow2f(-e);
            const float2 y01 = make_float2(u[ps].x * sc, u[ps].y * sc);
            const float2 y23 = make_float2(u[ps].z * sc, u[ps].w * sc);
            const __half2 h01 = __floats2half2_rn(y01.x, y01.y), h23 = __floats2half2_rn(y23.x, y23.y);
            const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
            const __half2 l01 = __floats2half2_rn(y01.x - f01.x, y01.y - f01.y);
            const __half2 l23 = __floats2half2_rn(y23.x - f23.x, y23.y - f23.y);
            const int k0 = 4 * li;  // four elements: half of a 16-byte chunk
            const int off = sw128_chunk(row, k0 & ~7, 16384) + (k0 & 7) * 2;
            *reinterpret_cast<uint2 *>(smem + L::kA + off) = make_uint2(half2_bits(h01), half2_bits(h23));
            *reinterpret_cast<uint2 *>(smem + L::kA + L::kATerm + off) =
                make_uint2(half2_bits(l01), half2_bits(l23));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_ready);
    }

    const int nch = (nkb + kScChunk - 1) / kScChunk;
    const int njobs = nch == 1 ? 1 : 2 * nch;
    auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, flag));
    };

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (elect_one()) prefetch_tmap(&tmKB);
        __syncwarp();
        int pos = 0;
        bool ok = true;
        for (int j = 0; j < njobs && ok; ++j) {
            const int ch = j < nch ? j : j - nch;
            const int ns = (min(kScChunk, nkb - ch * kScChunk) + 63) >> 6;
            for (int st = 0; st < ns; ++st) {
                const int s = pos % L::kStages;
                if (!wait(&empty[s], ((pos / L::kStages) & 1) ^ 1)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    uint8_t *dst = smem + L::kB + s * L::kStageBytes;
                    mbar_arrive_expect_tx(&full[s], L::kStageBytes);
#pragma unroll
                    for (int t = 0; t < 2; ++t)
#pragma unroll
                        for (int h = 0; h < L::kPanels; ++h)
                            tma_load_3d(dst + t * L::kBTerm + h * 8192, &tmKB, &full[s], h * 64,
                                        ch * kScChunk + st * 64, t * BH + bh);
                }
                __syncwarp();
                ++pos;
            }
        }
        if (!ok) {
            // drain: the last loads issued may still be in flight
            if (elect_one()) {
                for (int k = pos - 1; k >= 0 && k >= pos - L::kStages; --k)
                    drain_wait(&full[k % L::kStages], (k / L::kStages) & 1);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer -------------------------------
        const uint64_t a0 = smem_desc_sw128(smem_u32(smem + L::kA), 16, 1024);
        const uint64_t b0 = smem_desc_sw128(smem_u32(smem + L::kB), 16, 1024);
        constexpr uint32_t idesc = idesc_f16_f32(128, 64, 0, 0);
        int pos = 0;
        bool ok = wait(a_ready, 0);
        for (int j = 0; j < njobs && ok; ++j) {
            const int buf = j & 1;
            const int ch = j < nch ? j : j - nch;
            const int ns = (min(kScChunk, nkb - ch * kScChunk) + 63) >> 6;
            if (j >= 2 && !wait(&tempty[buf], ((j >> 1) - 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int st = 0; st < ns; ++st) {
                const int s = pos % L::kStages;
                if (!wait(&full[s], (pos / L::kStages) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * kScChunk + st * 64;
                const uint64_t bs = b0 + (uint64_t)((s * L::kStageBytes) >> 4);
                if (elect_one()) {
#pragma unroll
                    for (int pr = 0; pr < 3; ++pr) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const int ta = prod_term_a(pr), tb = prod_term_b(pr);
                            mma_ss(d_tmem,
                                   a0 + (uint64_t)((ta * L::kATerm + (kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                                   bs + (uint64_t)((tb * L::kBTerm + (kk >> 2) * 8192 + (kk & 3) * 32) >> 4),
                                   idesc, (pr | kk) != 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(&empty[s]);
                }
                __syncwarp();
                ++pos;
            }
            if (!ok) break;
            if (elect_one()) mma_commit(&tfull[buf]);
            __syncwarp();
        }
        if (!ok) {
            if (elect_one()) {
                mma_commit(drain);
                drain_wait(drain, 0);
            }
            __syncwarp();
        }
    } else {
        // -------------------------------- epilogue --------------------------------
        const int qd = warp & 3;
        const int half = (warp - 2) >> 2;  // slices half, half + 2, .. of each chunk
        const int row = qd * 32 + lane;
        const int qb = g * 16 + (row >> 3), c = row & 7;
        const bool row_ok = qb < nqb;
        const float wr = (row_ok && c < C) ? __ldg(cw + ((size_t)bh * nqb + qb) * C + c) : 0.f;
        float *dst = scores + ((size_t)bh * nqb + (row_ok ? qb : 0)) * nkb;
        const uint32_t t_lane = tmem + ((uint32_t)(qd * 32) << 16);
        // the row factors are written by the other epilogue warps' operand build
        const bool ok_a = wait(a_ready, 0);
        const float rs = row_unscale[row] * scale_log2;
        // x = L * 2^-(e_row + e_j) * log2(e) / sqrt(d): the logit in log2 units from the
        // scaled product. Each warp copies a job's 256 column factors into its own shared
        // buffer (one per job parity) before it waits for the job's logits, and every
        // lane then reads the 32 factors of a TMEM slice from there (broadcast reads; the
        // factor rows are padded to a multiple of the chunk, so no read passes them).
        const float *ks_row = kscale + (size_t)bh * ks_stride;
        float *fac_w = reinterpret_cast<float *>(smem + L::kFac) + (warp - 2) * 2 * 256;
        auto stage_factors = [&](int job, int col0) {
            const float4 *src = reinterpret_cast<const float4 *>(ks_row + col0);
            float4 *fdst = reinterpret_cast<float4 *>(fac_w + (job & 1) * 256);
            fdst[lane] = __ldg(src + lane);
            fdst[32 + lane] = __ldg(src + 32 + lane);
            __syncwarp();
        };
        auto factors = [&](int job, int sl, float (&f)[32]) {
            const float4 *src = reinterpret_cast<const float4 *>(fac_w + (job & 1) * 256 + sl * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 u = src[q];
                f[4 * q + 0] = u.x * rs;
                f[4 * q + 1] = u.y * rs;
                f[4 * q + 2] = u.z * rs;
                f[4 * q + 3] = u.w * rs;
            }
        };
        float *xm = reinterpret_cast<float *>(smem + L::kXch);  // [2 halves][128]
        float *xz = xm + 2 * 128;                                // [2 halves][128]
        const int r8 = lane & 7;
        const bool b4 = (r8 & 4) != 0, b2 = (r8 & 2) != 0, b1 = (r8 & 1) != 0;
        float m = -INFINITY, z = 0.f, coef = 0.f;
        // After a failed wait a warp skips the remaining waits and work but still walks
        // every job, so both warps of a lane group always meet at the merge's barrier.
        bool ok = ok_a;
        for (int j = 0; j < njobs; ++j) {
            const int buf = j & 1;
            const int ch = j < nch ? j : j - nch;
            // this warp read the buffer of parity j & 1 for job j - 2, which it has finished
            stage_factors(j, ch * kScChunk);
            ok = ok && wait(&tfull[buf], (j >> 1) & 1);
            const int c0 = ch * kScChunk;
            const int ncols = min(kScChunk, nkb - c0);
            const int nsl = (ncols + 31) >> 5;
            // key units past the sequence end (j >= nkb_valid) take no part and score 0
            const int nvcols = max(0, min(ncols, nkb_valid - c0));
            const int nvsl = (nvcols + 31) >> 5;
            const uint32_t tb = t_lane + buf * kScChunk;
            if (ok) tc_fence_after();
            if (ok && j < nch) {
                // row statistics of this warp's slices in log2 units, online per slice: the
                // slice max (a tree of three-way maxima), then the running sum rescaled to
                // the new max plus the slice's 2^(x - max) in four partial sums
                for (int sl = half; sl < nvsl; sl += 2) {
                    uint32_t v[32];
                    float f[32];
                    tmem_ld32(tb + sl * 32, v);
                    factors(j, sl, f);
                    tmem_wait_ld();
                    const int lim = nvcols - sl * 32;
                    float x[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = i < lim ? __uint_as_float(v[i]) * f[i] : -INFINITY;
                    float t[11];
#pragma unroll
                    for (int i = 0; i < 10; ++i) t[i] = fmax3(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
                    t[10] = fmaxf(x[30], x[31]);
                    const float smax = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]),
                                             fmax3(fmax3(t[6], t[7], t[8]), t[9], t[10]));
                    const float mx = fmaxf(m, smax);
                    float zp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < lim) zp[i & 3] += fast_exp2(x[i] - mx);
                    z = (m == -INFINITY ? 0.f : z * fast_exp2(m - mx)) + ((zp[0] + zp[1]) + (zp[2] + zp[3]));
                    m = mx;
                }
            }
            if (j == nch - 1) {
                // merge the two warps' (max, sum) of each row: named barrier 1 + qd
                xm[half * 128 + row] = m;
                xz[half * 128 + row] = z;
                asm volatile("bar.sync %0, 64;" ::"r"(1 + qd) : "memory");
                const float m_o = xm[(half ^ 1) * 128 + row], z_o = xz[(half ^ 1) * 128 + row];
                const float mt = fmaxf(m, m_o);
                z = (m == -INFINITY ? 0.f : z * fast_exp2(m - mt)) +
                    (m_o == -INFINITY ? 0.f : z_o * fast_exp2(m_o - mt));
                m = mt;
                coef = z > 0.f ? wr / z : 0.f;
            }
            if (ok && (nch == 1 || j >= nch)) {
                for (int sl = half; sl < nsl; sl += 2) {
                    uint32_t v[32];
                    float f[32];
                    tmem_ld32(tb + sl * 32, v);
                    factors(j, sl, f);
                    tmem_wait_ld();
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        float e[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            e[i] = c0 + sl * 32 + q8 * 8 + i < nkb_valid
                                       ? coef * fast_exp2(fmaf(__uint_as_float(v[q8 * 8 + i]), f[q8 * 8 + i], -m))
                                       : 0.f;
                        // sum over the 8 rows (lanes) of this query block; lane r8 ends
                        // with column q8 * 8 + r8
                        float u[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float send = b4 ? e[i] : e[i + 4];
                            const float keep = b4 ? e[i + 4] : e[i];
                            u[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
                        }
                        float w2[2];
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const float send = b2 ? u[i] : u[i + 2];
                            const float keep = b2 ? u[i + 2] : u[i];
                            w2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                        }
                        const float send = b1 ? w2[0] : w2[1];
                        const float keep = b1 ? w2[1] : w2[0];
                        const float res = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                        const int col = c0 + sl * 32 + q8 * 8 + r8;
                        if (row_ok && col < nkb) dst[col] = res;
                    }
                }
            }
            if (ok) {
                tc_fence_before();
                mbar_arrive(&tempty[buf]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kScTmemCols);
    }
}

// ---------------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------------
cudaError_t launch_meankey_units(const void *k, float *kbar, void *kbar_terms, float *kscale,
                                 int BH, int N, int N_pad, int d, int unit, cudaStream_t st)
{
    if (unit != 4) return launch_meankey(k, kbar, kbar_terms, kscale, BH, N, N_pad, d, st);
    const int nspan = N_pad / 128;
    const int ks_stride = (int)kscale_stride((size_t)N_pad / 4);
    const dim3 grid((unsigned)(BH * nspan));
    __half *kbs = static_cast<__half *>(kbar_terms);
    if (d == 128)
        meankey4_kernel<128><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)k, kbar, kbs, kscale, N, N_pad,
                                                   nspan, ks_stride);
    else
        meankey4_kernel<64><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)k, kbar, kbs, kscale, N, N_pad,
                                                  nspan, ks_stride);
    return cudaGetLastError();
}

cudaError_t launch_meankey(const void *k, float *kbar, void *kbar_terms, float *kscale, int BH,
                           int N, int N_pad, int d, cudaStream_t st)
{
    const int nkb = N_pad / 128;
    const int ks_stride = (int)kscale_stride((size_t)nkb);
    const dim3 grid((unsigned)(BH * nkb));
    __half *kbs = static_cast<__half *>(kbar_terms);
    if (d == 128)
        meankey_kernel<128><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)k, kbar, kbs, kscale, N, N_pad,
                                                  nkb, ks_stride);
    else
        meankey_kernel<64><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)k, kbar, kbs, kscale, N, N_pad,
                                                 nkb, ks_stride);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_kmeans_t(const void *q, float *cent, float *cw, uint8_t *assign, int BH,
                                   int N, int N_pad, int C, int T, int *flag, cudaStream_t st)
{
    CUtensorMap tm;
    if (!make_tmap_bf16_3d(&tm, q, D, (uint64_t)N, (uint64_t)BH, (uint64_t)D * 2,
                           (uint64_t)N_pad * D * 2, 64, 128))
        return cudaErrorInvalidValue;
    const int nqb = N_pad / 128;
    const int smem = KmSmem<D>::kAlloc;
    cudaError_t e =
        cudaFuncSetAttribute(kmeans_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kmeans_kernel<D><<<(unsigned)(BH * nqb), 128, smem, st>>>(tm, N, N_pad, nqb, C, T, cent, cw,
                                                                assign, flag);
    return cudaGetLastError();
}

cudaError_t launch_kmeans(const void *q, float *cent, float *cw, uint8_t *assign, int BH, int N,
                          int N_pad, int d, int C, int T, int *flag, cudaStream_t st)
{
    return d == 128 ? launch_kmeans_t<128>(q, cent, cw, assign, BH, N, N_pad, C, T, flag, st)
                    : launch_kmeans_t<64>(q, cent, cw, assign, BH, N, N_pad, C, T, flag, st);
}

template <int D>
static cudaError_t launch_score_t(const float *cent, const float *cw, const void *kbar_terms,
                                  const float *kscale, float *scores, int BH, int nqb, int nkb,
                                  int nkb_valid, int C, int *flag, cudaStream_t st)
{
    CUtensorMap tm;
    // the fp16 terms travel as 2-byte elements (the map's type only sets the element size
    // and the zero fill)
    if (!make_tmap_bf16_3d(&tm, kbar_terms, D, (uint64_t)nkb, (uint64_t)2 * BH, (uint64_t)D * 2,
                           (uint64_t)nkb * D * 2, 64, 64))
        return cudaErrorInvalidValue;
    const int smem = ScSmem<D>::kAlloc;
    cudaError_t e =
        cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    const dim3 grid((unsigned)((nqb + 15) / 16), (unsigned)BH);
    score_kernel<D><<<grid, kScThreads, smem, st>>>(tm, cent, cw, kscale, (int)kscale_stride((size_t)nkb), BH,
                                                    nqb, nkb, nkb_valid, C, scale_log2, scores, flag);
    return cudaGetLastError();
}

cudaError_t launch_score(const float *cent, const float *cw, const void *kbar_terms,
                         const float *kscale, float *scores, int BH, int nqb, int nkb,
                         int nkb_valid, int d, int C, int *flag, cudaStream_t st)
{
    return d == 128 ? launch_score_t<128>(cent, cw, kbar_terms, kscale, scores, BH, nqb, nkb,
                                          nkb_valid, C, flag, st)
                    : launch_score_t<64>(cent, cw, kbar_terms, kscale, scores, BH, nqb, nkb,
                                         nkb_valid, C, flag, st);
}

}  // namespace ab
