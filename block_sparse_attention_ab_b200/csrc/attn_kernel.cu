// attn_kernel.cu -- block-sparse flash-attention forward with Horvitz-Thompson block
// weights on sm_100a (AB-Attention news page, section «Три приёма AB-Attention»: each
// sampled block counts with weight 1/p in the numerator and the softmax normaliser,
// which keeps the computation ordinary softmax attention with a logit shift; the
// kernel gathers the chosen key/value blocks by index, tokens stay in order).
//
// One persistent CTA per SM works through (b, h, query block) items, claimed one at a
// time from a global counter in head-major order (see the item scheduler below), so the
// CTAs running at any time share a head's K/V in L2 and finish together. Per CTA, 352
// threads (384 for 4-token units) in four roles:
//   warps 0-7  softmax: warps q and q+4 own query rows 32q..32q+31 (TMEM lanes), warp
//              q the first 64 key columns of each S row and warp q+4 the last 64; the
//              online softmax runs in the log2 domain with the block's log2(w) added,
//              writes P (bf16) back over S and lazily rescales O. Key blocks: the two
//              warps exchange each block's row max and share one O; 4-token units: each
//              warp keeps its own max, sum and O accumulator and the two merge once per
//              item. Each warp normalises and stores half of every output row;
//   warp 8     TMA producer: Q tile and a ring of K / V tiles
//              fetched by block index with 3-D tensor maps whose row extent is N, so
//              rows past the sequence end arrive as zeros (units: warps 8 and 10 gather
//              the tiles with cp.async);
//   warp 9     TMEM owner and MMA issuer: S = Q K^T (both operands from shared
//              memory) into S buffer g mod kSB, O (+)= P V with P read from TMEM (units:
//              O_h += P_h V_h for the two key halves h);
//   warp 10    item scheduler (warp 11 for units): claims the items and publishes them
//              to the other roles through a ring in shared memory.
// TMEM: kSB S buffers of 128 columns, then the O accumulator(s) (d fp32 columns each):
// 3 S buffers and one O for key blocks; O_0 and O_1 for units, with 2 S buffers at
// d = 128. Issue order of the MMA warp over the CTA's block stream:
//   S(0), .., S(kSB - 1), PV(0), S(kSB), PV(1), ...  S runs kSB blocks ahead, so the
// softmax never waits for a QK^T product, and nothing in the softmax waits for a PV
// product except an O rescale (PV(g-1)) and the end of an item (PV(g)).
// Every wait is bounded (2 s); on a timeout the roles unwind, drain their own
// asynchronous work and the CTA frees its TMEM before returning.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ab_device.cuh"
#include "ab_kernels.h"
#include "tmap_host.h"

namespace ab {

constexpr int kWarpTma = 8, kWarpMma = 9;
// 4-token units: a second gather warp (on another SM sub-partition) copies half of every
// K and V tile: warp 8 units 0..15, warp 10 units 16..31; warp 8 also loads Q
constexpr int kWarpGather2 = 10;
// the item scheduler: warp 10 (key blocks) or 11 (units)
constexpr int sched_warp(bool units) { return units ? 11 : 10; }
constexpr int attn_threads(bool units) { return (sched_warp(units) + 1) * 32; }
constexpr int kTmemCols = 512;
constexpr int kSBufsMax = 3;
constexpr int kRing = 16;  // work items published ahead to the roles (more than any role's lead)
// TMEM columns: S / P buffers (128 b .. 128 b + 127), then the O accumulator(s) of D
// fp32 columns each. Shared softmax rows (blocks): 3 S buffers and one O. Split halves
// (4-token units): O_0 and O_1 (O_h at kColO + h D), with 2 S buffers for D = 128.
template <int D, bool kSplit>
struct TmemPlan {
    static constexpr int kSBufs = (kSplit && D == 128) ? 2 : 3;
    static constexpr int kColO = kSBufs * 128;
    static_assert(kColO + (kSplit ? 2 : 1) * D <= kTmemCols, "TMEM plan exceeds 512 columns");
};
constexpr float kRescaleThreshold = 20.0f;  // log2 units: P stays <= 2^20 without a rescale (bf16 P and fp32 l / O hold that with room to spare)

struct AttnParams {
    const int32_t *idx;
    const int32_t *cnt;
    const float *w;  // nullptr: all weights 1 (top-k)
    void *out;       // bf16 or fp32 [B*H, N_pad, D]
    float *lse;
    int *flag;
    const __nv_bfloat16 *kg, *vg;  // K, V in global memory (4-token units: gathered per unit)
    int H, N, N_pad, nqb;
    int nkb;       // entries per idx / w row: key blocks (N_pad / 128) or key units (N_pad / 4)
    int per_tile;  // selected entries per 128-key tile: 1 (blocks) or 32 (units)
    int n_items;
    float scale_log2;       // log2(e) / sqrt(d)
    unsigned int *counter;  // claim slot [4]: items claimed, owner tag (zeroed on the
                            // launch's stream just before the kernel)
    unsigned int tag;       // this launch's owner tag (never 0 or kSlotPoison)
    unsigned long long wait_ns;  // limit of every bounded wait (kWaitLimitNs; shorter in tests)
};

// A claim slot is zeroed on the launch's stream right before the kernel; the first CTA
// to arrive writes the launch's tag into it. A CTA that finds another tag (or, at a
// claim or at its exit, a slot that no longer carries its tag) knows that a second
// launch is using the same slot at the same time: it raises AB_FLAG_SCHED_COLLISION and
// poisons the slot, so that the other launch finds out too.
constexpr unsigned kSlotPoison = 0xFFFFFFFFu;

__device__ __forceinline__ void slot_collision(const AttnParams &p)
{
    raise_flag(p.flag, AB_FLAG_SCHED_COLLISION);
    atomicExch(p.counter + 1, kSlotPoison);
}

__device__ __forceinline__ void slot_join(const AttnParams &p)
{
    const unsigned old = atomicCAS(p.counter + 1, 0u, p.tag);
    if (old != 0u && old != p.tag) slot_collision(p);
}

__device__ __forceinline__ void slot_check(const AttnParams &p)
{
    __threadfence();
    if (atomicOr(p.counter + 1, 0u) != p.tag) slot_collision(p);
}

// 4-token key units: one 16-byte cp.async per lane (zero fill when src_bytes == 0) and
// an arrive on an mbarrier when this thread's earlier cp.async copies have landed.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Shared memory of one attention CTA: one Q tile and a ring of 5 K/V tiles (d = 128; 9 at
// d = 64). Items hold many tiles, so a deeper K/V prefetch is worth more than loading the
// next item's Q during the current one (a second Q buffer in place of a ring stage was
// 1-2% slower on the 262k-token, 720p and Wan2.1-1.3B shapes).
template <int D, bool kUnits>
struct AttnSmem {
    static constexpr int kTileBytes = 128 * D * 2;  // one 128-row bf16 tile
    static constexpr int kBoxes = D / 64;           // 64-column (128-byte) TMA boxes per tile
    static constexpr int kQBufs = 1;
    static constexpr int kStages = D == 128 ? 5 : 9;
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = kQBufs * kTileBytes;
    static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
    // barriers: q_full[2], q_empty[2], kv_full[S], kv_empty[S], s_full[3], p_full[2][3],
    // o_full[2][3], drain, ring_full[R], ring_empty[R], started
    static constexpr int kNumBars = 2 + 2 + kStages + kStages + 5 * kSBufsMax + 1 + 2 * kRing + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    // softmax exchange: float row max [2 blocks][2 halves][128], m [2][128], l [2][128]
    static constexpr int kXchOff = kMiscOff + 16;
    static constexpr int kRingOff = kXchOff + (2 * 2 * 128 + 2 * 128 + 2 * 128) * 4;  // int [R][2]
    static constexpr int kItemXchOff = kRingOff + kRing * 8;  // softmax pairs: int [2][2][4]
    static constexpr int kBytes = kItemXchOff + 2 * 2 * 4 * 4;
    static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 B
};

// Work items are handed out dynamically. A scheduler warp per CTA takes the CTA's first
// item c = blockIdx.x and then claims each further item from a global counter (r =
// gridDim.x + the counter's old value; r >= n_items ends the CTA's stream), one item
// ahead of the CTA's K loads: claim t + 1 waits until the TMA warp has started item t.
// It writes the output of an empty item itself (O = 0, lse = -inf) and publishes the
// others in a ring of kRing entries in shared memory, from which every role reads the
// CTA's item sequence, so all roles walk the same items in the same order. A CTA takes
// a new item only when it is nearly done with the last, so the CTAs finish together
// however unevenly the selected blocks are spread over the items (a fixed assignment of
// items c, c + grid, ... leaves the CTAs whose items hold the most blocks running last).
// Claims follow the natural head-major order, so the CTAs running at any time still work
// on neighbouring items and share a head's K/V in L2.
struct ItemRing {
    volatile int *items;     // [kRing][2]: item t of the sequence and its clamped entry count,
                             // in entry t mod kRing
    uint64_t *full, *empty;  // [kRing] each: entry published; entry read by every reader
    uint64_t *started;       // one phase per item the TMA warp's K loads enter (t >= 1)
    volatile int *abort;
    int *flag;
    unsigned long long wait_ns;
};

// Item t of the sequence and its entry count once published; one arrive per reading warp
// releases the entry. False (and r = n_items) when the wait failed (timeout or abort).
__device__ __forceinline__ bool ring_read(const ItemRing &q, int n_items, int t, int &r, int &cnt)
{
    const int slot = t % kRing;
    r = n_items;
    cnt = 0;
    if (!__all_sync(0xffffffffu, mbar_wait(&q.full[slot], (t / kRing) & 1, q.abort, q.flag, q.wait_ns)))
        return false;
    r = q.items[2 * slot];
    cnt = q.items[2 * slot + 1];
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&q.empty[slot]);
    return true;
}

// One role's walk over the CTA's (item, tile) stream.
struct Cursor {
    int r;    // work item (flat (b*H + h)*nqb + qb); >= n_items when done
    int i;    // tile position within the item
    int n;    // tiles of the item: cnt / per_tile, rounded up
    int seq;  // index of the item among this CTA's items
    int cnt;  // selected entries of item r, clamped to [0, nkb]
    int t;    // position of item r in the CTA's item sequence
};

// Read item t of the sequence into the cursor. `lead`: the TMA warp's K cursor, which
// tells the scheduler each time it starts an item (the scheduler then claims the next).
__device__ __forceinline__ bool cursor_load(Cursor &c, const AttnParams &p, const ItemRing &q, bool lead)
{
    const bool ok = ring_read(q, p.n_items, c.t, c.r, c.cnt);
    c.n = (c.cnt + p.per_tile - 1) / p.per_tile;
    c.i = 0;
    if (lead && c.t >= 1 && c.r < p.n_items) {
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(q.started);
    }
    return ok;
}

// Move past finished items.
__device__ __forceinline__ bool cursor_seek(Cursor &c, const AttnParams &p, const ItemRing &q,
                                            bool lead)
{
    while (c.r < p.n_items && c.i >= c.n) {
        if (c.n > 0) ++c.seq;
        ++c.t;
        if (!cursor_load(c, p, q, lead)) return false;
    }
    return true;
}

__device__ __forceinline__ bool cursor_first(Cursor &c, const AttnParams &p, const ItemRing &q,
                                             bool lead)
{
    c.seq = 0;
    c.t = 0;
    return cursor_load(c, p, q, lead) && cursor_seek(c, p, q, lead);
}

__device__ __forceinline__ bool cursor_next(Cursor &c, const AttnParams &p, const ItemRing &q, bool lead)
{
    ++c.i;
    return cursor_seek(c, p, q, lead);
}

__device__ __forceinline__ int block_index(const AttnParams &p, int r, int i, bool report)
{
    int j = __ldg(p.idx + (size_t)r * p.nkb + i);
    if (j < 0 || j >= p.nkb) {
        if (report) raise_flag(p.flag, AB_FLAG_BAD_INDEX);
        j = j < 0 ? 0 : p.nkb - 1;
    }
    return j;
}

template <int D, bool kWeighted, bool kOutF32, bool kUnits>
__global__ void __launch_bounds__(attn_threads(kUnits), 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p)
{
    using L = AttnSmem<D, kUnits>;
    // 4-token units: the two softmax halves of a row keep separate maxima and O
    // accumulators (their per-unit masks and weights make the shared-max exchange the
    // longer path); blocks: one shared row max per block and one O
    constexpr bool kSplit = kUnits;
    constexpr int kSB = TmemPlan<D, kSplit>::kSBufs;
    constexpr int kColO = TmemPlan<D, kSplit>::kColO;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
    uint64_t *q_full = bars;
    uint64_t *q_empty = bars + 2;
    uint64_t *kv_full = bars + 4;
    uint64_t *kv_empty = kv_full + L::kStages;
    uint64_t *s_full = kv_empty + L::kStages;
    uint64_t *p_full = s_full + kSBufsMax;  // [h][b]: P_h of the block in S buffer b is in TMEM
    uint64_t *o_full = p_full + 2 * kSBufsMax;  // [h][b]: PV_h of that block is complete
    uint64_t *drain = o_full + 2 * kSBufsMax;
    uint64_t *ring_full = drain + 1, *ring_empty = ring_full + kRing, *started = ring_empty + kRing;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    ItemRing iq;
    iq.items = reinterpret_cast<volatile int *>(smem + L::kRingOff);
    iq.full = ring_full;
    iq.empty = ring_empty;
    iq.started = started;
    iq.abort = abort_flag;
    iq.flag = p.flag;
    iq.wait_ns = p.wait_ns;
    // readers of every ring entry, one arrive each: the K and V cursors of warp 8 (and of
    // warp 10 for units), the S and PV cursors of the MMA warp, the 8 softmax warps
    constexpr int kRingReaders = 2 + (kUnits ? 2 : 0) + 2 + 8;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], 1);
            mbar_init(&q_empty[b], 1);
        }
        for (int b = 0; b < kSB; ++b) {
            mbar_init(&s_full[b], 1);
            for (int h = 0; h < (kSplit ? 2 : 1); ++h) {
                mbar_init(&p_full[h * kSBufsMax + b], kSplit ? 128 : 256);
                mbar_init(&o_full[h * kSBufsMax + b], 1);
            }
        }
        for (int s = 0; s < L::kStages; ++s) {
            // TMA: one arrive with the tile's byte count; units: one cp.async arrive per
            // lane of the two gather warps
            mbar_init(&kv_full[s], kUnits ? 64 : 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(drain, 1);
        for (int e = 0; e < kRing; ++e) {
            mbar_init(&ring_full[e], 1);
            mbar_init(&ring_empty[e], kRingReaders);
        }
        mbar_init(started, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kWarpTma || (kUnits && warp == kWarpGather2)) {
        // ------------------------------ TMA producer ------------------------------
        // 4-token units: warps 8 and 10 both walk every ring position in order (so each
        // warp's stage waits stay within one phase) and each copies its half of the
        // tile's units; only warp 8 loads Q.
        const bool do_q = warp == kWarpTma;
        const int unit_half = warp == kWarpTma ? 0 : 1;
        // The whole warp runs the control flow (warp-uniform values); one elected lane
        // issues each copy.
        if (elect_one() && do_q) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
        }
        __syncwarp();
        int kv_pos = 0;
        int q_loads = 0;
        bool ok = true;
        auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.flag, p.wait_ns));
        };
        auto load_q = [&](const Cursor &c) -> bool {
            if (!do_q) return true;
            const int b = c.seq % L::kQBufs;
            if (!wait(&q_empty[b], ((c.seq / L::kQBufs) & 1) ^ 1)) return false;
            uint8_t *dst = smem + L::kQOff + b * L::kTileBytes;
            const int bh = c.r / p.nqb, qb = c.r % p.nqb;
            if (elect_one()) {
                mbar_arrive_expect_tx(&q_full[b], L::kTileBytes);
#pragma unroll
                for (int x = 0; x < L::kBoxes; ++x)
                    tma_load_3d(dst + x * 16384, &tmQ, &q_full[b], x * 64, qb * 128, bh);
            }
            __syncwarp();
            ++q_loads;
            return true;
        };
        auto load_kv = [&](const Cursor &c, const CUtensorMap *tm) -> bool {
            const int s = kv_pos % L::kStages;
            if (!wait(&kv_empty[s], ((kv_pos / L::kStages) & 1) ^ 1)) return false;
            if constexpr (kUnits) {
                // gather 32 units of 4 key rows into tile rows 4 s' .. 4 s' + 3, in the
                // 128-byte-swizzled layout the MMA descriptors read; this warp copies its
                // 16 units, one warp instruction per unit and 64-column box (lane = row rr,
                // 16-byte chunk c8). The loop over the units is unrolled by eight: the
                // fastest of the unroll factors measured (8: 0.90x the time of 4, 16:
                // 1.02x, 2: 1.22x, 1: 1.40x), so each unit's destination (tile row
                // 64 half + 4 k + rr, swizzle phase rr + 4 (k mod 2)) is a per-lane base
                // plus a small offset: per unit one shuffle, one address and one validity
                // test before the copies.
                const int cnt = c.cnt;
                const int slot = c.i * 32 + unit_half * 16 + (lane & 15);
                int u = -1;
                if (slot < cnt) {
                    u = __ldg(p.idx + (size_t)c.r * p.nkb + slot);
                    if (u < 0 || u >= p.nkb) {
                        if (tm == &tmK && lane < 16) raise_flag(p.flag, AB_FLAG_BAD_INDEX);
                        u = -1;
                    }
                }
                const int rr = lane >> 3, c8 = lane & 7;
                const char *src = reinterpret_cast<const char *>(tm == &tmK ? p.kg : p.vg) +
                                  ((size_t)(c.r / p.nqb) * p.N_pad + rr) * (D * 2) + c8 * 16;
                const uint32_t dst = smem_u32(smem + L::kKVOff + s * L::kTileBytes) +
                                     (uint32_t)(unit_half * 64 + rr) * 128;
                const uint32_t sw_even = (uint32_t)(c8 ^ rr) << 4, sw_odd = (uint32_t)(c8 ^ (rr + 4)) << 4;
                const int rows_left = p.N - rr;  // unit us holds a valid row here iff 4 us < rows_left
#pragma unroll 8
                for (int k = 0; k < 16; ++k) {
                    const int us = __shfl_sync(0xffffffffu, u, k);
                    const bool valid = us >= 0 && us * 4 < rows_left;
                    const char *g = src + (size_t)(valid ? us : 0) * (4 * D * 2);
                    const uint32_t d0 = dst + k * 512 + ((k & 1) ? sw_odd : sw_even);
                    const uint32_t nbytes = valid ? 16u : 0u;
#pragma unroll
                    for (int h = 0; h < L::kBoxes; ++h) cp_async_16(d0 + h * 16384, g + h * 128, nbytes);
                }
                cp_async_arrive_noinc(&kv_full[s]);
                ++kv_pos;
                return true;
            }
            const int j = block_index(p, c.r, c.i, tm == &tmK && lane == 0);
            uint8_t *dst = smem + L::kKVOff + s * L::kTileBytes;
            const int bh = c.r / p.nqb;
            if (elect_one()) {
                mbar_arrive_expect_tx(&kv_full[s], L::kTileBytes);
#pragma unroll
                for (int x = 0; x < L::kBoxes; ++x)
                    tma_load_3d(dst + x * 16384, tm, &kv_full[s], x * 64, j * 128, bh);
            }
            __syncwarp();
            ++kv_pos;
            return true;
        };
        // tile order = the MMA warp's consumption order: K of the first kSB blocks,
        // then V(g), K(g + kSB), V(g + 1), ...; a Q tile precedes its item's first K
        // warp 8's K cursor tells the scheduler when it starts an item
        Cursor kc, vc;
        ok = cursor_first(kc, p, iq, warp == kWarpTma);
        ok = cursor_first(vc, p, iq, false) && ok;
        auto next_k = [&]() -> bool {
            bool r = true;
            if (kc.i == 0) r = load_q(kc);
            r = r && load_kv(kc, &tmK);
            return cursor_next(kc, p, iq, warp == kWarpTma) && r;
        };
        for (int a = 0; a < kSB && ok && kc.r < p.n_items; ++a) ok = next_k();
        while (ok && vc.r < p.n_items) {
            ok = load_kv(vc, &tmV);
            ok = cursor_next(vc, p, iq, false) && ok;
            if (ok && kc.r < p.n_items) ok = next_k();
        }
        if (!ok) {
            // drain: the last loads issued may still be in flight
            for (int k = kv_pos - L::kStages; k < kv_pos; ++k)
                if (k >= 0) drain_wait(&kv_full[k % L::kStages], (k / L::kStages) & 1);
            for (int k = q_loads - L::kQBufs; k < q_loads; ++k)
                if (k >= 0) drain_wait(&q_full[k % L::kQBufs], (k / L::kQBufs) & 1);
        }
    } else if (warp == kWarpMma) {
        // ------------------------------- MMA issuer -------------------------------
        // The whole warp runs the control flow, so descriptors and addresses are
        // warp-uniform values; one elected lane issues each tcgen05.mma / commit.
        // Per MMA only a constant is added to a precomputed descriptor's start-address
        // field (addresses stay below 256 KB, so the 14-bit field never carries): a
        // lean issue path lets one thread keep up with the tensor core.
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
        constexpr uint64_t kTileDesc = L::kTileBytes >> 4;
        const uint64_t q_desc0 = smem_desc_sw128(smem_u32(smem + L::kQOff), 16, 1024);
        const uint64_t k_desc0 = smem_desc_sw128(smem_u32(smem + L::kKVOff), 16, 1024);
        const uint64_t v_desc0 = smem_desc_sw128(smem_u32(smem + L::kKVOff), 16384, 1024);
        int kv_pos = 0;
        bool ok = true;
        auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.flag, p.wait_ns));
        };
        auto issue_s = [&](const Cursor &c, int g) -> bool {
            const int qbuf = c.seq % L::kQBufs;
            if (c.i == 0 && !wait(&q_full[qbuf], (c.seq / L::kQBufs) & 1)) return false;
            const int s = kv_pos % L::kStages;
            if (!wait(&kv_full[s], (kv_pos / L::kStages) & 1)) return false;
            if constexpr (kUnits) fence_proxy_async_smem();  // tile written by cp.async
            tc_fence_after();
            const uint64_t qd = q_desc0 + (uint64_t)qbuf * kTileDesc;
            const uint64_t kd = k_desc0 + (uint64_t)s * kTileDesc;
            const uint32_t d_tmem = tmem + (g % kSB) * 128;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                    mma_ss(d_tmem, qd + off, kd + off, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[g % kSB]);
                mma_commit(&kv_empty[s]);
                if (c.i == c.n - 1) mma_commit(&q_empty[qbuf]);
            }
            __syncwarp();
            ++kv_pos;
            return true;
        };
        Cursor sc, pc;  // next S to issue, next PV to issue
        ok = cursor_first(sc, p, iq, false);
        ok = cursor_first(pc, p, iq, false) && ok;
        int gs = 0;  // index of the next S
        for (int a = 0; a < kSB && ok && sc.r < p.n_items; ++a) {
            ok = issue_s(sc, gs++);
            ok = cursor_next(sc, p, iq, false) && ok;
        }
        for (int g = 0; ok && pc.r < p.n_items; ++g) {
            const int b = g % kSB;
            const uint32_t par = (g / kSB) & 1;
            const bool first = pc.i == 0;
            const uint32_t p_tmem = tmem + b * 128;
            const uint32_t acc0 = first ? 0u : 1u;
            if constexpr (!kSplit) {
                // O (+)= P(g) V(g)
                if (!wait(&p_full[b], par)) {
                    ok = false;
                    break;
                }
                const int s = kv_pos % L::kStages;
                if (!wait(&kv_full[s], (kv_pos / L::kStages) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t vd = v_desc0 + (uint64_t)s * kTileDesc;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 128 / 16; ++kk)
                        mma_ts(tmem + kColO, p_tmem + kk * 8, vd + (uint64_t)(kk * (2048 >> 4)),
                               idesc_pv, kk > 0 ? 1u : acc0);
                    mma_commit(&kv_empty[s]);
                    mma_commit(&o_full[b]);
                }
                __syncwarp();
            } else {
                // O_h (+)= P_h(g) V_h(g), h = 0, 1: the block's keys 64 h .. 64 h + 63 (P_h
                // in TMEM columns 64 h .. 64 h + 31 of S buffer g mod kSB, V_h = V tile
                // rows 64 h ..). An item's first PVs overwrite O_0 and O_1, which both
                // softmax halves read in the previous item's epilogue: they wait for both
                // P halves.
                if ((first && !wait(&p_full[kSBufsMax + b], par)) || !wait(&p_full[b], par)) {
                    ok = false;
                    break;
                }
                const int s = kv_pos % L::kStages;
                if (!wait(&kv_full[s], (kv_pos / L::kStages) & 1)) {
                    ok = false;
                    break;
                }
                if constexpr (kUnits) fence_proxy_async_smem();  // tile written by cp.async
                tc_fence_after();
                const uint64_t vd = v_desc0 + (uint64_t)s * kTileDesc;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tmem + kColO, p_tmem + kk * 8, vd + (uint64_t)(kk * (2048 >> 4)),
                               idesc_pv, kk > 0 ? 1u : acc0);
                    mma_commit(&o_full[b]);
                }
                __syncwarp();
                if (!first && !wait(&p_full[kSBufsMax + b], par)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tmem + kColO + D, p_tmem + 64 + kk * 8,
                               vd + (uint64_t)((4 + kk) * (2048 >> 4)), idesc_pv, kk > 0 ? 1u : acc0);
                    mma_commit(&kv_empty[s]);
                    mma_commit(&o_full[kSBufsMax + b]);
                }
                __syncwarp();
            }
            ++kv_pos;
            ok = cursor_next(pc, p, iq, false);
            // S(g + kSB) reuses the buffer whose P(g) was just consumed (in order)
            if (ok && sc.r < p.n_items) {
                ok = issue_s(sc, gs++);
                ok = cursor_next(sc, p, iq, false) && ok;
            }
        }
        if (!ok) {
            if (elect_one()) {
                mma_commit(drain);
                drain_wait(drain, 0);
            }
            __syncwarp();
        }
    } else if (warp == sched_warp(kUnits)) {
        // ------------------------------ item scheduler ----------------------------
        // Entry 0: the CTA's first item; entry t >= 2 once the K loads have entered item
        // t - 1; empty items get their output here (O = 0; lse = -inf, 0 on padding rows)
        // and are not published. Its waits sleep between polls: it shares an SM
        // sub-partition with two softmax warps.
        bool ok = true;
        if (lane == 0) slot_join(p);
        auto claim = [&]() -> int {
            int c = 0;
            if (lane == 0) {
                c = (int)min(atomicAdd(p.counter, 1u), (unsigned)p.n_items);
                slot_check(p);
            }
            c = __shfl_sync(0xffffffffu, c, 0);
            return min((int)gridDim.x + c, p.n_items);
        };
        auto write_empty = [&](int r) {
            const int bh = r / p.nqb, qb = r % p.nqb;
            constexpr int kVecs = D * (kOutF32 ? 4 : 2) / 16;  // uint4 per output row
            for (int rr = lane; rr < 128; rr += 32) {
                const int tok = qb * 128 + rr;
                const size_t off = ((size_t)bh * p.N_pad + tok) * D;
                uint4 *o4 = kOutF32 ? reinterpret_cast<uint4 *>(static_cast<float *>(p.out) + off)
                                    : reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) + off);
#pragma unroll 4
                for (int e = 0; e < kVecs; ++e) o4[e] = make_uint4(0, 0, 0, 0);
                if (p.lse) p.lse[(size_t)bh * p.N_pad + tok] = tok < p.N ? -INFINITY : 0.f;
            }
        };
        int r = blockIdx.x < (unsigned)p.n_items ? (int)blockIdx.x : p.n_items;
        for (int t = 0; ok; ++t) {
            if (t >= 2) ok = __all_sync(0xffffffffu, mbar_wait_sleepy(started, (t - 2) & 1, abort_flag, p.flag, 500, p.wait_ns));
            if (!ok) break;
            if (t > 0) r = claim();
            int c_raw = 0;
            while (r < p.n_items) {
                c_raw = __ldg(p.cnt + r);
                if ((c_raw < 0 || c_raw > p.nkb) && lane == 0) raise_flag(p.flag, AB_FLAG_BAD_INDEX);
                if (c_raw > 0) break;
                write_empty(r);
                r = claim();
            }
            // entry t once every reader has read its previous use
            const int slot = t % kRing;
            if (t >= kRing &&
                !__all_sync(0xffffffffu, mbar_wait_sleepy(&ring_empty[slot], ((t / kRing) - 1) & 1, abort_flag, p.flag, 500, p.wait_ns)))
                break;
            if (lane == 0) {
                iq.items[2 * slot] = r;
                iq.items[2 * slot + 1] = r < p.n_items ? min(c_raw, p.nkb) : 0;
                mbar_arrive(&ring_full[slot]);  // release: the entry is visible to a reader's acquire
            }
            __syncwarp();
            if (r >= p.n_items) break;
        }
    } else {
        // -------------------------------- softmax ---------------------------------
        // Warps q and q + 4 share TMEM lanes 32q..32q+31 (query rows); warp q (half
        // h = 0) takes S columns 0..63 of each block, warp q + 4 (h = 1) columns 64..127.
        // Shared rows (blocks): the two exchange their block row max through shared
        // memory across a 64-thread named barrier and run one online softmax into one O;
        // warp q + 4 writes P into columns 32..63, which warp q reads as S, only after
        // that barrier. Split halves (units): each warp runs its own online softmax over
        // its columns (running max m_h, sum l_h) into its own accumulator O_h += P_h V_h,
        // writing P_h over its own S columns 64 h .. 64 h + 31, so the two never wait for
        // each other inside an item; at the end of an item they exchange (m, l) once and
        // each writes half of the output columns from both accumulators:
        //   O = (O_0 2^(m_0 - m) + O_1 2^(m_1 - m)) / (l_0 2^(m_0 - m) + l_1 2^(m_1 - m)),
        //   m = max(m_0, m_1).
        // These warps never leave their loops early: after a failed (timed-out) wait
        // they skip the remaining waits but keep the same sequence of named barriers,
        // so a pair can never be left waiting for its partner.
        const int quad = warp & 3, half = warp >> 2;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t col_o_own = kColO + (kSplit ? half * D : half * (D / 2));
        const uint32_t col_o_oth = kColO + (half ^ 1) * D;  // split halves only
        float *xmax_sh = reinterpret_cast<float *>(smem + L::kXchOff);  // [2][2][128]
        float *xm_sh = xmax_sh + 2 * 2 * 128;                            // [2][128]
        float *xl_sh = xm_sh + 2 * 128;                                  // [2][128]
        const int hb = kSplit ? half * kSBufsMax : 0;
        uint64_t *p_own = p_full + hb;
        uint64_t *o_own = o_full + hb, *o_oth = o_full + (half ^ 1) * kSBufsMax;
        auto pair_sync = [&]() {
            tc_fence_before();
            asm volatile("bar.sync %0, 64;" ::"r"(1 + quad) : "memory");
            tc_fence_after();
        };
        int g = 0;
        int o_seen = 0, o_seen_oth = 0;  // PV_h completions observed so far (own, other half)
        bool ok = true;
        auto wait_bar = [&](uint64_t *bar, uint32_t parity) {
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.flag, p.wait_ns));
        };
        // wait until PV_h(k) is complete (own half: k = g - 1 for a rescale; both halves:
        // k = g at the end of an item). PV_h(k) completes phase k / kSB of o_full[h][k mod
        // kSB]. A parity wait is exact only within one phase of the barrier's state:
        // PV_h(k - kSB) is complete (S(g) was issued after it and has completed), and
        // PV_h(k + kSB) cannot complete first: for the own half it needs P_h(k + kSB),
        // which this warp has not written; for the other half at the end of an item it
        // comes after the next item's first PV, which waits for this warp's next P.
        auto wait_o = [&](int k) {
            if (o_seen > k) return;
            wait_bar(&o_own[k % kSB], (k / kSB) & 1);
            o_seen = k + 1;
        };
        auto wait_o_oth = [&](int k) {
            if (o_seen_oth > k) return;
            wait_bar(&o_oth[k % kSB], (k / kSB) & 1);
            o_seen_oth = k + 1;
        };
        auto lw_of = [&](float wj) -> float {  // log2 of a block weight (0 for top-k)
            if (!kWeighted) return 0.f;
            if (wj > 0.f && wj < INFINITY) return fast_log2(wj);
            if (warp == 0 && lane == 0) raise_flag(p.flag, AB_FLAG_BAD_WEIGHT);
            return 0.f;
        };
        auto clamp_j = [&](int j) { return j < 0 ? 0 : (j >= p.nkb ? p.nkb - 1 : j); };
        constexpr int kHalfD = D / 2;
        // pairs e with e % 5 == 4 (6 of 32 per block) take the FMA-pipe exp2, spread through
        // the loop so that FMA-pipe and MUFU work interleave
        constexpr int kSoftEvery = 5;
        const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
        // Item t of the CTA's sequence from the ring. The two warps of a pair take the
        // smaller of their two reads (n_items after a failed wait), so they always walk
        // the same items and meet at the same named barriers.
        int *item_xch = reinterpret_cast<int *>(smem + L::kItemXchOff);  // [2 parities][2][4]
        int t_item = 0, cnt_item = 0;
        auto next_item = [&]() -> int {
            int r2;
            ring_read(iq, p.n_items, t_item, r2, cnt_item);
            item_xch[((t_item & 1) * 2 + half) * 4 + quad] = r2;
            pair_sync();
            r2 = min(r2, item_xch[((t_item & 1) * 2 + (half ^ 1)) * 4 + quad]);
            ++t_item;
            return r2;
        };
        for (int r = next_item(); r < p.n_items; r = next_item()) {
            const int cnt_r = cnt_item;
            const int n = kUnits ? (cnt_r + 31) / 32 : cnt_r;  // 128-key tiles of this item
            const int bh = r / p.nqb, qb = r % p.nqb;
            const int tok = qb * 128 + row;
            const size_t orow_off = ((size_t)bh * p.N_pad + tok) * D + half * kHalfD;
            // this thread's half output row: D/2 bf16 (D/16 uint4) or D/2 fp32 (D/8 uint4)
            uint4 *o4 = kOutF32 ? reinterpret_cast<uint4 *>(static_cast<float *>(p.out) + orow_off)
                                : reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) + orow_off);
            constexpr int kRowVecs = kOutF32 ? kHalfD / 4 : kHalfD / 8;
            if (n == 0) {
#pragma unroll
                for (int e = 0; e < kRowVecs; ++e) o4[e] = make_uint4(0, 0, 0, 0);
                if (p.lse && half == 0) p.lse[(size_t)bh * p.N_pad + tok] = tok < p.N ? -INFINITY : 0.f;
                continue;
            }
            const int32_t *idx_row = p.idx + (size_t)r * p.nkb;
            const float *w_row = kWeighted ? p.w + (size_t)r * p.nkb : nullptr;
            // blocks: index and weight are loaded two blocks ahead; the next block's log2
            // weight is taken right after this block's max exchange, while the MUFU unit
            // is free of exp2 work.
            // units: lane l < 16 of each warp holds unit slot 32 i + 16 half + l of tile i
            // (this warp's 64 columns = 16 units); its log2 weight (-inf for an empty
            // slot) and valid-token count reach the other lanes by shuffles.
            int j = 0;
            float lw = 0.f;
            int j_n1 = 0;
            float w_n1 = 1.f;
            auto unit_of = [&](int t, int &u, float &wv) {
                const int slot = t * 32 + half * 16 + (lane & 15);
                u = -1;
                wv = 1.f;
                if (lane < 16 && slot < cnt_r) {
                    const int x = __ldg(idx_row + slot);
                    if (x >= 0 && x < p.nkb) {
                        u = x;
                        if (kWeighted) wv = __ldg(w_row + slot);
                    }
                }
            };
            auto unit_lw = [&](int u, float wv, int &nv) -> float {
                nv = u >= 0 ? max(0, min(4, p.N - 4 * u)) : 0;
                if (nv == 0) return -INFINITY;
                if (!kWeighted) return 0.f;
                if (wv > 0.f && wv < INFINITY) return fast_log2(wv);
                raise_flag(p.flag, AB_FLAG_BAD_WEIGHT);
                return 0.f;
            };
            int nv_l = 0, nv_n = 0;  // units: valid tokens of this lane's slot (tile i, i + 1)
            if constexpr (kUnits) {
                int u;
                float wv;
                unit_of(0, u, wv);
                lw = unit_lw(u, wv, nv_l);
                if (n > 1) unit_of(1, j_n1, w_n1);
            } else {
                j = clamp_j(__ldg(idx_row));
                lw = lw_of(kWeighted ? __ldg(w_row) : 1.f);
                if (n > 1) {
                    j_n1 = __ldg(idx_row + 1);
                    if (kWeighted) w_n1 = __ldg(w_row + 1);
                }
            }
            float m_run = -INFINITY, l_run = 0.f;
            for (int i = 0; i < n; ++i, ++g) {
                int j_n2 = 0;
                float w_n2 = 1.f;
                if (i + 2 < n) {
                    if constexpr (kUnits) {
                        unit_of(i + 2, j_n2, w_n2);
                    } else {
                        j_n2 = __ldg(idx_row + i + 2);
                        if (kWeighted) w_n2 = __ldg(w_row + i + 2);
                    }
                }
                const int nvalid = min(128, p.N - j * 128) - half * 64;  // blocks: valid columns here
                const uint32_t s_col = (g % kSB) * 128;
                wait_bar(&s_full[g % kSB], (g / kSB) & 1);
                tc_fence_after();
                // the destination registers are only read after tcgen05.wait::ld
                uint32_t su[64];
                tmem_ld32(tmem + lane_off + s_col + half * 64,
                          *reinterpret_cast<uint32_t(*)[32]>(&su[0]));
                tmem_ld32(tmem + lane_off + s_col + half * 64 + 32,
                          *reinterpret_cast<uint32_t(*)[32]>(&su[32]));
                tmem_wait_ld();
                float sv[64];
#pragma unroll
                for (int e = 0; e < 64; ++e) sv[e] = __uint_as_float(su[e]);
                if constexpr (kUnits) {
                    // x = s * scale_log2 + log2 w of the column's unit (-inf: empty slot
                    // or a token past the sequence end)
                    float lwu[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) lwu[k] = __shfl_sync(0xffffffffu, lw, k);
#pragma unroll
                    for (int e = 0; e < 64; ++e) sv[e] = fmaf(sv[e], p.scale_log2, lwu[e >> 2]);
                    if (__any_sync(0xffffffffu, nv_l > 0 && nv_l < 4)) {
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const int nvk = __shfl_sync(0xffffffffu, nv_l, k);
#pragma unroll
                            for (int t = 0; t < 4; ++t)
                                if (t >= nvk) sv[4 * k + t] = -INFINITY;
                        }
                    }
                } else if (nvalid < 64) {
#pragma unroll
                    for (int e = 0; e < 64; ++e)
                        if (e >= nvalid) sv[e] = -INFINITY;
                }
                // this half's row max: 8 independent chains of three-input max, then a tree;
                // shared rows exchange theirs
                float mx[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    mx[t] = fmax3(sv[t], sv[8 + t], sv[16 + t]);
                    mx[t] = fmax3(mx[t], sv[24 + t], sv[32 + t]);
                    mx[t] = fmax3(mx[t], sv[40 + t], sv[48 + t]);
                    mx[t] = fmaxf(mx[t], sv[56 + t]);
                }
                mx[0] = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                              fmaxf(mx[6], mx[7]));
                float smax = mx[0];
                if constexpr (!kSplit) {
                    xmax_sh[((g & 1) * 2 + half) * 128 + row] = mx[0];
                    pair_sync();
                    smax = fmaxf(mx[0], xmax_sh[((g & 1) * 2 + (half ^ 1)) * 128 + row]);
                }
                float lw_n1 = 0.f;
                if constexpr (kUnits) {
                    if (i + 1 < n) lw_n1 = unit_lw(j_n1, w_n1, nv_n);
                } else if (kWeighted && i + 1 < n) {
                    lw_n1 = lw_of(w_n1);
                }
                // units: the maxima were taken over scaled, weight-shifted logits
                const float xmax = kUnits ? smax : smax * p.scale_log2 + lw;
                const float m_new = fmaxf(m_run, xmax);
                bool rescale = false;
                if (i == 0) {
                    m_run = m_new;
                } else if (m_new > m_run + kRescaleThreshold) {
                    rescale = true;
                }
                if (__any_sync(0xffffffffu, rescale)) {
                    // O (split: O_h) *= 2^(m_run - m_new) on the rows that need it, this
                    // warp's columns of it; PV(g-1) must be done
                    wait_o(g - 1);
                    tc_fence_after();
                    const float f = rescale ? fast_exp2(m_run - m_new) : 1.0f;
#pragma unroll 1
                    for (int ch = 0; ch < (kSplit ? D : D / 2) / 32; ++ch) {
                        uint32_t r32[32];
                        const uint32_t oc = col_o_own + ch * 32;
                        tmem_ld32(tmem + lane_off + oc, r32);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            r32[e] = __float_as_uint(__uint_as_float(r32[e]) * f);
                        tmem_st32(tmem + lane_off + oc, r32);
                    }
                    if (rescale) {
                        l_run *= f;
                        m_run = m_new;
                    }
                }
                // P = 2^(s * scale_log2 + lw - m_run) in fp32 pairs, packed to bf16 over
                // the S columns; every fifth pair uses the FMA-pipe exp2.
                // A half row may have seen no valid key yet (its columns of the block
                // past the sequence end, or every kept unit there); its P is then 0, not
                // NaN
                const float m_ref = m_run == -INFINITY ? 0.f : m_run;
                const float bias = kUnits ? -m_ref : lw - m_ref;
                const uint64_t bias2 = f2_pack(bias, bias);
                uint64_t ls2[4] = {0, 0, 0, 0};
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const uint64_t x2 = kUnits ? f2_add(f2_pack(sv[2 * e], sv[2 * e + 1]), bias2)
                                               : f2_fma(f2_pack(sv[2 * e], sv[2 * e + 1]), scale2, bias2);
                    float2 pr;
                    if (e % kSoftEvery == kSoftEvery - 1) {
                        pr = soft_exp2_pair(x2);
                    } else {
                        const float2 xv = f2_unpack(x2);
                        pr.x = fast_exp2(xv.x);
                        pr.y = fast_exp2(xv.y);
                    }
                    ls2[e & 3] = f2_add(ls2[e & 3], f2_pack(pr.x, pr.y));
                    pk[e] = pack_bf16x2(pr.x, pr.y);
                }
                tmem_st32(tmem + lane_off + s_col + half * (kSplit ? 64 : 32), pk);
                {
                    const float2 a = f2_unpack(f2_add(f2_add(ls2[0], ls2[1]), f2_add(ls2[2], ls2[3])));
                    l_run += a.x + a.y;
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&p_own[g % kSB]);
                if (i + 1 < n) {
                    j = kUnits ? 0 : clamp_j(j_n1);
                    lw = lw_n1;
                    nv_l = nv_n;
                    j_n1 = j_n2;
                    w_n1 = w_n2;
                }

                if (i == n - 1) {
                    // epilogue: the item's last PV(s) done, (m, l) exchanged, this warp's
                    // half of the output columns (split halves: from O_0 and O_1) divided
                    // by l, straight to global memory
                    wait_o(g);
                    if constexpr (kSplit) wait_o_oth(g);
                    xm_sh[half * 128 + row] = m_run;
                    xl_sh[half * 128 + row] = l_run;
                    pair_sync();
                    const float m_o = xm_sh[(half ^ 1) * 128 + row];
                    const float l_o = xl_sh[(half ^ 1) * 128 + row];
                    // shared rows: one max, l = l_0 + l_1; split halves: weight of each
                    // accumulator 2^(m_h - m), 0 for a half that saw no key
                    const float m_tot = kSplit ? fmaxf(m_run, m_o) : m_run;
                    const float a_own = !kSplit ? 1.f : (m_run == -INFINITY ? 0.f : fast_exp2(m_run - m_tot));
                    const float a_oth = !kSplit ? 1.f : (m_o == -INFINITY ? 0.f : fast_exp2(m_o - m_tot));
                    const float l_tot = kSplit ? l_run * a_own + l_o * a_oth : l_run + l_o;
                    const float inv = (tok < p.N && l_tot > 0.f) ? 1.0f / l_tot : 0.f;
                    const float c_own = a_own * inv, c_oth = a_oth * inv;
#pragma unroll 1
                    for (int ch = 0; ch < kHalfD / 32; ++ch) {
                        uint32_t ra[32], rb[32];
                        float o[32];
                        if constexpr (kSplit) {
                            tmem_ld32(tmem + lane_off + col_o_own + half * kHalfD + ch * 32, ra);
                            tmem_ld32(tmem + lane_off + col_o_oth + half * kHalfD + ch * 32, rb);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                o[e] = fmaf(__uint_as_float(ra[e]), c_own, __uint_as_float(rb[e]) * c_oth);
                        } else {
                            tmem_ld32(tmem + lane_off + col_o_own + ch * 32, ra);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(ra[e]) * inv;
                        }
                        if (kOutF32) {
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                o4[ch * 8 + e] = make_uint4(__float_as_uint(o[4 * e + 0]), __float_as_uint(o[4 * e + 1]),
                                                            __float_as_uint(o[4 * e + 2]), __float_as_uint(o[4 * e + 3]));
                        } else {
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                o4[ch * 4 + e] = make_uint4(pack_bf16x2(o[8 * e + 0], o[8 * e + 1]),
                                                            pack_bf16x2(o[8 * e + 2], o[8 * e + 3]),
                                                            pack_bf16x2(o[8 * e + 4], o[8 * e + 5]),
                                                            pack_bf16x2(o[8 * e + 6], o[8 * e + 7]));
                        }
                    }
                    if (p.lse && half == 0)
                        p.lse[(size_t)bh * p.N_pad + tok] =
                            tok < p.N ? (l_tot > 0.f ? (m_tot + log2f(l_tot)) * 0.69314718055994531f
                                                     : -INFINITY)
                                      : 0.f;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    // every claim of this CTA is made: the slot must still carry this launch's tag
    if (threadIdx.x == 0) slot_check(p);
}

// ---------------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------------
// 3-D map over a [B*H, N_pad, d] bf16 tensor with row extent N (rows >= N read as 0),
// box 64 columns x 128 rows, 128-byte swizzle.
static bool make_tmap(CUtensorMap *tm, const void *base, int BH, int N, int N_pad, int d)
{
    return make_tmap_bf16_3d(tm, base, (uint64_t)d, (uint64_t)N, (uint64_t)BH, (uint64_t)d * 2,
                             (uint64_t)N_pad * d * 2, 64, 128);
}

// Claim slots of the item scheduler (16 bytes each: items claimed, owner tag, two unused
// words). A launch takes the next slot in turn, zeroes it on its own stream just before
// the kernel and tags it with its launch number; launches that share a slot while both
// run are detected (slot_join / slot_check).
constexpr unsigned kCounterSlots = 4096;
__device__ unsigned int g_item_counters[kCounterSlots][4];
static std::atomic<unsigned long long> g_counter_next{0};
static std::atomic<int> g_forced_slot{-1};

static cudaError_t counter_slot(cudaStream_t st, unsigned int **slot, unsigned *tag)
{
    void *base = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&base, g_item_counters);
    if (e != cudaSuccess) return e;
    const unsigned long long gen = g_counter_next.fetch_add(1, std::memory_order_relaxed);
    const int forced = g_forced_slot.exchange(-1);
    const unsigned k = forced >= 0 ? (unsigned)forced : (unsigned)(gen % kCounterSlots);
    *slot = static_cast<unsigned int *>(base) + 4 * k;
    *tag = 1u + (unsigned)(gen % 0xFFFFFFFEull);  // 1 .. 0xFFFFFFFE: never 0 or kSlotPoison
    return cudaMemsetAsync(*slot, 0, 4 * sizeof(unsigned int), st);
}

void force_next_counter_slot(int slot) { g_forced_slot.store(slot % (int)kCounterSlots); }

template <int D, bool W, bool F32, bool U4>
static cudaError_t launch_attn_t(const AttnLaunch &a, cudaStream_t st)
{
    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, a.q, a.B * a.H, a.N, a.N_pad, D) ||
        !make_tmap(&tk, a.k, a.B * a.H, a.N, a.N_pad, D) ||
        !make_tmap(&tv, a.v, a.B * a.H, a.N, a.N_pad, D))
        return cudaErrorInvalidValue;
    AttnParams p;
    p.idx = a.idx;
    p.cnt = a.cnt;
    p.w = a.w;
    p.out = a.out;
    p.lse = a.lse;
    p.flag = a.flag;
    p.kg = static_cast<const __nv_bfloat16 *>(a.k);
    p.vg = static_cast<const __nv_bfloat16 *>(a.v);
    p.H = a.H;
    p.N = a.N;
    p.N_pad = a.N_pad;
    p.nqb = a.N_pad / 128;
    p.nkb = a.N_pad / (U4 ? 4 : 128);
    p.per_tile = U4 ? 32 : 1;
    p.n_items = a.B * a.H * p.nqb;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    p.wait_ns = a.wait_ns > 0 ? a.wait_ns : kWaitLimitNs;
    cudaError_t e = counter_slot(st, &p.counter, &p.tag);
    if (e != cudaSuccess) return e;
    const int smem = AttnSmem<D, U4>::kAlloc;
    e = cudaFuncSetAttribute(attn_fwd_kernel<D, W, F32, U4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = a.grid_override > 0 ? a.grid_override : (p.n_items < sms ? p.n_items : sms);
    attn_fwd_kernel<D, W, F32, U4><<<grid, attn_threads(U4), smem, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

template <int D, bool W, bool F32>
static cudaError_t launch_attn_u(const AttnLaunch &a, cudaStream_t st)
{
    return a.unit == 4 ? launch_attn_t<D, W, F32, true>(a, st) : launch_attn_t<D, W, F32, false>(a, st);
}

template <int D, bool W>
static cudaError_t launch_attn_o(const AttnLaunch &a, cudaStream_t st)
{
    return a.out_f32 ? launch_attn_u<D, W, true>(a, st) : launch_attn_u<D, W, false>(a, st);
}

cudaError_t launch_attn(const AttnLaunch &a, cudaStream_t st)
{
    const bool weighted = a.w != nullptr;
    if (a.d == 128) return weighted ? launch_attn_o<128, true>(a, st) : launch_attn_o<128, false>(a, st);
    return weighted ? launch_attn_o<64, true>(a, st) : launch_attn_o<64, false>(a, st);
}

}  // namespace ab
