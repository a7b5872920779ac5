// Multi-query (prefill / chunked-prefill) paged attention on the sm_100a
// tensor cores.
//
// What it computes (brentwoodlivery.com "5.3.18 …": prefill handles all
// prompt tokens at once and is compute-bound; comfyai.app "6.4 PagedAttention",
// 6.4.3: the prompt's blocks are written in the prefill stage): sequence b
// has L tokens in the paged cache, the last n of which are new; new token i
// (position p = L - n + i) attends causally to the cached tokens t <= p:
//   out = softmax_t(scale q.K_t) V_t, K_t / V_t read through the block table.
//
// How: persistent CTAs (one per SM) claim items (256 new tokens = two
// 128-row query tiles, head, sequence) from a global counter; each CTA is
// warp-specialised, with the two query tiles in ping-pong so the tensor core
// works on one tile while the other tile's softmax runs, and one item's
// epilogue overlaps the next item's loads and score products.
//   * warp 8 (loads): claims the next item and passes its index to the other
//     roles through a two-deep shared-memory queue; TMA tensor loads of Q,
//     then of each 128-token K and V
//     tile, (block, head) run by run through the block table, into a ring of
//     four 128-byte-swizzled shared-memory tiles;
//   * warp 9 (matrix unit, one thread): S_t = Q_t K^T into TMEM, and, once
//     the softmax of tile t has written P_t, O_t += P_t V with P_t read
//     straight from TMEM (P overwrites S in place) and V from shared memory;
//     the order S_0 PV_0 S_0' PV_1 S_1' keeps one tile's matrix work in
//     flight while the other tile's softmax runs;
//   * warps 0-3 / 4-7 (softmax of query tile 0 / 1, one query row per
//     thread = TMEM lane): read the S row back (all 128 columns, one wait),
//     causal mask, online softmax in the
//     log2 domain, P as fp16 into TMEM (the row sum l is taken from P before
//     its fp16 rounding).  Only warps holding a diagonal or context-end tile
//     pay for the mask.  The running max is only moved when
//     it grows by more than 2^8 (in base-2 exponent units); then the warp
//     rescales its O rows and l in TMEM.  Otherwise P is taken against the
//     stale max (P <= 2^8, exact up to fp16 rounding, no overflow).  The
//     result is the same softmax: O and l always share one reference max.
//   * epilogue: O / l to fp16, written straight to global memory; O_t is
//     then released to the next item (o_empty), Q once the item's last score
//     product is done (q_empty).
// TMEM: S0 / S1 at columns 0 / 128, O0 / O1 at 256 / 384 (all 512 columns;
// one CTA per SM).  Every wait is bounded: a wait that runs out records
// PA_DEVERR_TIMEOUT and raises an abort flag that ends every role's loop,
// after which in-flight copies and matrix operations are drained (bounded)
// before TMEM is released.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "../../include/pa.h"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace pa {

struct PrefillParams {
    __half *out;                      // [num_tokens, H, D]
    const int32_t *block_tables;      // [B, MB]
    const int32_t *context_lens;      // [B]
    const int32_t *query_start_loc;   // [B + 1]
    int max_blocks_per_seq;
    int max_context_len;
    int num_heads;
    int block_size;
    int num_blocks;
    float qk_scale_log2;              // softmax scale * log2(e), > 0
    unsigned int *error_word;         // PA_DEVERR_* bits
    int num_seqs;
    int num_pairs;                    // query-tile pairs per sequence: ceil(max_query_len / 256)
    unsigned int *sched;              // [2]: next item to hand out, CTAs finished (both 0 at launch)
    int num_rows;                     // T: rows of q and out
};

constexpr int kPM = 128;              // query rows per tile (MMA M)
constexpr int kPN = 128;              // context tokens per tile (MMA N of Q K^T)
constexpr int kPD = 128;              // head dim handled here
constexpr int kQTiles = 2;            // query tiles per CTA
constexpr int kRing = 4;              // K / V tile slots
constexpr uint32_t kSub = 128 * 128;  // bytes of one [128 rows x 64 fp16] swizzled half tile
constexpr uint32_t kTileBytes = 2 * kSub;
constexpr uint32_t kOffRing = kQTiles * kTileBytes;
constexpr uint32_t kPrefillSmem = kOffRing + kRing * kTileBytes + 1024;  // + 1024-B alignment slack
constexpr int kLoadWarp = 8, kMmaWarp = 9;
constexpr int kPrefillThreads = 10 * 32;
constexpr uint32_t kTmemCols = 512;
// move the reference max only past this growth (base-2 units)
constexpr float kRescaleLog2 = 8.0f;
constexpr int kItemRing = 2;          // items handed from the load warp to the other roles
constexpr int kItemConsumers = 1 + 8; // the MMA thread and the eight softmax warps
constexpr int kGroupHB = 32;          // (head, sequence) units per scheduling group

__device__ __forceinline__ void prefill_error(const PrefillParams &p, unsigned int bits)
{
    atomicOr(p.error_word, bits);
}

// Bounded wait that also gives up as soon as another role raised the abort
// flag; a wait that runs out raises it (and records the timeout).
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int *abort,
                                              const PrefillParams &p)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort)
            return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            prefill_error(p, PA_DEVERR_TIMEOUT);
            *abort = 1;
            return false;
        }
    }
    return true;
}

// ---- softmax arithmetic helpers (inline PTX of documented sm_100 forms) ----

__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x on the special-function unit (approximate, subnormal results flushed).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One S tile row in registers: all 128 scores of this thread's TMEM lane,
// loaded with one wait.
struct ScoreRow {
    uint32_t s[kPN];
};

__device__ __forceinline__ void load_score_row(uint32_t tS, ScoreRow &r)
{
#pragma unroll
    for (int cc = 0; cc < kPN / 32; ++cc)
        tmem_load32_into(tS + uint32_t(cc * 32), r.s + cc * 32);
    tmem_wait_ld();
}

// Row max of the raw scores; with kMasked only the first `lim` columns count.
template <bool kMasked>
__device__ __forceinline__ float score_row_max(const ScoreRow &r, int lim)
{
    float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < kPN; i += 8) {
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            float x = __uint_as_float(r.s[i + 2 * a]), y = __uint_as_float(r.s[i + 2 * a + 1]);
            if (kMasked) {
                x = i + 2 * a < lim ? x : -INFINITY;
                y = i + 2 * a + 1 < lim ? y : -INFINITY;
            }
            m[a] = max3f(m[a], x, y);
        }
    }
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// P = 2^(c * s - m) of the row, as fp16 pairs written into TMEM over the
// first 64 columns of S; returns the row sum of P (fp32, before the fp16
// rounding).  With kMasked, columns >= lim give P = 0.
template <bool kMasked>
__device__ __forceinline__ float write_p_row(uint32_t tS, const ScoreRow &r, int lim, float c,
                                             float m)
{
    float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int cc = 0; cc < kPN / 32; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int i = cc * 32 + 2 * e;
            const float x0 = fmaf(__uint_as_float(r.s[i]), c, -m);
            const float x1 = fmaf(__uint_as_float(r.s[i + 1]), c, -m);
            float p0 = ex2_approx(x0);
            float p1 = ex2_approx(x1);
            if (kMasked) {
                p0 = i < lim ? p0 : 0.f;
                p1 = i + 1 < lim ? p1 : 0.f;
            }
            sum[(e & 1) * 2] += p0;
            sum[(e & 1) * 2 + 1] += p1;
            const __half2 ph = __floats2half2_rn(p0, p1);
            pk[e] = *reinterpret_cast<const uint32_t *>(&ph);
        }
        tmem_store16(tS + uint32_t(cc * 16), pk);
    }
    return (sum[0] + sum[1]) + (sum[2] + sum[3]);
}

// One unit of work: two query tiles (256 new tokens) of one (head, sequence).
struct PrefillItem {
    int b, h, row0, q_first, L;
    int table_row;       // block-table row of the context
    int rows[kQTiles];   // new tokens in query tile t (0 = tile absent)
    int pos0[kQTiles];   // position of row 0 of tile t
    int nt[kQTiles];     // context tiles tile t attends to
    int ntiles;          // context tiles the item walks
};

// Item numbering.  The (head, sequence) units are cut into groups of
// kGroupHB; within a group the items run pair-major, the latest (heaviest)
// pair of every unit first: k -> group g = k / (kGroupHB P), then
// pair = P - 1 - r / n_g and unit = g kGroupHB + r % n_g for r = k mod
// (kGroupHB P) and n_g units in the group.  CTAs take the next item from a
// global counter when their load warp is ready, so the work balances itself;
// the items in flight at one time belong to about one group, whose K / V
// (kGroupHB units) stay in L2; and each group ends with its lightest items.
// Empty items (past a sequence's new tokens, or with more new tokens than
// context) are skipped by the load warp and never reach the other roles.
// `report` lets exactly one thread record per-sequence argument errors.
__device__ __forceinline__ bool prefill_item(const PrefillParams &p, int k, PrefillItem &it,
                                             bool report)
{
    const int units = p.num_heads * p.num_seqs;
    const int per_group = kGroupHB * p.num_pairs;
    const int g = k / per_group, r = k % per_group;
    const int n_g = min(kGroupHB, units - g * kGroupHB);
    const int pair = p.num_pairs - 1 - r / n_g;
    const int hb = g * kGroupHB + r % n_g;
    it.h = hb % p.num_heads;
    it.b = hb / p.num_heads;
    it.q_first = p.query_start_loc[it.b];
    const int n = p.query_start_loc[it.b + 1] - it.q_first;
    int L = p.context_lens[it.b];
    const bool first = report && pair == 0 && it.h == 0;
    if (L < 0 || L > p.max_context_len) {
        if (first)
            prefill_error(p, PA_DEVERR_CONTEXT_LEN);
        L = max(0, min(L, p.max_context_len));
    }
    it.L = L;
    it.row0 = pair * kQTiles * kPM;
    it.table_row = it.b;
    if (n <= 0 || it.row0 >= n)
        return false;
    if (it.q_first < 0 || n > p.num_rows - it.q_first) {  // rows outside q / out
        if (first)
            prefill_error(p, PA_DEVERR_CONTEXT_LEN);
        return false;
    }
    if (n > L) {  // more new tokens than the context holds: nothing sensible to do
        if (first)
            prefill_error(p, PA_DEVERR_CONTEXT_LEN);
        return false;
    }
    it.ntiles = 0;
#pragma unroll
    for (int t = 0; t < kQTiles; ++t) {
        const int r0 = it.row0 + t * kPM;
        it.rows[t] = max(0, min(kPM, n - r0));
        it.pos0[t] = L - n + r0;
        const int last = it.pos0[t] + it.rows[t] - 1;  // last position seen
        it.nt[t] = it.rows[t] > 0 ? last / kPN + 1 : 0;
        it.ntiles = max(it.ntiles, it.nt[t]);
    }
    return true;
}

struct PrefillShared {
    uint64_t item_full[kItemRing], item_empty[kItemRing];
    uint64_t q_full, q_empty, drain;
    uint64_t kv_full[kRing], kv_empty[kRing];
    uint64_t s_full[kQTiles], p_full[kQTiles], o_full[kQTiles], o_empty[kQTiles];
    int item[kItemRing];   // item index, or -1 = no more items
    uint32_t tmem;
    int abort;
};

// Next item for the MMA / softmax roles: the load warp's choice, in order.
// Returns -1 when there are no more items (or on abort).  The caller
// releases the slot right away (it copies the index).
__device__ __forceinline__ int prefill_pop_item(const PrefillParams &p, PrefillShared &sh, int u,
                                                bool arrive)
{
    const int slot = u % kItemRing;
    if (!wait_or_abort(smem_u32(&sh.item_full[slot]), uint32_t(u / kItemRing) & 1u, &sh.abort, p))
        return -1;
    const int k = *reinterpret_cast<volatile int *>(&sh.item[slot]);
    if (arrive)
        mbar_arrive(smem_u32(&sh.item_empty[slot]));
    return k;
}

// ---------------------------------------------------------------- loads
__device__ __forceinline__ void prefill_load_role(const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                                  const CUtensorMap *tm_v, const PrefillParams &p,
                                                  PrefillShared &sh, uint32_t sbase, int lane)
{
    volatile int *abort = &sh.abort;
    const int H = p.num_heads, bsz = p.block_size;
    const int box_rows = bsz < kPN ? bsz : kPN;
    const int total = p.num_pairs * H * p.num_seqs;
    int last_use[kRing];
#pragma unroll
    for (int i = 0; i < kRing; ++i)
        last_use[i] = -1;
    int ring = 0, items = 0;
    bool go = true;
    for (;;) {
        // claim the next non-empty item and hand it to the other roles
        int k = -1;
        PrefillItem it;
        for (;;) {
            int kk = 0;
            if (lane == 0)
                kk = *abort ? total : int(atomicAdd(p.sched, 1u));
            kk = __shfl_sync(kFullMask, kk, 0);
            if (kk >= total)
                break;
            if (prefill_item(p, kk, it, lane == 0)) {
                k = kk;
                break;
            }
        }
        {
            const int slot = items % kItemRing, use = items / kItemRing;
            bool ok = true;
            if (use > 0 && lane == 0)
                ok = wait_or_abort(smem_u32(&sh.item_empty[slot]), uint32_t(use - 1) & 1u, abort, p);
            if (!__shfl_sync(kFullMask, int(ok), 0))
                break;
            if (lane == 0) {
                sh.item[slot] = k;
                mbar_arrive(smem_u32(&sh.item_full[slot]));  // release: the index is visible
            }
            __syncwarp();
        }
        if (k < 0)
            break;
        // Q of this item once the previous item's score products are done
        if (items > 0) {
            const bool ok = lane == 0 ? wait_or_abort(smem_u32(&sh.q_empty), uint32_t(items - 1) & 1u,
                                                      abort, p)
                                      : true;
            if (!(go = __shfl_sync(kFullMask, int(ok), 0) != 0))
                break;
        }
        if (lane == 0) {
            uint32_t qbytes = 0;
            for (int t = 0; t < kQTiles; ++t)
                qbytes += it.rows[t] > 0 ? kTileBytes : 0u;
            mbar_arrive_expect_tx(smem_u32(&sh.q_full), qbytes);
            for (int t = 0; t < kQTiles; ++t) {
                if (it.rows[t] <= 0)
                    continue;
                const int y = it.q_first + it.row0 + t * kPM;
                tma_load_2d(sbase + t * kTileBytes, tm_q, it.h * kPD, y, smem_u32(&sh.q_full));
                tma_load_2d(sbase + t * kTileBytes + kSub, tm_q, it.h * kPD + 64, y,
                            smem_u32(&sh.q_full));
            }
        }
        ++items;
        const int32_t *trow = p.block_tables + size_t(it.table_row) * p.max_blocks_per_seq;
        for (int j = 0; go && j < it.ntiles; ++j) {
            const int t0 = j * kPN;
            const int valid = min(kPN, it.L - t0);
            const int runs = (valid + box_rows - 1) / box_rows;
            int y = 0;
            bool ok_id = false;
            if (lane < runs) {
                const int tok = t0 + lane * box_rows;
                const int id = trow[tok / bsz];
                ok_id = unsigned(id) < unsigned(p.num_blocks);
                if (!ok_id)
                    prefill_error(p, PA_DEVERR_BLOCK_ID);
                y = (id * H + it.h) * bsz + tok % bsz;
            }
            const uint32_t bytes = uint32_t(__popc(__ballot_sync(kFullMask, ok_id))) *
                                   uint32_t(box_rows) * 256u;
            for (int kind = 0; kind < 2; ++kind) {  // K, then V
                const int i = ring + 2 * j + kind, slot = i % kRing, use = i / kRing;
                const uint32_t full = smem_u32(&sh.kv_full[slot]);
                if (use > 0) {
                    const bool ok = lane == 0 ? wait_or_abort(smem_u32(&sh.kv_empty[slot]),
                                                              uint32_t(use - 1) & 1u, abort, p)
                                              : true;
                    if (!(go = __shfl_sync(kFullMask, int(ok), 0) != 0))
                        break;
                }
                if (lane == 0)
                    mbar_arrive_expect_tx(full, bytes);
                last_use[slot] = use;
                __syncwarp();
                if (ok_id) {
                    const CUtensorMap *map = kind == 0 ? tm_k : tm_v;
                    const uint32_t dst = sbase + kOffRing + uint32_t(slot) * kTileBytes +
                                         uint32_t(lane * box_rows) * 128u;
                    tma_load_2d(dst, map, 0, y, full);
                    tma_load_2d(dst + kSub, map, 64, y, full);
                }
            }
        }
        ring += 2 * it.ntiles;
        if (!go)
            break;
    }
    // After an abort, let the copies already issued land before the CTA (and
    // its shared memory) goes away.
    if (*abort && lane == 0) {
        for (int i = 0; i < kRing; ++i)
            if (last_use[i] >= 0)
                mbar_wait_bounded(smem_u32(&sh.kv_full[i]), uint32_t(last_use[i]) & 1u);
        if (items > 0)
            mbar_wait_bounded(smem_u32(&sh.q_full), uint32_t(items - 1) & 1u);
    }
}

// ------------------------------------------------------------ matrix unit
__device__ __forceinline__ void prefill_mma_role(const PrefillParams &p, PrefillShared &sh,
                                                 uint32_t sbase)
{
    constexpr uint32_t kIdescS = idesc_f16_f32(kPM, kPN, false);
    constexpr uint32_t kIdescO = idesc_f16_f32(kPM, kPD, true);
    volatile int *abort = &sh.abort;
    const uint32_t tmem = sh.tmem;
    auto slot_addr = [&](int i) { return sbase + kOffRing + uint32_t(i % kRing) * kTileBytes; };
    auto wait_full = [&](int i) {
        const bool ok = wait_or_abort(smem_u32(&sh.kv_full[i % kRing]), uint32_t(i / kRing) & 1u,
                                      abort, p);
        tc_fence_after_sync();
        return ok;
    };
    auto issue_s = [&](int t, uint32_t k_addr) {
        const uint32_t q_addr = sbase + uint32_t(t) * kTileBytes;
#pragma unroll
        for (int k = 0; k < kPD / 16; ++k) {
            const uint32_t kb = uint32_t(k >> 2) * kSub, kk = uint32_t(k & 3) * 32u;
            umma_f16(tmem + uint32_t(t) * kPN, smem_desc_sw128(q_addr + kb + kk, 16, 1024),
                     smem_desc_sw128(k_addr + kb + kk, 16, 1024), kIdescS, k > 0);
        }
        umma_commit(smem_u32(&sh.s_full[t]));
    };
    auto issue_pv = [&](int t, uint32_t v_addr, bool accumulate) {
        const uint32_t p_tmem = tmem + uint32_t(t) * kPN;  // P aliases S
        const uint32_t o_tmem = tmem + 2u * kPN + uint32_t(t) * kPD;
#pragma unroll
        for (int k = 0; k < kPN / 16; ++k)
            umma_f16_ts(o_tmem, p_tmem + uint32_t(k) * 8u,
                        smem_desc_sw128(v_addr + uint32_t(k) * 2048u, kSub, 1024), kIdescO,
                        accumulate || k > 0);
        umma_commit(smem_u32(&sh.o_full[t]));
    };

    int ring = 0, items = 0;
    int cnt[kQTiles] = {0, 0};       // context tiles processed per query tile (all items)
    int t_items[kQTiles] = {0, 0};   // items in which query tile t took part
    bool ok = true;
    for (int u = 0; ok; ++u) {
        const int k = prefill_pop_item(p, sh, u, true);
        if (k < 0)
            break;
        PrefillItem it;
        prefill_item(p, k, it, false);
        const bool act[kQTiles] = {it.rows[0] > 0, it.rows[1] > 0};
        // P V of tile t at context tile j: the softmax has written P_t, and,
        // for an item's first tile, the previous item's epilogue has read O_t
        auto pv = [&](int t, int j, uint32_t v_addr) {
            if (j == 0 && t_items[t] > 0 &&
                !wait_or_abort(smem_u32(&sh.o_empty[t]), uint32_t(t_items[t] - 1) & 1u, abort, p))
                return false;
            if (!wait_or_abort(smem_u32(&sh.p_full[t]), uint32_t(cnt[t] + j) & 1u, abort, p))
                return false;
            tc_fence_after_sync();
            issue_pv(t, v_addr, j > 0);
            return true;
        };
        if (!(ok = wait_or_abort(smem_u32(&sh.q_full), uint32_t(items) & 1u, abort, p) &&
                   wait_full(ring)))
            break;
        ++items;
        for (int t = 0; t < kQTiles; ++t)
            if (act[t] && it.nt[t] > 0)
                issue_s(t, slot_addr(ring));
        umma_commit(smem_u32(&sh.kv_empty[ring % kRing]));
        if (it.ntiles == 1)
            umma_commit(smem_u32(&sh.q_empty));  // last score product of the item issued
        for (int j = 0; j < it.ntiles; ++j) {
            const int iv = ring + 2 * j + 1, ik = ring + 2 * j + 2;
            const bool next = j + 1 < it.ntiles;
            if (!(ok = wait_full(iv)))
                break;
            if (act[0] && j < it.nt[0] && !(ok = pv(0, j, slot_addr(iv))))
                break;
            if (next) {
                if (!(ok = wait_full(ik)))
                    break;
                if (act[0] && j + 1 < it.nt[0])
                    issue_s(0, slot_addr(ik));
            }
            if (act[1] && j < it.nt[1] && !(ok = pv(1, j, slot_addr(iv))))
                break;
            umma_commit(smem_u32(&sh.kv_empty[iv % kRing]));
            if (next) {
                if (act[1] && j + 1 < it.nt[1])
                    issue_s(1, slot_addr(ik));
                umma_commit(smem_u32(&sh.kv_empty[ik % kRing]));
                if (j + 2 == it.ntiles)
                    umma_commit(smem_u32(&sh.q_empty));
            }
        }
        for (int t = 0; t < kQTiles; ++t)
            if (act[t]) {
                cnt[t] += it.nt[t];
                ++t_items[t];
            }
        ring += 2 * it.ntiles;
    }
    // every matrix operation issued has finished before TMEM and the shared
    // tiles are released
    umma_commit(smem_u32(&sh.drain));
    mbar_wait_bounded(smem_u32(&sh.drain), 0u);
}

// ---------------------------------------------------------------- softmax
__device__ __forceinline__ void prefill_softmax_role(const PrefillParams &p, PrefillShared &sh,
                                                     unsigned char *smem, int warp, int lane)
{
    volatile int *abort = &sh.abort;
    const int t = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = sh.tmem + uint32_t(t) * kPN + lane_base;
    const uint32_t tO = sh.tmem + 2u * kPN + uint32_t(t) * kPD + lane_base;
    const float c = p.qk_scale_log2;
    const int H = p.num_heads;
    int ring = 0, cnt = 0;
    for (int u = 0;; ++u) {
        const int k = __shfl_sync(kFullMask, lane == 0 ? prefill_pop_item(p, sh, u, false) : 0, 0);
        __syncwarp();
        if (lane == 0 && k >= 0)
            mbar_arrive(smem_u32(&sh.item_empty[u % kItemRing]));
        if (k < 0)
            break;
        PrefillItem it;
        prefill_item(p, k, it, false);
        const int item_ring = ring;
        ring += 2 * it.ntiles;
        if (it.rows[t] <= 0)
            continue;
        const int my_pos = it.pos0[t] + r;
        const int L = it.L;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < it.nt[t]; ++j) {
            ok = __all_sync(kFullMask,
                            wait_or_abort(smem_u32(&sh.s_full[t]), uint32_t(cnt + j) & 1u, abort, p));
            if (!ok)
                break;
            tc_fence_after_sync();
            const int t0 = j * kPN;
            // columns of this tile this row may see: t <= my_pos and t < L
            const int lim = min(my_pos, L - 1) - t0 + 1;
            const bool masked = __any_sync(kFullMask, lim < kPN);
            ScoreRow row;
            load_score_row(tS, row);
            const float mx = (masked ? score_row_max<true>(row, lim) : score_row_max<false>(row, lim)) * c;
            const float m_new = fmaxf(m_ref, mx);
            if (j == 0) {
                m_ref = m_new;
            } else if (__any_sync(kFullMask, m_new > m_ref + kRescaleLog2)) {
                // move this warp's reference max: rescale O and l
                ok = __all_sync(kFullMask, wait_or_abort(smem_u32(&sh.o_full[t]),
                                                          uint32_t(cnt + j - 1) & 1u, abort, p));
                if (!ok)
                    break;
                tc_fence_after_sync();
                const float alpha = ex2_approx(m_ref - m_new);
#pragma unroll 1
                for (int cc = 0; cc < kPD / 16; ++cc) {  // 16 columns at a time: the score row is live
                    uint32_t o[16];
                    tmem_load16_async(tO + uint32_t(cc * 16), o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_store16(tO + uint32_t(cc * 16), o);
                }
                l *= alpha;
                m_ref = m_new;
            }
            // P = 2^(scaled score - m_ref) as fp16 into TMEM over S
            l += masked ? write_p_row<true>(tS, row, lim, c, m_ref)
                        : write_p_row<false>(tS, row, lim, c, m_ref);
            tmem_wait_st();
            // V rows past the context end (the tail of the last block, or
            // stale ring contents) are zeroed, so 0 * garbage cannot reach O.
            // Done by the first query tile that uses this context tile.
            const int valid = L - t0;
            const int tz = (it.rows[0] > 0 && j < it.nt[0]) ? 0 : 1;
            if (valid < kPN && t == tz) {
                const int iv = item_ring + 2 * j + 1;
                ok = __all_sync(kFullMask, wait_or_abort(smem_u32(&sh.kv_full[iv % kRing]),
                                                          uint32_t(iv / kRing) & 1u, abort, p));
                if (!ok)
                    break;
                if (r >= valid) {
                    unsigned char *row =
                        smem + kOffRing + uint32_t(iv % kRing) * kTileBytes + uint32_t(r) * 128u;
#pragma unroll
                    for (int q16 = 0; q16 < 8; ++q16) {
                        *reinterpret_cast<uint4 *>(row + q16 * 16) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(row + kSub + q16 * 16) = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&sh.p_full[t]));
        }
        if (!ok)
            break;
        // epilogue: out = O / l, then O_t is free for the next item
        ok = __all_sync(kFullMask, wait_or_abort(smem_u32(&sh.o_full[t]),
                                                  uint32_t(cnt + it.nt[t] - 1) & 1u, abort, p));
        if (!ok)
            break;
        cnt += it.nt[t];
        tc_fence_after_sync();
        const float inv = 1.f / l;
        const size_t out_row = size_t(it.q_first + it.row0 + t * kPM + r) * H + it.h;
        uint4 *dst = reinterpret_cast<uint4 *>(p.out + out_row * kPD);
        const bool store = r < it.rows[t];
#pragma unroll 1
        for (int cc = 0; cc < kPD / 32; ++cc) {
            uint32_t o[32];
            tmem_load32_async(tO + uint32_t(cc * 32), o);
            tmem_wait_ld();
            if (store) {
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    __half2 v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        v[e] = __floats2half2_rn(__uint_as_float(o[g * 8 + 2 * e]) * inv,
                                                 __uint_as_float(o[g * 8 + 2 * e + 1]) * inv);
                    dst[cc * 4 + g] = *reinterpret_cast<const uint4 *>(v);
                }
            }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(smem_u32(&sh.o_empty[t]));
    }
}

__global__ void __launch_bounds__(kPrefillThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const PrefillParams p)
{
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) PrefillShared sh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    grid_dependency_wait();
    allow_dependent_launch();

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - raw);
    if (tid == 0) {
        for (int i = 0; i < kItemRing; ++i) {
            mbar_init(smem_u32(&sh.item_full[i]), 1);
            mbar_init(smem_u32(&sh.item_empty[i]), kItemConsumers);
        }
        mbar_init(smem_u32(&sh.q_full), 1);
        mbar_init(smem_u32(&sh.q_empty), 1);
        mbar_init(smem_u32(&sh.drain), 1);
        for (int i = 0; i < kRing; ++i) {
            mbar_init(smem_u32(&sh.kv_full[i]), 1);
            mbar_init(smem_u32(&sh.kv_empty[i]), 1);
        }
        for (int t = 0; t < kQTiles; ++t) {
            mbar_init(smem_u32(&sh.s_full[t]), 1);
            mbar_init(smem_u32(&sh.p_full[t]), 4);   // one arrival per softmax warp
            mbar_init(smem_u32(&sh.o_full[t]), 1);
            mbar_init(smem_u32(&sh.o_empty[t]), 4);  // one arrival per softmax warp
        }
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp)
        tmem_alloc(smem_u32(&sh.tmem), kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    if (warp == kLoadWarp) {
        prefill_load_role(&tm_q, &tm_k, &tm_v, p, sh, sbase, lane);
    } else if (warp == kMmaWarp) {
        if (lane == 0)
            prefill_mma_role(p, sh, sbase);
        __syncwarp();
    } else {
        prefill_softmax_role(p, sh, smem, warp, lane);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_free(sh.tmem, kTmemCols);
    }
    // The last CTA to finish resets the item counter for the launch that
    // next uses this scheduling slot (every CTA has stopped claiming items).
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
            atomicExch(p.sched, 0u);
            atomicExch(p.sched + 1, 0u);
            __threadfence();
        }
    }
}

} // namespace pa
