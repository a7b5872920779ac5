// The shared-prefix part of the decode of sequence groups (beam candidates,
// parallel samples of one prompt) on the sm_100a tensor cores.
//
// What it computes (comfyai.app "6.4 PagedAttention", 6.4.2: the samples of
// one prompt share its KV blocks; polomodov.tech "vLLM and PagedAttention",
// slides 13-14): the members of group g share the physical blocks of their
// first P_g tokens, so for every member b and head h the attention over those
// tokens, softmax_t(scale q[b, h] . K_t) V_t for t < P_g, can be computed
// with K and V read once per (group, head) and all the group's queries scored
// against each K tile together.  This kernel leaves, per member, head and
// 512-token chunk of the prefix, the unnormalised partial result (reference
// max m in base-2 units, sum l, o = sum_t 2^(s_t - m) V_t); the members'
// private tails are decoded by the paged decode kernel and the two parts are
// merged by their softmax normalisers (grouped.cu).
//
// How: the score product is computed transposed, S^T = K Q^T, so the MMA's
// M dimension is 128 context tokens and N is 16 query columns (up to 16
// members); a softmax thread then owns one token (one TMEM lane) and handles
// its <= 16 scores, so the per-tile softmax stays short.  The output
// O = P V accumulates in TMEM with the queries as M (rows 0-15 of 128; the
// other rows of the A operand are whatever follows P in shared memory and
// their results are never read) and the head dimension as N = 128: P is a
// K-major operand and V an N-major one, both as the loads left them.  (A
// small tcgen05.mma costs about the same for any N up to 64, and taking V
// as an M-major A operand instead costs about twice as much per
// instruction, so this orientation halves the P.V's tensor-pipe time.)
//   * Work items ("chunks", built by a set-up kernel): up to 512 tokens of a
//     group's prefix for a slice of up to 16 members, read through the first
//     member's table.  Items are (chunk, head) pairs; persistent CTAs (one per
//     SM) start with one each and claim the rest from a counter.
//   * warp 5 (loads): walks the CTA's items, passes each to the other roles
//     through a small shared-memory ring, and issues the TMA loads: the 16 Q
//     rows of the next item, and per 128-token tile K and V through the block
//     table, one 4-D box per (block, head) run, into six 32 KB slots.
//   * warp 6 (one thread): S^T(n) = K_n Q^T into one of two TMEM score
//     buffers and O += P_n V_n, each issued as soon as its inputs are ready;
//     a K slot is released when its score product completes, a V slot when
//     its P.V does.
//   * warps 0-3 (softmax, thread = token): the tile maximum per query column
//     (warp reduction, then the four warps' maxima through shared memory
//     behind one named barrier), exp2 against a reference max per column that
//     only moves when a tile's max exceeds it by more than 2^8 (then warp 0
//     rescales the rows of O and every thread its partial sums), P as fp16
//     into one of four shared-memory operand tiles; tokens past the prefix
//     end get P = 0 and their V rows are zeroed (by the MMA thread) so
//     garbage never meets a zero weight.
//   * warp 4 (epilogue, thread = query row of O): the rows of O and the
//     per-query sums are written to the workspace as (m, l, o).
// Every wait is bounded (1 s); the first to run out records PA_DEVERR_TIMEOUT
// and raises an abort flag that ends every role; copies and matrix
// operations in flight are drained (bounded) before TMEM is released.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <climits>
#include <cstdint>

#include "../../include/pa.h"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace pa {
namespace grp {

constexpr int kD = 128;                     // head dim handled here
constexpr int kT = 128;                     // context tokens per tile (M of S^T)
constexpr int kNQ = 16;                     // query columns per item (N of both products)
constexpr int kChunk = 512;                 // context tokens per work item
constexpr int kSlots = 6;                   // K / V tile slots
constexpr int kItemRing = 4;
// A K or V tile in shared memory: [16 row groups][2 halves][8 rows][64 fp16]
// with 128-byte swizzle, so every (row group, half) is one 1 KB swizzle atom.
constexpr uint32_t kTile = 128u * 256u;     // one K or V tile (32 KB)
constexpr uint32_t kAtom = 1024u;           // 8 rows x 128 bytes
constexpr uint32_t kGroupStride = 2048u;    // between 8-row groups
constexpr uint32_t kQHalf = kNQ * 128u;     // [16 rows x 64 fp16]
constexpr uint32_t kQTile = 2 * kQHalf;     // Q rows of an item, or P^T of a tile (4 KB)
constexpr int kQSlots = 2;                  // Q rows of the items in flight
constexpr int kPBufs = 4;                   // P operand tiles
// P tiles first: the P.V's A operand spans 128 rows (16 KB from a P tile's
// start), of which only the first 16 are P, so what follows a P tile must
// still be this CTA's shared memory.
constexpr uint32_t kOffP = 0;
constexpr uint32_t kOffQ = kOffP + kPBufs * kQTile;
constexpr uint32_t kOffKV = kOffQ + kQSlots * kQTile;
constexpr uint32_t kSmem = kOffKV + kSlots * kTile + 1024;  // + 1024-byte alignment slack
static_assert(kOffP + (kPBufs - 1) * kQTile + kQHalf + 16u * 1024u <= kOffKV + kSlots * kTile,
              "the P.V's A operand must stay inside the CTA's shared memory");
constexpr int kEpiWarp = 4, kLoadWarp = 5, kMmaWarp = 6;
constexpr int kThreads = 7 * 32;
constexpr uint32_t kTmemCols = 512;         // S0, S1 (16 columns each); O0, O1 (128 each)
constexpr uint32_t kTmemO = 128;            // O buffer b at kTmemO + 128 b
constexpr float kRescaleLog2 = 8.f;         // move a reference max only past this growth

// One work item's context part (head-independent): tokens [t0, t1) of
// block-table row `table_row`, scored for query rows q_row0 .. q_row0+nq-1.
struct Chunk {
    int table_row, q_row0, nq, t0, t1;
    int group;     // the sequence group whose members it contributes to
    int col;       // first partial-result column (column col + q: query row q_row0 + q)
    int pad;
};

// A group as the set-up kernel found it: members g0 .. g0+n-1, prefix chunks
// per 16-member slice (cp), the prefix length used (P), the first partial
// column of its prefix chunks (prefix chunk j of member b uses column
// colbase + j*n + (b - g0)), and the index of its first chunk in the work
// list.
struct Group {
    int g0, n, cp, P, colbase, pstart, pad0, pad1;
};

// A member b of group g: its tail length L_b - P_g (-1: in no group), its
// number of prefix chunks cp_g, and the partial column of its first prefix
// chunk (chunk j is column col0 + j * stride).
struct Member {
    int tail, cp, col0, stride;
};

// Work-list header at the start of the workspace.  The counters and the
// flag are zero when a call starts: the workspace is zeroed before its first
// use and every call's merge kernel sets them back to zero once it no longer
// needs them.
struct Meta {
    int nchunks;            // prefix chunks of all groups (from the set-up kernel)
    int ncols;              // partial columns they use
    int claimed;            // work items handed out past the first gridDim.x
    unsigned int tc_done;   // prefix CTAs finished (their partials written)
    unsigned int merge_done;// merge CTAs past their wait for the prefix kernel
    unsigned int ready;     // the set-up kernel's outputs are all visible
    int pad0, pad1;
};

// What a group contributes, by the same rules wherever it is worked out (the
// set-up kernel, or the prefix kernel itself when it builds its own work
// list): members g0 .. g0+n-1 when 0 <= g0 <= g1 <= B (else none); the prefix
// P when it is a multiple of the block size and at most every member's
// context (else 0); ceil(P / 512) chunks per slice of up to 16 members.
struct GroupPlan {
    int g0, n, P, cp, slices;
    bool bounds_ok, prefix_ok;
};

__host__ __device__ __forceinline__ GroupPlan plan_group(int g0, int g1, int P, int min_len, int B, int bs)
{
    GroupPlan r{};
    r.bounds_ok = 0 <= g0 && g0 <= g1 && g1 <= B;
    r.n = r.bounds_ok ? g1 - g0 : 0;
    r.g0 = r.bounds_ok ? g0 : 0;
    r.prefix_ok = r.n > 0 && P >= 0 && P % bs == 0 && P <= min_len;
    r.P = r.prefix_ok ? P : 0;
    r.cp = (r.P + kChunk - 1) / kChunk;
    r.slices = (r.n + 15) / 16;
    return r;
}

struct Params {
    __half *out;                      // [B, H, D]
    const int32_t *block_tables;      // [B, MB]
    const Chunk *chunks;              // capacity max_chunks
    Meta *meta;
    int max_chunks;
    // Set (at most 32 groups): the kernel builds its own work list from these
    // inputs instead of reading the set-up kernel's `chunks`, and so does not
    // wait for that kernel (which was launched before it and let it start
    // only after its own wait for the inputs).
    const int32_t *group_start;       // [G + 1]
    const int32_t *prefix_lens;       // [G]
    const int32_t *context_lens;      // [B]
    int num_groups, num_seqs, max_context_len;
    float *part_ml;                   // [columns, H, 2]: (reference max, sum)
    float *part_o;                    // [columns, H, D]
    int max_blocks_per_seq;
    int num_heads;
    int block_size;
    int num_blocks;
    float qk_scale_log2;              // softmax scale * log2(e), > 0
    unsigned int *error_word;
};

struct Item {
    Chunk c;
    int h;
    int k;  // item index, -1 = no more items
};

// softmax -> epilogue hand-off of one finished item
struct Epi {
    Chunk c;
    int h;
    int end;
    float m[kNQ];      // reference max per column (base-2 units)
    float l[4][kNQ];   // per-warp partial sums per column
};

struct Shared {
    uint64_t item_full[kItemRing], item_empty[kItemRing];
    uint64_t q_full[kQSlots], q_empty[kQSlots];
    uint64_t kv_full[kSlots], kv_empty[kSlots];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[kPBufs], p_empty[kPBufs];
    uint64_t o_full[2], o_empty[2], e_full[2];
    uint64_t drain;
    Item item[kItemRing];
    Epi epi[2];
    float red[2][4][kNQ];
    uint32_t tmem;
    int abort;
};

__device__ __forceinline__ bool gwait(uint32_t bar, uint32_t parity, volatile int *abort,
                                      unsigned int *err)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort)
            return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, PA_DEVERR_TIMEOUT);
            *abort = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ int chunk_tiles(const Chunk &c)
{
    return (c.t1 - c.t0 + kT - 1) / kT;
}

__device__ __forceinline__ float ex2f(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float warp_max(float x)
{
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
    return r;
}

// Barrier over the four softmax warps (named barrier 1) that also ANDs a
// flag across them, so that all four take the same branch afterwards.
__device__ __forceinline__ bool softmax_bar_and(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(v))
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        x += __shfl_xor_sync(kFullMask, x, off);
    return x;
}

// ---------------------------------------------------------------- loads
// Chunk field f (0..7) of the descriptor a lane holds.
__device__ __forceinline__ Chunk shfl_chunk(const Chunk &c, int src)
{
    Chunk r;
    r.table_row = __shfl_sync(kFullMask, c.table_row, src);
    r.q_row0 = __shfl_sync(kFullMask, c.q_row0, src);
    r.nq = __shfl_sync(kFullMask, c.nq, src);
    r.t0 = __shfl_sync(kFullMask, c.t0, src);
    r.t1 = __shfl_sync(kFullMask, c.t1, src);
    r.group = __shfl_sync(kFullMask, c.group, src);
    r.col = __shfl_sync(kFullMask, c.col, src);
    r.pad = 0;
    return r;
}

// Block ids of a whole chunk (at most 512 / 8 = 64 runs of `box` tokens):
// lane l holds runs l and l + 32.
__device__ __forceinline__ void load_chunk_ids(const Params &p, const Chunk &c, int box, int lane,
                                               int (&ids)[2])
{
    const int runs = (c.t1 - c.t0 + box - 1) / box;
    const int32_t *row = p.block_tables + size_t(c.table_row) * p.max_blocks_per_seq;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int run = lane + 32 * r;
        ids[r] = run < runs ? row[(c.t0 + run * box) / p.block_size] : 0;
    }
}

// Items are numbered chunk-major (k = chunk * H + head).  CTA c starts with
// item c and then claims one item at a time from a counter in the work-list
// header, so a CTA that streams faster takes more items and all CTAs finish
// within about one item of each other.  Every step that waits on memory is
// started a stage ahead: while item u's tiles are issued, item u + 1's
// descriptor is loaded (its index was claimed during item u - 1), then its
// block ids (after u's first tile), the index of item u + 2 is being
// claimed, and u + 1's Q rows go out after u's last tile.
// Tile m's K goes to slot (2m) % kSlots and its V to slot (2m + 1) % kSlots,
// so slots 0, 2, 4 only ever hold K tiles and slots 1, 3, 5 V tiles.
__device__ __forceinline__ void load_role(const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                          const CUtensorMap *tm_v, const Params &p, Shared &sh,
                                          uint32_t sbase, int lane)
{
    volatile int *abort = &sh.abort;
    unsigned int *err = p.error_word;
    const int H = p.num_heads, bs = p.block_size;
    const int box = bs < kT ? bs : kT;
    int last_use[kSlots];
#pragma unroll
    for (int i = 0; i < kSlots; ++i)
        last_use[i] = -1;
    int last_q[kQSlots];
#pragma unroll
    for (int i = 0; i < kQSlots; ++i)
        last_q[i] = -1;
    // the descriptor of item k (a broadcast load), or an empty one past the
    // work-list capacity
    // Self-built work list: lane g holds group g's plan and the exclusive
    // prefix sums of the groups' chunk and column counts.
    const bool self_list = p.group_start != nullptr;
    int sg0 = 0, sn = 0, sP = 0, sslices = 0, scount = 0, spstart = 0, scolbase = 0;
    int self_chunks = 0, self_cols = 0;
    if (self_list) {
        const int G = p.num_groups, B = p.num_seqs;
        if (lane < G) {
            const int g0 = p.group_start[lane], g1 = p.group_start[lane + 1], P = p.prefix_lens[lane];
            int min_len = INT_MAX;
            if (0 <= g0 && g0 <= g1 && g1 <= B)
                for (int b = g0; b < g1; ++b) {
                    const int L = p.context_lens[b];
                    min_len = min(min_len, L < 0 ? 0 : (L > p.max_context_len ? p.max_context_len : L));
                }
            const GroupPlan gp = plan_group(g0, g1, P, min_len, B, bs);
            sg0 = gp.g0;
            sn = gp.n;
            sP = gp.P;
            sslices = gp.slices;
            scount = gp.slices * gp.cp;
            scolbase = gp.n * gp.cp;
        }
        int xp = scount, xc = scolbase;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int yp = __shfl_up_sync(kFullMask, xp, off), yc = __shfl_up_sync(kFullMask, xc, off);
            if (lane >= off) {
                xp += yp;
                xc += yc;
            }
        }
        self_chunks = __shfl_sync(kFullMask, xp, 31);
        self_cols = __shfl_sync(kFullMask, xc, 31);
        spstart = xp - scount;
        scolbase = xc - scolbase;
        if (self_chunks > p.max_chunks || self_cols > p.max_chunks) {  // not with the host's bound
            if (lane == 0)
                atomicOr(err, PA_DEVERR_CONTEXT_LEN);
            self_chunks = 0;
        }
    }
    // the descriptor of item k (all lanes, k uniform): from the self-built
    // list, or a broadcast load of the set-up kernel's (an empty one past the
    // work-list capacity)
    auto descriptor = [&](int k) {
        Chunk c{};
        if (self_list) {
            const int ci = k / H;
            const unsigned mask = __ballot_sync(kFullMask, scount > 0 && spstart <= ci);
            if (k >= 0 && mask != 0u) {
                const int g = 31 - __clz(int(mask));
                const int g0 = __shfl_sync(kFullMask, sg0, g), n = __shfl_sync(kFullMask, sn, g);
                const int P = __shfl_sync(kFullMask, sP, g), sl = __shfl_sync(kFullMask, sslices, g);
                const int ps = __shfl_sync(kFullMask, spstart, g), cb = __shfl_sync(kFullMask, scolbase, g);
                const int idx = ci - ps, j = idx / sl, sli = idx - j * sl;
                c = Chunk{g0, g0 + 16 * sli, min(16, n - 16 * sli), j * kChunk, min((j + 1) * kChunk, P), g,
                          cb + j * n + 16 * sli, 0};
            }
        } else if (k >= 0 && k / H < p.max_chunks) {
            c = p.chunks[k / H];
        }
        return c;
    };
    // the next item index: one atomic by lane 0, not waited for here
    auto claim = [&]() { return lane == 0 ? int(gridDim.x) + atomicAdd(&p.meta->claimed, 1) : 0; };
    // the Q rows of item `it` (index k) into Q slot it % kQSlots, once its
    // previous user's score products are done
    auto issue_q = [&](int it, int k, const Chunk &c) {
        const int qs = it % kQSlots, use = it / kQSlots;
        bool ok = true;
        if (use > 0 && lane == 0)
            ok = gwait(smem_u32(&sh.q_empty[qs]), uint32_t(use - 1) & 1u, abort, err);
        if (!__shfl_sync(kFullMask, int(ok), 0))
            return false;
        if (lane == 0) {
            const int h = k % H;
            const uint32_t bar = smem_u32(&sh.q_full[qs]);
            mbar_arrive_expect_tx(bar, kQTile);
            const uint32_t dst = sbase + kOffQ + uint32_t(qs) * kQTile;
            tma_load_2d(dst, tm_q, h * kD, c.q_row0, bar);
            tma_load_2d(dst + kQHalf, tm_q, h * kD + 64, c.q_row0, bar);
        }
        last_q[qs] = use;
        return true;
    };
    struct TileRef {
        int y8;     // this lane's run: first 8-row group (valid when ok)
        bool ok;    // this lane has a run and its block id is in range
    };
    auto issue = [&](int kind, const TileRef &t, int i) {
        const int s = i % kSlots, use = i / kSlots;
        const uint32_t full = smem_u32(&sh.kv_full[s]);
        if (use > 0) {
            const bool ok = lane == 0 ? gwait(smem_u32(&sh.kv_empty[s]), uint32_t(use - 1) & 1u, abort, err)
                                      : true;
            if (!__shfl_sync(kFullMask, int(ok), 0))
                return false;
        }
        const uint32_t bytes = uint32_t(__popc(__ballot_sync(kFullMask, t.ok))) * uint32_t(box) * 256u;
        if (lane == 0)
            mbar_arrive_expect_tx(full, bytes);
        last_use[s] = use;
        __syncwarp();
        if (t.ok)
            tma_load_4d(sbase + kOffKV + uint32_t(s) * kTile + uint32_t(lane * box) * 256u, kind == 0 ? tm_k : tm_v,
                        0, 0, 0, t.y8, full);
        return true;
    };
    int m = 0;  // tiles issued
    bool go = true;
    // item 0 of this CTA: its descriptor and the item count come in together
    int kk = int(blockIdx.x);
    Chunk c = descriptor(kk);
    const int total = (self_list ? self_chunks : p.meta->nchunks) * H;
    if (kk >= total)
        kk = -1;
    int kn = -1, kclaim = 0;  // the next item; the claim after it (lane 0)
    int ids[2] = {0, 0};
    if (kk >= 0) {
        kclaim = claim();
        load_chunk_ids(p, c, box, lane, ids);
        go = issue_q(0, kk, c);
        kn = __shfl_sync(kFullMask, kclaim, 0);
        kclaim = claim();
    }
    for (int items = 0; go; ++items) {
        if (*abort)
            kk = -1;
        const bool has_next = kk >= 0 && kn < total;
        // the next item's descriptor; its block ids are loaded after this
        // item's first tile, when the descriptor has arrived
        const Chunk cn = has_next ? descriptor(kn) : Chunk{};
        int ids_n[2] = {0, 0};
        bool ids_pending = has_next;
        {
            const int slot = items % kItemRing, use = items / kItemRing;
            bool ok = true;
            if (use > 0 && lane == 0)
                ok = gwait(smem_u32(&sh.item_empty[slot]), uint32_t(use - 1) & 1u, abort, err);
            if (!__shfl_sync(kFullMask, int(ok), 0))
                break;
            if (lane == 0) {
                sh.item[slot].c = c;
                sh.item[slot].h = kk >= 0 ? kk % H : 0;
                sh.item[slot].k = kk;
                mbar_arrive(smem_u32(&sh.item_full[slot]));
            }
            __syncwarp();
        }
        if (kk < 0)
            break;
        const int h = kk % H;
        const int nt = chunk_tiles(c);
        const int runs_per_tile = kT / box;
        for (int j = 0; go && j < nt; ++j, ++m) {
            const int valid = min(kT, c.t1 - (c.t0 + j * kT));
            const int runs = (valid + box - 1) / box;
            const int run = j * runs_per_tile + lane;  // this lane's run within the chunk
            const int a = __shfl_sync(kFullMask, ids[0], run & 31);
            const int b = __shfl_sync(kFullMask, ids[1], run & 31);
            const int id = (run >> 5) ? b : a;
            TileRef t;
            t.ok = lane < runs && unsigned(id) < unsigned(p.num_blocks);
            if (lane < runs && !t.ok)
                atomicOr(err, PA_DEVERR_BLOCK_ID);
            t.y8 = (id * H + h) * (bs / 8);  // first 8-row group of the run
            go = issue(0, t, 2 * m) && issue(1, t, 2 * m + 1);
            if (ids_pending) {
                load_chunk_ids(p, cn, box, lane, ids_n);
                ids_pending = false;
            }
        }
        if (go && has_next)
            go = issue_q(items + 1, kn, cn);
        kk = has_next ? kn : -1;
        c = cn;
        ids[0] = ids_n[0];
        ids[1] = ids_n[1];
        if (kk >= 0) {  // the claim started one item ago becomes the next item; start another
            kn = __shfl_sync(kFullMask, kclaim, 0);
            if (kn < total)
                kclaim = claim();
        }
    }
    // After an abort, let the copies already issued land before the CTA (and
    // its shared memory) goes away.
    if (*abort && lane == 0) {
        for (int i = 0; i < kSlots; ++i)
            if (last_use[i] >= 0)
                mbar_wait_bounded(smem_u32(&sh.kv_full[i]), uint32_t(last_use[i]) & 1u);
        for (int i = 0; i < kQSlots; ++i)
            if (last_q[i] >= 0)
                mbar_wait_bounded(smem_u32(&sh.q_full[i]), uint32_t(last_q[i]) & 1u);
    }
}

// ------------------------------------------------------------ matrix unit
// One thread.  Two streams of tensor-core work: S^T(n) = K_n Q^T once K_n has
// landed and score buffer n % 2 is free, and O += P_n V_n once the softmax
// has written P_n and V_n has landed.  The thread polls both and
// issues whichever is ready, so a P.V never waits behind a later tile's K.
// A tile with fewer than 128 valid rows takes only the P.V steps that hold
// valid rows; the V rows past the end inside the last step are zeroed first.
struct PvInfo {
    int u, j, nt, valid;
};

__device__ __forceinline__ void mma_role(const Params &p, Shared &sh, uint32_t sbase, unsigned char *smem)
{
    constexpr uint32_t kIdS = idesc_f16_f32_mn(kT, kNQ, false, false);  // K-major K, K-major Q
    constexpr uint32_t kIdO = idesc_f16_f32_mn(128, kD, false, true);   // K-major P, N-major V
    volatile int *abort = &sh.abort;
    const uint32_t tmem = sh.tmem;
    int u = -1, j = 0, nt = 0, t0 = 0, t1 = 0;  // item and tile of the next score product
    bool need_item = true, more = true;
    int ns = 0, np = 0;                         // score products / P.V products issued
    PvInfo pend[4];
    uint64_t idle_since = 0;
    while (!*abort) {
        bool prog = false;
        if (need_item && more) {
            const int slot = (u + 1) % kItemRing;
            if (mbar_test_wait(smem_u32(&sh.item_full[slot]), uint32_t((u + 1) / kItemRing) & 1u)) {
                const Item it = sh.item[slot];
                mbar_arrive(smem_u32(&sh.item_empty[slot]));
                if (it.k < 0) {
                    more = false;
                } else {
                    ++u;
                    j = 0;
                    nt = chunk_tiles(it.c);
                    t0 = it.c.t0;
                    t1 = it.c.t1;
                    need_item = false;
                }
                prog = true;
            }
        }
        if (!need_item && ns - np < 4) {
            const int sb = ns & 1, ks = (2 * ns) % kSlots;
            if ((ns < 2 || mbar_test_wait(smem_u32(&sh.s_empty[sb]), uint32_t((ns >> 1) - 1) & 1u)) &&
                mbar_test_wait(smem_u32(&sh.q_full[u % kQSlots]), uint32_t(u / kQSlots) & 1u) &&
                mbar_test_wait(smem_u32(&sh.kv_full[ks]), uint32_t((2 * ns) / kSlots) & 1u)) {
                tc_fence_after_sync();
                const uint32_t ka = sbase + kOffKV + uint32_t(ks) * kTile;
                const uint32_t qa = sbase + kOffQ + uint32_t(u % kQSlots) * kQTile;
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint32_t kb = uint32_t(k >> 2), kk = uint32_t(k & 3) * 32u;
                    umma_f16(tmem + uint32_t(sb) * kNQ,
                             smem_desc_sw128(ka + kb * kAtom + kk, 16, kGroupStride),
                             smem_desc_sw128(qa + kb * kQHalf + kk, 16, 1024), kIdS, k > 0);
                }
                umma_commit(smem_u32(&sh.s_full[sb]));
                umma_commit(smem_u32(&sh.kv_empty[ks]));
                if (j == nt - 1)
                    umma_commit(smem_u32(&sh.q_empty[u % kQSlots]));
                pend[ns & 3] = PvInfo{u, j, nt, min(kT, t1 - (t0 + j * kT))};
                ++ns;
                if (++j == nt)
                    need_item = true;
                prog = true;
            }
        }
        if (np < ns) {
            const PvInfo f = pend[np & 3];
            const int vpos = 2 * np + 1;  // V(np)'s load position
            const int pb = np % kPBufs, ob = f.u & 1, vs = vpos % kSlots;
            if (mbar_test_wait(smem_u32(&sh.p_full[pb]), uint32_t(np / kPBufs) & 1u) &&
                mbar_test_wait(smem_u32(&sh.kv_full[vs]), uint32_t(vpos / kSlots) & 1u) &&
                (f.j > 0 || f.u < 2 ||
                 mbar_test_wait(smem_u32(&sh.o_empty[ob]), uint32_t((f.u >> 1) - 1) & 1u))) {
                const int steps = (f.valid + 15) / 16;
                if (f.valid < steps * 16) {  // zero V rows past the end inside the last step
                    unsigned char *vt = smem + kOffKV + uint32_t(vs) * kTile;
                    for (int r = f.valid; r < steps * 16; ++r) {
                        unsigned char *row = vt + uint32_t(r >> 3) * kGroupStride + uint32_t(r & 7) * 128u;
#pragma unroll
                        for (int c16 = 0; c16 < 8; ++c16) {
                            *reinterpret_cast<uint4 *>(row + c16 * 16) = make_uint4(0, 0, 0, 0);
                            *reinterpret_cast<uint4 *>(row + kAtom + c16 * 16) = make_uint4(0, 0, 0, 0);
                        }
                    }
                    fence_proxy_async_smem();
                }
                tc_fence_after_sync();
                const uint32_t va = sbase + kOffKV + uint32_t(vs) * kTile;
                const uint32_t pa = sbase + kOffP + uint32_t(pb) * kQTile;
                for (int k = 0; k < steps; ++k) {
                    const uint32_t kb = uint32_t(k >> 2), kk = uint32_t(k & 3) * 32u;
                    // A: P rows (8-row groups 1 KB apart), tokens 16k .. 16k+15;
                    // B: V rows 16k .. 16k+15 (8-row groups kGroupStride apart),
                    // the head dimension in two 64-wide halves kAtom apart
                    umma_f16(tmem + kTmemO + uint32_t(ob) * kD,
                             smem_desc_sw128(pa + kb * kQHalf + kk, 16, 1024),
                             smem_desc_sw128(va + uint32_t(k) * 2u * kGroupStride, kAtom, kGroupStride),
                             kIdO, f.j > 0 || k > 0);
                }
                umma_commit(smem_u32(&sh.p_empty[pb]));
                umma_commit(smem_u32(&sh.kv_empty[vs]));
                if (f.j == f.nt - 1)
                    umma_commit(smem_u32(&sh.o_full[ob]));
                ++np;
                prog = true;
            }
        }
        if (!more && need_item && np == ns)
            break;
        if (prog) {
            idle_since = 0;
        } else {
            const uint64_t t = global_timer_ns();
            if (idle_since == 0) {
                idle_since = t;
            } else if (t - idle_since > kWaitLimitNs) {
                atomicOr(p.error_word, PA_DEVERR_TIMEOUT);
                *abort = 1;
            }
        }
    }
    // every matrix operation issued has finished before TMEM and the shared
    // tiles are released
    umma_commit(smem_u32(&sh.drain));
    mbar_wait_bounded(smem_u32(&sh.drain), 0u);
}

// ---------------------------------------------------------------- softmax
// One tile for a thread holding token `row`.  NQ = 1 (a tail), 8 or 16 (a
// prefix slice, of which the first nq columns are real).  Returns false once
// a wait has failed; the next tile's (or item's) barrier then ends the role
// in all four warps together.
template <int NQ>
__device__ __forceinline__ bool softmax_tile(const Params &p, Shared &sh, unsigned char *smem,
                                             int warp, int lane, int n, int u, int j, int nq,
                                             int valid, float (&m_ref)[kNQ], float (&l)[kNQ])
{
    volatile int *abort = &sh.abort;
    unsigned int *err = p.error_word;
    const int row = warp * 32 + lane;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const int sb = n & 1;
    bool ok = gwait(smem_u32(&sh.s_full[sb]), uint32_t(n >> 1) & 1u, abort, err);
    tc_fence_after_sync();
    uint32_t s[16];
    tmem_load16_async(sh.tmem + uint32_t(sb) * kNQ + lane_base, s);
    tmem_wait_ld();
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0)
        mbar_arrive(smem_u32(&sh.s_empty[sb]));

    const bool live = row < valid;
    const float c = p.qk_scale_log2;
    float x[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q)
        x[q] = live ? __uint_as_float(s[q]) * c : -INFINITY;
    // tile max per column: warp reduction, then the four warps' maxima
    // through shared memory (double-buffered by tile parity) behind one
    // named barrier
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        const float wm = warp_max(x[q]);
        if (lane == q)
            sh.red[sb][warp][q] = wm;
    }
    if (!softmax_bar_and(ok))
        return false;
    float tm[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q)
        tm[q] = fmaxf(fmaxf(sh.red[sb][0][q], sh.red[sb][1][q]), fmaxf(sh.red[sb][2][q], sh.red[sb][3][q]));
    if (j == 0) {
#pragma unroll
        for (int q = 0; q < NQ; ++q)
            m_ref[q] = tm[q];
    } else {
        bool need = false;
#pragma unroll
        for (int q = 0; q < NQ; ++q)
            need |= q < nq && tm[q] > m_ref[q] + kRescaleLog2;
        if (need) {  // uniform: every thread sees the same maxima
            // move the reference: the partial sums (every thread) and the rows
            // of O (warp 0: TMEM lane q holds query q) are rescaled once the
            // previous P.V has completed
            ok = gwait(smem_u32(&sh.p_empty[(n - 1) % kPBufs]), uint32_t((n - 1) / kPBufs) & 1u, abort, err) &&
                 ok;
            tc_fence_after_sync();
            float a_lane = 1.f;
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const float mn = fmaxf(m_ref[q], tm[q]);
                const float alpha = ex2f(m_ref[q] - mn);
                m_ref[q] = mn;
                l[q] *= alpha;
                if (lane == q)
                    a_lane = alpha;
            }
            if (warp == 0) {
                const uint32_t tO = sh.tmem + kTmemO + uint32_t(u & 1) * kD;
#pragma unroll 1
                for (int c = 0; c < kD / 16; ++c) {
                    uint32_t o[16];
                    tmem_load16_async(tO + uint32_t(c) * 16u, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        o[e] = __float_as_uint(__uint_as_float(o[e]) * a_lane);
                    tmem_store16(tO + uint32_t(c) * 16u, o);
                }
                tmem_wait_st();
            }
        }
    }
    float pv[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        pv[q] = live ? ex2f(x[q] - m_ref[q]) : 0.f;
        l[q] += pv[q];
    }
    // P (row q = query, 128 tokens as K, 128-byte swizzle) into the tile's
    // operand buffer once the P.V kPBufs tiles back has read it
    const int pb = n % kPBufs;
    if (n >= kPBufs)
        ok = gwait(smem_u32(&sh.p_empty[pb]), uint32_t(n / kPBufs - 1) & 1u, abort, err) && ok;
    {
        unsigned char *pt = smem + kOffP + uint32_t(pb) * kQTile + uint32_t(row >> 6) * kQHalf;
        const int tt = row & 63;
#pragma unroll
        for (int q = 0; q < NQ; ++q)
            if (q < nq)
                *reinterpret_cast<__half *>(pt + q * 128 + ((((tt >> 3) ^ (q & 7))) << 4) + (tt & 7) * 2) =
                    __float2half_rn(pv[q]);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0)
        mbar_arrive(smem_u32(&sh.p_full[pb]));
    return ok;
}

__device__ __forceinline__ void softmax_role(const Params &p, Shared &sh, unsigned char *smem, int warp,
                                             int lane)
{
    volatile int *abort = &sh.abort;
    unsigned int *err = p.error_word;
    int n = 0;
    for (int u = 0;; ++u) {
        const int slot = u % kItemRing;
        const bool got = gwait(smem_u32(&sh.item_full[slot]), uint32_t(u / kItemRing) & 1u, abort, err);
        if (!softmax_bar_and(got))
            break;
        const Item it = sh.item[slot];
        __syncwarp();
        if (lane == 0)
            mbar_arrive(smem_u32(&sh.item_empty[slot]));
        float m_ref[kNQ], l[kNQ];
#pragma unroll
        for (int q = 0; q < kNQ; ++q) {
            m_ref[q] = -INFINITY;
            l[q] = 0.f;
        }
        bool ok = true;
        if (it.k >= 0) {
            const int nt = chunk_tiles(it.c), nq = it.c.nq;
            for (int j = 0; j < nt; ++j, ++n) {
                const int valid = min(kT, it.c.t1 - (it.c.t0 + j * kT));
                const bool r = nq == 1   ? softmax_tile<1>(p, sh, smem, warp, lane, n, u, j, 1, valid, m_ref, l)
                               : nq <= 8 ? softmax_tile<8>(p, sh, smem, warp, lane, n, u, j, nq, valid, m_ref, l)
                                         : softmax_tile<kNQ>(p, sh, smem, warp, lane, n, u, j, nq, valid, m_ref, l);
                ok = ok && r;
            }
        }
        // hand the item to the epilogue once it has taken the item two back
        Epi &e = sh.epi[u & 1];
        if (u >= 2)
            ok = gwait(smem_u32(&sh.o_empty[u & 1]), uint32_t((u >> 1) - 1) & 1u, abort, err) && ok;
        if (!softmax_bar_and(ok))
            break;
        if (it.k >= 0) {
#pragma unroll
            for (int q = 0; q < kNQ; ++q) {
                if (q < it.c.nq) {
                    const float sm = warp_sum(l[q]);
                    if (lane == 0)
                        e.l[warp][q] = sm;
                }
            }
        }
        if (warp == 0 && lane == 0) {
            e.c = it.c;
            e.h = it.h;
            e.end = it.k < 0;
#pragma unroll
            for (int q = 0; q < kNQ; ++q)
                e.m[q] = m_ref[q];
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(smem_u32(&sh.e_full[u & 1]));
        if (it.k < 0)
            break;
    }
}

// ---------------------------------------------------------------- epilogue
// Warp 4 (TMEM lanes 0-31), thread q = query row q of O: per item, the row
// (128 head dimensions) and the query's (m, l) go to the workspace.
__device__ __forceinline__ void epilogue_role(const Params &p, Shared &sh, int lane)
{
    volatile int *abort = &sh.abort;
    unsigned int *err = p.error_word;
    const int H = p.num_heads;
    const int q = lane < kNQ ? lane : 0;
    for (int u = 0;; ++u) {
        const bool got = gwait(smem_u32(&sh.e_full[u & 1]), uint32_t(u >> 1) & 1u, abort, err);
        if (!__all_sync(kFullMask, got))
            break;
        const Epi &e = sh.epi[u & 1];
        if (e.end)
            break;
        const Chunk c = e.c;
        const int h = e.h;
        const float m_q = e.m[q];
        const float l_q = (e.l[0][q] + e.l[1][q]) + (e.l[2][q] + e.l[3][q]);
        const bool ok = gwait(smem_u32(&sh.o_full[u & 1]), uint32_t(u >> 1) & 1u, abort, err);
        if (!__all_sync(kFullMask, ok))
            break;
        tc_fence_after_sync();
        const uint32_t tO = sh.tmem + kTmemO + uint32_t(u & 1) * kD;
        uint32_t o[kD];
        tmem_load32_into(tO, o);
        tmem_load32_into(tO + 32u, o + 32);
        tmem_load32_into(tO + 64u, o + 64);
        tmem_load32_into(tO + 96u, o + 96);
        tmem_wait_ld();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(smem_u32(&sh.o_empty[u & 1]));
        if (lane < c.nq) {
            float4 *dst = reinterpret_cast<float4 *>(p.part_o + (size_t(c.col + q) * H + h) * kD);
#pragma unroll
            for (int i = 0; i < kD / 4; ++i)
                dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                     __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
            reinterpret_cast<float2 *>(p.part_ml)[size_t(c.col + q) * H + h] = make_float2(m_q, l_q);
        }
    }
    // the partials are visible device-wide before the CTA counts itself done
    __threadfence();
}

__global__ void __launch_bounds__(kThreads, 1)
    grouped_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const Params p)
{
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(16) Shared sh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - raw);
    if (tid == 0) {
        for (int i = 0; i < kItemRing; ++i) {
            mbar_init(smem_u32(&sh.item_full[i]), 1);
            mbar_init(smem_u32(&sh.item_empty[i]), 1 + 4);  // the MMA thread and the softmax warps
        }
        for (int i = 0; i < kQSlots; ++i) {
            mbar_init(smem_u32(&sh.q_full[i]), 1);
            mbar_init(smem_u32(&sh.q_empty[i]), 1);
        }
        for (int i = 0; i < kPBufs; ++i) {
            mbar_init(smem_u32(&sh.p_full[i]), 4);
            mbar_init(smem_u32(&sh.p_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sh.s_full[i]), 1);
            mbar_init(smem_u32(&sh.s_empty[i]), 4);
            mbar_init(smem_u32(&sh.o_full[i]), 1);
            mbar_init(smem_u32(&sh.o_empty[i]), 1);
            mbar_init(smem_u32(&sh.e_full[i]), 4);
        }
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(smem_u32(&sh.kv_full[i]), 1);
            mbar_init(smem_u32(&sh.kv_empty[i]), 1);
        }
        mbar_init(smem_u32(&sh.drain), 1);
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp)
        tmem_alloc(smem_u32(&sh.tmem), kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    // the work list comes from the set-up kernel that precedes this one,
    // unless the kernel builds its own
    if (p.group_start == nullptr)
        grid_dependency_wait();
    allow_dependent_launch();

    if (warp == kLoadWarp) {
        load_role(&tm_q, &tm_k, &tm_v, p, sh, sbase, lane);
    } else if (warp == kMmaWarp) {
        if (lane == 0)
            mma_role(p, sh, sbase, smem);
        __syncwarp();
    } else if (warp < 4) {
        softmax_role(p, sh, smem, warp, lane);
    } else if (warp == kEpiWarp) {
        epilogue_role(p, sh, lane);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {  // this CTA's partials are all written (the merge waits for every CTA)
        __threadfence();
        atomicAdd(&p.meta->tc_done, 1u);
    }
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_free(sh.tmem, kTmemCols);
    }
}

} // namespace grp
} // namespace pa
