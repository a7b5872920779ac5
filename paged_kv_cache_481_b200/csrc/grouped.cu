// libpa, shared-prefix decode: C ABI of pa_decode_grouped.  Host code here
// validates arguments, lays out the workspace, encodes the TMA tensor maps
// and launches four kernels on the caller's stream:
//   * a one-CTA set-up kernel: each member's tail table (its block-table row
//     from the first block past the shared prefix), tail length and merge
//     record, zero outputs for empty contexts, and (beyond 32 groups) the
//     prefix work list (chunks);
//   * the persistent tensor-core kernel of grouped_kernel.cuh over the
//     prefix chunks, leaving (m, l, o) per member, head and chunk, on a
//     share of the SMs;
//   * the paged decode kernel over the tails, with each (member, head)'s
//     base-2 log-normaliser, on the other SMs at the same time;
//   * a merge kernel: the prefix partials and the tail result combined by
//     their softmax normalisers, once every prefix CTA has counted itself
//     done.
// The order is set-up, prefix, tails, merge, each launched as a programmatic
// dependent of the one before.  The tails start as soon as every prefix CTA
// is resident and wait for the prefix kernel only at their end.  With at
// most 32 groups the prefix kernel works out its own work list and does not
// wait for the set-up kernel, so it streams while the set-up kernel works out
// the tails; the tail decode then waits for the set-up kernel's `ready`
// flag before it starts (a dependency wait there would wait for the prefix
// kernel too: such a wait covers everything launched before).  Nothing here
// allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>

#include "../../include/pa.h"
#include "grouped_kernel.cuh"
#include "host_common.cuh"
#include "tma_host.cuh"

namespace {

using pa::grp::Chunk;
using pa::grp::Group;
using pa::grp::kChunk;
using pa::grp::kD;
using pa::grp::Member;
using pa::grp::Meta;

struct SetupParams {
    const int32_t *group_start;   // [G + 1]
    const int32_t *prefix_lens;   // [G]
    const int32_t *context_lens;  // [B]
    const int32_t *block_tables;  // [B, MB]
    int num_groups, num_seqs, max_context_len, block_size, num_heads, max_blocks;
    int max_chunks;               // capacity of `chunks` and of the partial columns
    int self_list;                // the prefix kernel builds its own work list and runs
                                  // beside this kernel: leave the header alone, raise `ready`
    __half *out;                  // rows of empty contexts are zeroed here
    Meta *meta;
    Group *groups;                // used without the shared-memory working set
    Member *members;
    Chunk *chunks;
    int32_t *tail_tables;         // [B, MB]
    int32_t *tail_lens;           // [B]
    int32_t *group_of;            // [B] each member's group (-1: none); likewise
    unsigned int *dec_tickets;    // [B, H] merge tickets of the tail decode, cleared here
    unsigned int *err;
};

constexpr int kSetupThreads = 1024;

// Dynamic shared memory of the set-up kernel when its whole working set --
// the group records, bounds and prefixes, each member's group, tail length
// and context length, and the block-table rows -- fits in it (0: it does
// not, and the workspace and the inputs serve instead).
constexpr size_t kSetupSmemMax = 200u * 1024u;

size_t setup_smem_bytes(int num_groups, int num_seqs, int max_blocks)
{
    const size_t bytes = size_t(num_groups) * (sizeof(Group) + 2 * sizeof(int32_t)) + sizeof(int32_t) +
                         size_t(num_seqs) * 3 * sizeof(int32_t) +
                         size_t(num_seqs) * size_t(max_blocks) * sizeof(int32_t);
    return bytes <= kSetupSmemMax ? bytes : 0;
}

// Share of the SMs the prefix kernel runs on; the tail decode takes the
// rest.  Which part is larger is known only on the device, so the split is
// fixed: a prefix SM streams a little slower than a decode SM (its pipeline
// holds fewer tiles in flight), and this share balances prefixes and tails
// of similar size (parallel samples of a prompt with tails of a few
// hundred tokens).  On 8 groups of 8 with ~1000-token prefixes and tails
// of 1-256 tokens, 0.50 suits copy-on-write tables (each tail also holds
// the copied last prefix block) and 0.55 fully aliased ones.
constexpr float kPrefixSmShare = 0.53f;

// With its own work list (at most kSelfListMaxGroups groups: one per lane of
// its load warp) the prefix kernel streams several microseconds before the
// tails start, and takes a smaller share.
constexpr int kSelfListMaxGroups = 32;
constexpr float kSelfListSmShare = 0.49f;

__device__ __forceinline__ int clamp_len(const SetupParams &p, int raw)
{
    if (raw < 0 || raw > p.max_context_len) {
        atomicOr(p.err, PA_DEVERR_CONTEXT_LEN);
        return raw < 0 ? 0 : p.max_context_len;
    }
    return raw;
}

// Exclusive scans of the groups' chunk counts (pstart) and partial-column
// counts (colbase) by one warp, 32 groups a step; returns the totals.
__device__ int2 warp_scan_groups(Group *gr, int G, int lane)
{
    int carry_p = 0, carry_c = 0;
    for (int base = 0; base < G; base += 32) {
        const int i = base + lane;
        const int vp = i < G ? gr[i].pstart : 0, vc = i < G ? gr[i].colbase : 0;
        int xp = vp, xc = vc;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int yp = __shfl_up_sync(pa::kFullMask, xp, off);
            const int yc = __shfl_up_sync(pa::kFullMask, xc, off);
            if (lane >= off) {
                xp += yp;
                xc += yc;
            }
        }
        if (i < G) {
            gr[i].pstart = carry_p + xp - vp;
            gr[i].colbase = carry_c + xc - vc;
        }
        carry_p += __shfl_sync(pa::kFullMask, xp, 31);
        carry_c += __shfl_sync(pa::kFullMask, xc, 31);
    }
    return make_int2(carry_p, carry_c);
}

// Group g with members g0 .. g0+n-1 and a valid prefix P (a multiple of the
// block size, at most every member's context) gets ceil(P / 512) prefix
// chunks per slice of up to 16 members, read through the first member's
// table.  A prefix that breaks the rules is recorded (PA_DEVERR_CONTEXT_LEN)
// and the group decodes without one.  Member b's tail is tokens P .. L_b - 1
// of its own table: its tail table is that row from block P / bs on.
// The work is a few dependent steps over small arrays, so its time is set by
// round trips to memory, and a CTA barrier waits for every load and store
// its threads have outstanding.  With the working set in shared memory
// (kSmem) every input -- lengths, group bounds and prefixes, table rows --
// comes in at once in the first step, the groups are settled in shared
// memory, and every output is written after the last barrier: one round
// trip in all.  With at most 32 groups each warp scans the groups' counts
// itself (lane g holds group g) and needs no further barrier.
template <bool kSmem>
__global__ void __launch_bounds__(kSetupThreads) grouped_setup_kernel(const SetupParams p)
{
    extern __shared__ int4 setup_smem[];
    pa::grid_dependency_wait();
    pa::allow_dependent_launch();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.num_seqs, G = p.num_groups, bs = p.block_size, H = p.num_heads;
    const int MB = p.max_blocks;
    Group *gr;
    int32_t *gof, *tl, *len = nullptr, *gs = nullptr, *pl = nullptr, *rows = nullptr;
    if constexpr (kSmem) {
        gr = reinterpret_cast<Group *>(setup_smem);
        gs = reinterpret_cast<int32_t *>(gr + G);  // group bounds [G + 1]
        pl = gs + G + 1;                           // prefixes [G]
        gof = pl + G;                              // each member's group [B]
        tl = gof + B;                              // tail lengths [B]
        len = tl + B;                              // clamped context lengths [B]
        rows = len + B;                            // block-table rows [B, MB]
    } else {
        gr = p.groups;
        gof = p.group_of;
        tl = p.tail_lens;
    }

    // 1: the inputs in (one round trip)
    for (int b = tid; b < B; b += kSetupThreads) {
        gof[b] = -1;
        tl[b] = 0;
        if constexpr (kSmem)
            len[b] = clamp_len(p, p.context_lens[b]);
    }
    if constexpr (kSmem) {
        for (int g = tid; g <= G; g += kSetupThreads) {
            gs[g] = p.group_start[g];
            if (g < G)
                pl[g] = p.prefix_lens[g];
        }
        // loads before stores, so all go out at once
        const int entries = B * MB;
        constexpr int kBatch = 8;
        for (int base = 0; base < entries; base += kBatch * kSetupThreads) {
            int32_t v[kBatch];
#pragma unroll
            for (int r = 0; r < kBatch; ++r) {
                const int i = base + r * kSetupThreads + tid;
                v[r] = i < entries ? p.block_tables[i] : 0;
            }
#pragma unroll
            for (int r = 0; r < kBatch; ++r) {
                const int i = base + r * kSetupThreads + tid;
                if (i < entries)
                    rows[i] = v[r];
            }
        }
    }
    __syncthreads();
    auto length = [&](int b) {
        if constexpr (kSmem)
            return len[b];
        else
            return clamp_len(p, p.context_lens[b]);
    };

    // 2: per group (a warp each): bounds, prefix, tails
    for (int g = warp; g < G; g += kSetupThreads / 32) {
        int g0, g1, P;
        if constexpr (kSmem) {
            g0 = gs[g];
            g1 = gs[g + 1];
            P = pl[g];
        } else {
            g0 = p.group_start[g];
            g1 = p.group_start[g + 1];
            P = p.prefix_lens[g];
        }
        const bool okg = 0 <= g0 && g0 <= g1 && g1 <= B;
        if (!okg && lane == 0)
            atomicOr(p.err, PA_DEVERR_CONTEXT_LEN);
        int min_len = INT_MAX;
        if (okg)
            for (int b = g0 + lane; b < g1; b += 32)
                min_len = min(min_len, length(b));
        min_len = __reduce_min_sync(pa::kFullMask, min_len);
        const pa::grp::GroupPlan gp = pa::grp::plan_group(g0, g1, P, min_len, B, bs);
        if (!gp.prefix_ok && gp.n > 0 && P != 0 && lane == 0)
            atomicOr(p.err, PA_DEVERR_CONTEXT_LEN);
        for (int b = gp.g0 + lane; b < gp.g0 + gp.n; b += 32) {
            gof[b] = g;
            tl[b] = length(b) - gp.P;
        }
        if (lane == 0)  // colbase and pstart hold counts until the scan turns them into offsets
            gr[g] = Group{gp.g0, gp.n, gp.cp, gp.P, gp.n * gp.cp, gp.slices * gp.cp, 0, 0};
    }
    __syncthreads();

    // 3: the offsets: lane g of every warp holds group g's (at most 32
    // groups), else one warp scans in place behind a barrier
    const bool small = G <= 32;
    int xp = 0, xc = 0, nchunks, ncols;
    if (small) {
        const int vp = lane < G ? gr[lane].pstart : 0, vc = lane < G ? gr[lane].colbase : 0;
        xp = vp;
        xc = vc;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int yp = __shfl_up_sync(pa::kFullMask, xp, off);
            const int yc = __shfl_up_sync(pa::kFullMask, xc, off);
            if (lane >= off) {
                xp += yp;
                xc += yc;
            }
        }
        nchunks = __shfl_sync(pa::kFullMask, xp, 31);
        ncols = __shfl_sync(pa::kFullMask, xc, 31);
        xp -= vp;  // exclusive
        xc -= vc;
    } else {
        __shared__ int2 s_tot;
        if (warp == 0) {
            const int2 tot = warp_scan_groups(gr, G, lane);
            if (lane == 0)
                s_tot = tot;
        }
        __syncthreads();
        nchunks = s_tot.x;
        ncols = s_tot.y;
    }
    // group g's (first chunk, first partial column)
    auto offsets = [&](int g) {
        return small ? make_int2(__shfl_sync(pa::kFullMask, xp, g & 31), __shfl_sync(pa::kFullMask, xc, g & 31))
                     : make_int2(gr[g].pstart, gr[g].colbase);
    };
    const bool fits = nchunks <= p.max_chunks && ncols <= p.max_chunks;
    if (!fits) {  // cannot happen with the host's bound; refuse rather than overrun
        if (tid == 0) {
            atomicOr(p.err, PA_DEVERR_CONTEXT_LEN);
            if (!p.self_list) {
                p.meta->nchunks = 0;
                p.meta->ncols = 0;
            } else {
                atomicExch(&p.meta->ready, 1u);
            }
        }
        return;
    }

    // 4: every output: per member (a warp each) its record, tail length and
    // tail table (entry k is entry P / bs + k of its table row), zero rows
    // for empty contexts; the chunk descriptors; the decode's merge tickets;
    // the header
    for (int b = warp; b < B; b += kSetupThreads / 32) {
        const int g = gof[b];
        const Group gg = g >= 0 ? gr[g] : Group{0, 0, 0, 0, 0, 0, 0, 0};
        const int2 off = offsets(g >= 0 ? g : 0);
        const int tail = tl[b];
        const int pb = gg.P / bs;
        int32_t *trow = p.tail_tables + size_t(b) * MB;
        if constexpr (kSmem) {
            const int32_t *row = rows + b * MB;
            for (int k = lane; k < MB; k += 32)
                trow[k] = pb + k < MB ? row[pb + k] : -1;
        } else {  // loads before stores
            const int32_t *__restrict__ row = p.block_tables + size_t(b) * MB;
            constexpr int kBatch = 4;
            for (int k0 = 0; k0 < MB; k0 += 32 * kBatch) {
                int32_t v[kBatch];
#pragma unroll
                for (int r = 0; r < kBatch; ++r) {
                    const int k = k0 + r * 32 + lane;
                    v[r] = k < MB && pb + k < MB ? row[pb + k] : -1;
                }
#pragma unroll
                for (int r = 0; r < kBatch; ++r) {
                    const int k = k0 + r * 32 + lane;
                    if (k < MB)
                        trow[k] = v[r];
                }
            }
        }
        if (lane == 0) {
            p.members[b] = g >= 0 ? Member{tail, gg.cp, off.y + (b - gg.g0), gg.n} : Member{-1, 0, 0, 0};
            if constexpr (kSmem)
                p.tail_lens[b] = tail;
        }
        if (g >= 0 && tail + gg.P == 0) {  // nothing to attend to: the output is zero
            uint4 *o = reinterpret_cast<uint4 *>(p.out + size_t(b) * H * kD);
            for (int e = lane; e < H * kD / 8; e += 32)
                o[e] = make_uint4(0, 0, 0, 0);
        }
    }
    for (int g = warp; g < G; g += kSetupThreads / 32) {
        const Group gg = gr[g];
        const int2 off = offsets(g);
        const int slices = (gg.n + 15) / 16;
        for (int idx = lane; idx < slices * gg.cp; idx += 32) {
            const int j = idx / slices, s = idx % slices;
            p.chunks[off.x + idx] =
                Chunk{gg.g0, gg.g0 + 16 * s, min(16, gg.n - 16 * s), j * kChunk,
                      min((j + 1) * kChunk, gg.P), g, off.y + j * gg.n + 16 * s, 0};
        }
    }
    for (int i = tid; i < B * H; i += kSetupThreads)
        p.dec_tickets[i] = 0u;
    if (!p.self_list) {  // the prefix kernel's work list; it starts after this kernel
        if (tid == 0) {
            p.meta->nchunks = nchunks;
            p.meta->ncols = ncols;
            p.meta->claimed = 0;
        }
    } else {  // the tail decode is already running and waits for this flag
        __threadfence();
        __syncthreads();
        if (tid == 0)
            atomicExch(&p.meta->ready, 1u);
    }
}

// out[b, h] = (sum_j 2^(m_j - M) o_j + 2^(lse_t - M) o_t) /
//             (sum_j 2^(m_j - M) l_j + 2^(lse_t - M)),  M the largest exponent:
// the prefix chunks' partials (m_j, l_j, o_j unnormalised, fp32) and the
// tail's normalised fp16 result with its log-normaliser lse_t.  An empty
// part has weight 0.  One warp per (member, head), four dims per lane.
__device__ __forceinline__ void merge_unit(__half *__restrict__ out, const Member *__restrict__ members,
                                           const float *__restrict__ part_ml, const float *__restrict__ part_o,
                                           const __half *__restrict__ o_t, const float *__restrict__ lse_t,
                                           int num_heads, int unit, int lane)
{
    const int b = unit / num_heads, h = unit % num_heads;
    // the tail's result does not depend on the member record: load both at once
    const uint2 raw = reinterpret_cast<const uint2 *>(o_t + size_t(unit) * kD)[lane];
    const float lse = lse_t[unit];
    const Member mb = members[b];
    if (mb.tail < 0 || mb.cp + mb.tail == 0)
        return;  // in no group, or an empty context (zeroed by the set-up kernel)
    constexpr int kBatch = 4;
    float M = -INFINITY, den = 0.f, num[4] = {0.f, 0.f, 0.f, 0.f};
    auto add = [&](float m, float l, const float (&x)[4]) {
        const float mn = fmaxf(M, m);
        const float a = exp2f(M - mn), f = exp2f(m - mn);
        M = mn;
        den = fmaf(den, a, f * l);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            num[e] = fmaf(num[e], a, f * x[e]);
    };
    for (int j0 = 0; j0 < mb.cp; j0 += kBatch) {
        float2 v[kBatch];
        float4 o[kBatch];
#pragma unroll
        for (int c = 0; c < kBatch; ++c) {
            if (j0 + c < mb.cp) {
                const size_t ix = size_t(mb.col0 + (j0 + c) * mb.stride) * num_heads + h;
                v[c] = reinterpret_cast<const float2 *>(part_ml)[ix];
                o[c] = reinterpret_cast<const float4 *>(part_o + ix * kD)[lane];
            }
        }
#pragma unroll
        for (int c = 0; c < kBatch; ++c) {
            if (j0 + c < mb.cp) {
                const float x[4] = {o[c].x, o[c].y, o[c].z, o[c].w};
                add(v[c].x, v[c].y, x);
            }
        }
    }
    if (mb.tail > 0) {
        const float2 t01 = __half22float2(*reinterpret_cast<const __half2 *>(&raw.x));
        const float2 t23 = __half22float2(*reinterpret_cast<const __half2 *>(&raw.y));
        const float x[4] = {t01.x, t01.y, t23.x, t23.y};
        add(lse, 1.f, x);
    }
    const float inv = 1.f / den;
    const __half2 r01 = __floats2half2_rn(num[0] * inv, num[1] * inv);
    const __half2 r23 = __floats2half2_rn(num[2] * inv, num[3] * inv);
    uint2 res;
    res.x = *reinterpret_cast<const uint32_t *>(&r01);
    res.y = *reinterpret_cast<const uint32_t *>(&r23);
    reinterpret_cast<uint2 *>(out + size_t(unit) * kD)[lane] = res;
}

// The merge runs after the tail decode (programmatic dependent launch), which
// itself completes only after the prefix kernel.  Each CTA also checks (with
// a bounded wait) that all tc_ctas prefix CTAs have counted themselves done
// before it reads their partials.  Once every merge CTA is past that check,
// the last one sets the work-list counters and flag back to zero for the
// next call.
__global__ void __launch_bounds__(256) grouped_merge_kernel(
    __half *__restrict__ out, const Member *__restrict__ members, const float *__restrict__ part_ml,
    const float *__restrict__ part_o, const __half *__restrict__ o_t, const float *__restrict__ lse_t,
    int num_heads, int units, Meta *meta, unsigned int tc_ctas, unsigned int *err)
{
    pa::grid_dependency_wait();
    pa::allow_dependent_launch();
    if (threadIdx.x == 0) {
        volatile unsigned int *done = &meta->tc_done;
        bool ok = *done >= tc_ctas;
        if (!ok) {
            const uint64_t t0 = pa::global_timer_ns();
            while (!(ok = *done >= tc_ctas) && pa::global_timer_ns() - t0 < pa::kWaitLimitNs)
                __nanosleep(64);
        }
        if (!ok)
            atomicOr(err, PA_DEVERR_TIMEOUT);
        __threadfence();
    }
    __syncthreads();
    const int unit = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (unit < units)
        merge_unit(out, members, part_ml, part_o, o_t, lse_t, num_heads, unit, lane);
    if (threadIdx.x == 0 && atomicAdd(&meta->merge_done, 1u) == gridDim.x - 1) {
        meta->claimed = 0;
        meta->tc_done = 0u;
        meta->ready = 0u;
        meta->merge_done = 0u;
    }
}

// Workspace of pa_decode_grouped: work-list header, group and member
// records, prefix chunk descriptors, the prefix partials (reference max and
// sum, and the fp32 output, per column and head), the tail tables and
// lengths, the tail decode's own workspace, and its outputs and
// log-normalisers.  Prefix chunks and columns are each at most
// B ceil(max_context_len / 512): at most one column per member per 512
// prefix tokens.
struct Layout {
    size_t meta, groups, members, group_of, chunks, part_ml, part_o, tail_tables, tail_lens, dec,
        o_t, lse_t, total;
    int max_chunks;
};

Layout layout(int num_seqs, int num_groups, int num_heads, int max_context_len, int max_blocks)
{
    Layout w{};
    const size_t per_member = size_t((max_context_len + kChunk - 1) / kChunk);
    const size_t cap = size_t(num_seqs) * (per_member > 0 ? per_member : 1);
    const size_t units = size_t(num_seqs) * size_t(num_heads);
    w.max_chunks = cap > size_t(INT_MAX) ? INT_MAX : int(cap);
    // what the set-up kernel writes first and together, the large partial
    // buffers after it
    w.meta = 0;
    w.groups = align256(sizeof(Meta));
    w.members = w.groups + align256(size_t(num_groups) * sizeof(Group));
    w.group_of = w.members + align256(size_t(num_seqs) * sizeof(Member));
    w.chunks = w.group_of + align256(size_t(num_seqs) * sizeof(int32_t));
    w.tail_tables = w.chunks + align256(cap * sizeof(Chunk));
    w.tail_lens = w.tail_tables + align256(size_t(num_seqs) * size_t(max_blocks) * sizeof(int32_t));
    w.part_ml = w.tail_lens + align256(size_t(num_seqs) * sizeof(int32_t));
    w.lse_t = w.part_ml + align256(cap * num_heads * 2 * sizeof(float));
    w.o_t = w.lse_t + align256(units * sizeof(float));
    w.part_o = w.o_t + align256(units * kD * 2);
    w.dec = w.part_o + align256(cap * num_heads * kD * sizeof(float));
    w.total = w.dec + align256(pa_decode_workspace_size(num_seqs, num_heads, kD, max_context_len));
    return w;
}

} // namespace

extern "C" size_t pa_decode_grouped_workspace_size(int num_seqs, int num_groups, int num_heads,
                                                   int head_dim, int max_context_len,
                                                   int max_blocks_per_seq)
{
    if (num_seqs < 0 || num_groups < 0 || num_heads < 0 || head_dim < 0 || max_context_len < 0 ||
        max_blocks_per_seq < 0)
        return 0;
    return layout(num_seqs, num_groups, num_heads, max_context_len, max_blocks_per_seq).total;
}

extern "C" pa_status pa_decode_grouped(void *out, const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       int max_blocks_per_seq, const int32_t *context_lens,
                                       int max_context_len, const int32_t *group_start,
                                       const int32_t *prefix_lens, int num_groups,
                                       int max_group_size, int num_seqs, int num_heads,
                                       int head_dim, int block_size, int num_blocks, float scale,
                                       void *workspace, size_t workspace_bytes, pa_stream_t stream)
{
    if (num_seqs < 0 || num_groups < 0 || max_group_size < 0 || num_heads <= 0 ||
        num_blocks <= 0 || max_context_len < 0 || max_blocks_per_seq < 0)
        return PA_ERR_INVALID_ARG;
    if (head_dim != kD || !supported_block_size(block_size))
        return PA_ERR_UNSUPPORTED;
    if (int64_t(max_context_len) > int64_t(max_blocks_per_seq) * block_size ||
        !std::isfinite(scale) || !(scale > 0.f) || (num_seqs > 0 && num_groups == 0) ||
        num_groups > num_seqs)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0)
        return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !group_start ||
        !prefix_lens || max_group_size == 0)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u) ||
        (reinterpret_cast<uintptr_t>(group_start) & 3u) ||
        (reinterpret_cast<uintptr_t>(prefix_lens) & 3u))
        return PA_ERR_INVALID_ARG;
    if (num_seqs > 65535 || num_heads > 65535 || max_group_size > 65535 ||
        int64_t(num_blocks) * num_heads * block_size > INT32_MAX ||
        int64_t(num_heads) * ((max_context_len + kChunk - 1) / kChunk + 1) * num_seqs > INT32_MAX ||
        int64_t(num_seqs) * max_blocks_per_seq > INT32_MAX - 65536)
        return PA_ERR_INVALID_ARG;
    const Layout w = layout(num_seqs, num_groups, num_heads, max_context_len, max_blocks_per_seq);
    if (!workspace || workspace_bytes < w.total || !aligned16(workspace))
        return PA_ERR_WORKSPACE;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    unsigned int *err = device_error_word();
    if (!err)
        return PA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return PA_ERR_CUDA;
    static std::atomic<int> sm_count[kMaxDevices];  // 0 = not configured yet
    int sms = sm_count[dev].load(std::memory_order_acquire);
    if (sms == 0) {
        if (cudaFuncSetAttribute(pa::grp::grouped_decode_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(pa::grp::kSmem)) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_setup_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(kSetupSmemMax)) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            sms <= 0)
            return PA_ERR_CUDA;
        sm_count[dev].store(sms, std::memory_order_release);
    }

    CUtensorMap tm_q, tm_k, tm_v;
    const uint64_t cache_rows = uint64_t(num_blocks) * num_heads * block_size;
    const uint32_t box_rows = uint32_t(block_size < pa::grp::kT ? block_size : pa::grp::kT);
    if (!make_map(&tm_q, q, uint64_t(num_heads) * head_dim, uint64_t(num_seqs),
                  uint64_t(num_heads) * head_dim * 2, pa::grp::kNQ) ||
        !make_kv_map(&tm_k, k_cache, cache_rows, box_rows) ||
        !make_kv_map(&tm_v, v_cache, cache_rows, box_rows))
        return PA_ERR_CUDA;

    Meta *meta = reinterpret_cast<Meta *>(ws + w.meta);
    Group *groups = reinterpret_cast<Group *>(ws + w.groups);
    Member *members = reinterpret_cast<Member *>(ws + w.members);
    float *part_ml = reinterpret_cast<float *>(ws + w.part_ml);
    float *part_o = reinterpret_cast<float *>(ws + w.part_o);
    int32_t *tail_tables = reinterpret_cast<int32_t *>(ws + w.tail_tables);
    int32_t *tail_lens = reinterpret_cast<int32_t *>(ws + w.tail_lens);
    __half *o_t = reinterpret_cast<__half *>(ws + w.o_t);
    float *lse_t = reinterpret_cast<float *>(ws + w.lse_t);

    // With at most 32 groups the prefix kernel builds its own work list and
    // starts without waiting for the set-up kernel, so it streams while the
    // set-up kernel works out the tails; the tail decode then waits for the
    // set-up kernel's `ready` flag instead.  Otherwise the prefix kernel runs
    // on the set-up kernel's list, after it.
    const bool self_list = num_groups <= kSelfListMaxGroups;

    SetupParams sp{};
    sp.group_start = group_start;
    sp.prefix_lens = prefix_lens;
    sp.context_lens = context_lens;
    sp.block_tables = block_tables;
    sp.num_groups = num_groups;
    sp.num_seqs = num_seqs;
    sp.max_context_len = max_context_len;
    sp.block_size = block_size;
    sp.num_heads = num_heads;
    sp.max_blocks = max_blocks_per_seq;
    sp.max_chunks = w.max_chunks;
    sp.self_list = self_list ? 1 : 0;
    const size_t setup_smem = setup_smem_bytes(num_groups, num_seqs, max_blocks_per_seq);
    sp.out = static_cast<__half *>(out);
    sp.meta = meta;
    sp.groups = groups;
    sp.members = members;
    sp.chunks = reinterpret_cast<Chunk *>(ws + w.chunks);
    sp.tail_tables = tail_tables;
    sp.tail_lens = tail_lens;
    sp.group_of = reinterpret_cast<int32_t *>(ws + w.group_of);
    sp.dec_tickets = reinterpret_cast<unsigned int *>(
        ws + w.dec + pa_host::decode_ticket_offset(num_seqs, num_heads, kD));
    sp.err = err;
    auto launch_setup = [&]() {
        return (setup_smem > 0
                    ? launch_pdl(grouped_setup_kernel<true>, dim3(1), dim3(kSetupThreads), setup_smem, s, sp)
                    : launch_pdl(grouped_setup_kernel<false>, dim3(1), dim3(kSetupThreads), 0, s, sp)) ==
               cudaSuccess;
    };

    pa::grp::Params p{};
    p.out = static_cast<__half *>(out);
    p.block_tables = block_tables;
    p.chunks = sp.chunks;
    p.meta = meta;
    p.max_chunks = w.max_chunks;
    if (self_list) {
        p.group_start = group_start;
        p.prefix_lens = prefix_lens;
        p.context_lens = context_lens;
        p.num_groups = num_groups;
        p.num_seqs = num_seqs;
        p.max_context_len = max_context_len;
    }
    p.part_ml = part_ml;
    p.part_o = part_o;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_heads = num_heads;
    p.block_size = block_size;
    p.num_blocks = num_blocks;
    p.qk_scale_log2 = float(double(scale) * 1.4426950408889634);
    p.error_word = err;
    const float share = self_list ? kSelfListSmShare : kPrefixSmShare;
    const int prefix_ctas = std::max(1, std::min(sms - 1, int(float(sms) * share + 0.5f)));
    auto launch_prefix = [&]() {
        return launch_pdl(pa::grp::grouped_decode_kernel, dim3(unsigned(prefix_ctas)),
                          dim3(pa::grp::kThreads), pa::grp::kSmem, s, tm_q, tm_k, tm_v, p) == cudaSuccess;
    };

    // 1. the tails (and the work list); 2. the shared prefixes, once per
    // (group, head), on the tensor cores
    if (!launch_setup() || !launch_prefix())
        return PA_ERR_CUDA;

    // 3. each member's own tail, on the remaining SMs at the same time: it
    // starts as soon as every prefix CTA is resident and waits for the
    // prefix kernel only at its end (and, beside a prefix kernel on its own
    // list, for the set-up kernel's `ready` flag first)
    static std::atomic<int> dec_per_sm[kMaxDevices];  // 0 = not configured yet
    int per_sm = dec_per_sm[dev].load(std::memory_order_acquire);
    if (per_sm == 0) {
        per_sm = pa_host::decode_ctas_per_sm();
        if (per_sm <= 0)
            return PA_ERR_CUDA;
        dec_per_sm[dev].store(per_sm, std::memory_order_release);
    }
    const pa_status st = pa_host::decode_with_lse(
        o_t, q, k_cache, v_cache, tail_tables, max_blocks_per_seq, tail_lens, max_context_len,
        num_seqs, num_heads, head_dim, block_size, num_blocks, scale, ws + w.dec, w.total - w.dec, lse_t,
        stream, per_sm * (sms - prefix_ctas), true, self_list ? &meta->ready : nullptr);
    if (st != PA_OK)
        return st;

    // 4. merge the parts, once the prefix kernel's CTAs are all done
    const int units = num_seqs * num_heads;
    return launch_pdl(grouped_merge_kernel, dim3(unsigned((units + 7) / 8)), dim3(256), 0, s,
                      static_cast<__half *>(out), static_cast<const Member *>(members),
                      static_cast<const float *>(part_ml),
                      static_cast<const float *>(part_o), static_cast<const __half *>(o_t),
                      static_cast<const float *>(lse_t), num_heads, units, meta,
                      unsigned(prefix_ctas), err) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}
