// Paged single-token decode attention for sm_100a.
//
// What it computes (comfyai.app "6.4 PagedAttention", 6.4.1; polomodov.tech
// "vLLM and PagedAttention", slides 9-10; brentwoodlivery.com 5.3.18 on the
// attention arithmetic being unchanged by paging): for sequence b, head h and
// t < L_b, K_t / V_t are row t % bs of physical block block_tables[b][t / bs];
// out = softmax(scale * q.K) V.
//
// How — a persistent kernel with an even split of the work:
//   * The work is the flattened list of tiles over all (sequence, head)
//     units, unit by unit (b-major, then h); a tile is 4 KB of K plus 4 KB of
//     V (16 tokens at D = 128, 32 at D = 64), which inside one (block, head)
//     is one contiguous run in HBM.  Every warp of the grid is an independent
//     worker that owns an equal contiguous range of that list (+-1 tile), so
//     all workers finish together whatever the length mix.
//   * Each CTA first counts the tiles of every sequence (a scan over
//     context_lens) to find its warps' ranges; after that there is no
//     CTA-wide synchronisation.
//   * A worker streams its range through an S-stage ring of shared-memory
//     buffers filled by 1-D bulk copies (the TMA engine) with one mbarrier
//     per stage.  Lane 0 looks the block ids up one tile ahead (a register
//     prefetch; the first S tiles' lookups are issued by S lanes at once),
//     issues the copies and writes the tile's coordinates next to the
//     buffer; the q row of a (sequence, head) travels with its first tile.
//     Only valid rows of a partial block are fetched.
//   * QK: lanes split a row into 16-byte chunks and use the mixed-precision
//     FMA (f16 inputs, f32 accumulate, no conversions); per-row partial dot
//     products are combined with a transposing shuffle reduction (8 shuffles
//     for 16 rows); scores in the log2 domain (scale * log2 e applied once
//     per score).  Online softmax (running max m, sum l) with fp32 P.V.
//   * A (sequence, head) that lies inside one worker's range is written
//     straight to out.  One that straddles ranges (at most the first and the
//     last of each worker) leaves (m, l, o[D]) in the workspace; the last
//     contributor — found with a self-resetting atomic ticket — merges the
//     contributions in worker order (deterministic) and writes out.
//   * Every wait is bounded; on expiry the worker records PA_DEVERR_TIMEOUT,
//     lets its copies in flight land and stops.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"

namespace pa {

__device__ unsigned int g_device_error;

__device__ __forceinline__ void raise_device_error(unsigned int bits)
{
    atomicOr(&g_device_error, bits);
}

constexpr unsigned kErrBlockId = 1u << 0;
constexpr unsigned kErrContextLen = 1u << 1;
constexpr unsigned kErrTimeout = 1u << 4;

constexpr int kTileBytes = 4096;  // one K (or V) tile in shared memory
constexpr int kMaxWorkers = 4096; // warps per grid; sizes the workspace

struct DecodeParams {
    __half *out;
    const __half *q;
    const __half *k_cache;
    const __half *v_cache;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *ws_o;         // [kMaxWorkers, 2, D] partial outputs of straddling units
    float *ws_ml;        // [kMaxWorkers, 2, 2] their (max in log2 units, sum)
    unsigned *ws_count;  // [B*H] merge tickets, zero between calls
    int num_seqs;
    int max_blocks_per_seq;
    int max_context_len;
    int num_heads;
    int block_size;
    int num_blocks;
    float qk_scale_log2; // softmax scale * log2(e)
};

template <int D>
struct DecodeShape {
    static constexpr int kTokens = kTileBytes / (D * 2);  // rows per tile
    static constexpr int kChunks = D / 8;                 // 16-byte chunks per row
    static constexpr int kRowsPerStep = 32 / kChunks;     // rows one warp load covers
    static constexpr int kIters = kTokens / kRowsPerStep; // warp loads per tile
    static constexpr int kLogChunks = kChunks == 16 ? 4 : 3;
    static constexpr int kLogIters = kIters == 8 ? 3 : (kIters == 4 ? 2 : 1);
    // after the transposing reduction, kDup adjacent lanes hold the same row
    static constexpr int kDup = 1 << (kLogChunks - kLogIters);
    static constexpr int kMaxIds = 4;                     // block ids one tile can span (bs >= 8)
    static_assert(kChunks * kRowsPerStep == 32, "a warp covers whole rows");
    static_assert(kLogChunks >= kLogIters, "reduction keeps one row per lane group");
    static_assert(kTokens / 8 <= kMaxIds, "tile spans at most kMaxIds blocks of 8");
};

// Where one staged tile comes from; written by lane 0 before it arms the
// stage's barrier, read by the whole warp after the barrier completes.
struct TileMeta {
    int b, h, i, len;  // sequence, head, tile index in the unit, context length
    long long k;       // global tile index
};

template <int D, int NW, int S>
struct DecodeSmem {
    static constexpr size_t kStageBytes = 2 * kTileBytes + D * 2;  // K, V, q row
    static constexpr size_t kTiles = size_t(NW) * S * kStageBytes;
    static constexpr size_t kBars = size_t(NW) * S * sizeof(uint64_t);
    static constexpr size_t kMeta = size_t(NW) * S * sizeof(TileMeta);
    static constexpr size_t kBytes = kTiles + kBars + kMeta;
    static constexpr int kThreads = NW * 32;
};

__device__ __forceinline__ float2 h2f(uint32_t bits)
{
    __half2 h = *reinterpret_cast<const __half2 *>(&bits);
    return __half22float2(h);
}

// q . k over one 16-byte chunk (8 fp16 each), fp32 accumulation.
__device__ __forceinline__ float dot8(const uint4 &q, const uint4 &k)
{
    float s0 = fma2_f16_f32(q.x, k.x, 0.f);
    float s1 = fma2_f16_f32(q.y, k.y, 0.f);
    s0 = fma2_f16_f32(q.z, k.z, s0);
    s1 = fma2_f16_f32(q.w, k.w, s1);
    return s0 + s1;
}

__device__ __forceinline__ void axpy8(float (&acc)[8], float w, const uint4 &u)
{
    const float2 a = h2f(u.x), b = h2f(u.y), c = h2f(u.z), d = h2f(u.w);
    acc[0] = fmaf(w, a.x, acc[0]);
    acc[1] = fmaf(w, a.y, acc[1]);
    acc[2] = fmaf(w, b.x, acc[2]);
    acc[3] = fmaf(w, b.y, acc[3]);
    acc[4] = fmaf(w, c.x, acc[4]);
    acc[5] = fmaf(w, c.y, acc[5]);
    acc[6] = fmaf(w, d.x, acc[6]);
    acc[7] = fmaf(w, d.y, acc[7]);
}

// Consume one staged tile: scores, online-softmax update and PV accumulate.
// Lane (r, c) = (lane / kChunks, lane % kChunks) handles rows i*kRowsPerStep + r
// and dims [8c, 8c + 8).
template <int D, bool kFull>
__device__ __forceinline__ void consume_tile(const uint4 *__restrict__ ks, const uint4 *__restrict__ vs,
                                             int valid_rows, int r, int c, const uint4 &qh,
                                             float qk_scale_log2, float &m, float &l_part,
                                             float (&acc)[8])
{
    using S = DecodeShape<D>;
    float v[S::kIters];
#pragma unroll
    for (int i = 0; i < S::kIters; ++i)
        v[i] = dot8(qh, ks[(i * S::kRowsPerStep + r) * S::kChunks + c]);

    // Transposing reduction over the kChunks lanes of a row group: each step
    // halves the number of values a lane holds while summing across lanes.
#pragma unroll
    for (int step = 0; step < S::kLogChunks; ++step) {
        const int off = S::kChunks >> (step + 1);
        const int n = S::kIters >> step;
        if (n >= 2) {
            const bool upper = (c & off) != 0;
#pragma unroll
            for (int j = 0; j < n / 2; ++j) {
                const float send = upper ? v[j] : v[j + n / 2];
                const float keep = upper ? v[j + n / 2] : v[j];
                v[j] = keep + __shfl_xor_sync(kFullMask, send, off);
            }
        } else {
            v[0] += __shfl_xor_sync(kFullMask, v[0], off);
        }
    }
    const int my_row = (c / S::kDup) * S::kRowsPerStep + r;
    float s = v[0] * qk_scale_log2;
    if (!kFull && my_row >= valid_rows)
        s = -INFINITY;

    float tile_max = s;
#pragma unroll
    for (int off = 16; off >= S::kDup; off >>= 1)
        tile_max = fmaxf(tile_max, __shfl_xor_sync(kFullMask, tile_max, off));
    const float m_new = fmaxf(m, tile_max);
    const float alpha = exp2f(m - m_new);
    const float w = exp2f(s - m_new);
    l_part = l_part * alpha + ((c % S::kDup) == 0 ? w : 0.f);
#pragma unroll
    for (int k = 0; k < 8; ++k)
        acc[k] *= alpha;

#pragma unroll
    for (int i = 0; i < S::kIters; ++i) {
        const float wi = __shfl_sync(kFullMask, w, r * S::kChunks + i * S::kDup);
        if (kFull || i * S::kRowsPerStep + r < valid_rows)
            axpy8(acc, wi, vs[(i * S::kRowsPerStep + r) * S::kChunks + c]);
    }
    m = m_new;
}

__device__ __forceinline__ int clamp_len(int len, int max_len)
{
    return len < 0 ? 0 : (len > max_len ? max_len : len);
}

// Worker owning global tile t when `workers` workers split `total` tiles:
// worker w owns [floor(w*total/workers), floor((w+1)*total/workers)).
__device__ __forceinline__ long long worker_of(long long t, long long total, long long workers)
{
    return ((t + 1) * workers - 1) / total;
}

__device__ __forceinline__ long long range_start(long long w, long long total, long long workers)
{
    return w * total / workers;
}

// Walks the flattened (sequence, head, tile) list.
struct TileCursor {
    long long k;   // global tile index
    int b, h, i;   // sequence, head, tile within the unit
    int len, nt;   // context length of b and its tiles per head

    template <int T>
    __device__ __forceinline__ void advance(const DecodeParams &p)
    {
        ++k;
        if (++i < nt)
            return;
        i = 0;
        if (++h < p.num_heads)
            return;
        h = 0;
        do {  // sequences of length 0 own no tiles
            ++b;
            len = clamp_len(p.context_lens[b], p.max_context_len);
        } while (len == 0);
        nt = (len + T - 1) / T;
    }
};

// Block ids of the tile under the cursor, loaded one tile ahead of their use;
// they are range-checked when the copies are issued.
template <int D>
__device__ __forceinline__ void load_tile_ids(const DecodeParams &p, const TileCursor &cur,
                                              int (&ids)[DecodeShape<D>::kMaxIds])
{
    using Sh = DecodeShape<D>;
    const int bs = p.block_size;
    const int t0 = cur.i * Sh::kTokens;
    const int nv = min(Sh::kTokens, cur.len - t0);
    const int first = t0 / bs;
    const int nsub = bs >= Sh::kTokens ? 1 : (nv + bs - 1) / bs;
    const int32_t *row = p.block_tables + size_t(cur.b) * p.max_blocks_per_seq;
#pragma unroll
    for (int s = 0; s < Sh::kMaxIds; ++s)
        ids[s] = s < nsub ? row[first + s] : 0;
}

// Arm the stage's full barrier and issue the bulk copies of the tile under
// the cursor (K rows, V rows, and the q row when `with_q`).  K and V are read
// exactly once, so they go through L2 with an evict-first policy that keeps
// the small reused data (block tables, q, split partials) resident.
template <int D>
__device__ __forceinline__ void issue_tile(const DecodeParams &p, const TileCursor &cur,
                                           const int (&ids)[DecodeShape<D>::kMaxIds], bool with_q,
                                           unsigned char *stage_buf, uint32_t bar, TileMeta *meta,
                                           uint64_t stream_policy)
{
    using Sh = DecodeShape<D>;
    const int bs = p.block_size;
    const int t0 = cur.i * Sh::kTokens;
    const int nv = min(Sh::kTokens, cur.len - t0);
    meta->b = cur.b;
    meta->h = cur.h;
    meta->i = cur.i;
    meta->len = cur.len;
    meta->k = cur.k;

    const uint32_t kdst = smem_u32(stage_buf);
    const uint32_t vdst = kdst + kTileBytes;
    const uint32_t qdst = kdst + 2 * kTileBytes;
    const size_t head_stride = size_t(bs) * D;  // elements between heads of a block
    // an id outside the pool is recorded and its rows are not fetched
    bool ok[Sh::kMaxIds];
#pragma unroll
    for (int s = 0; s < Sh::kMaxIds; ++s)
        ok[s] = unsigned(ids[s]) < unsigned(p.num_blocks);
    uint32_t total = with_q ? uint32_t(D * 2) : 0u;
    bool bad = false;
    if (bs >= Sh::kTokens) {
        if (ok[0])
            total += 2u * uint32_t(nv) * D * 2;
        else
            bad = true;
    } else {
#pragma unroll
        for (int s = 0; s < Sh::kMaxIds; ++s) {
            if (s * bs >= nv)
                break;
            if (ok[s])
                total += 2u * uint32_t(min(bs, nv - s * bs)) * D * 2;
            else
                bad = true;
        }
    }
    if (bad)
        raise_device_error(kErrBlockId);
    mbar_arrive_expect_tx(bar, total);
    if (with_q)
        bulk_copy_g2s(qdst, p.q + (size_t(cur.b) * p.num_heads + cur.h) * D, D * 2, bar);
    if (bs >= Sh::kTokens) {
        if (ok[0]) {
            const uint32_t bytes = uint32_t(nv) * D * 2;
            const size_t off = (size_t(ids[0]) * p.num_heads + cur.h) * head_stride + size_t(t0 % bs) * D;
            bulk_copy_g2s_hint(kdst, p.k_cache + off, bytes, bar, stream_policy);
            bulk_copy_g2s_hint(vdst, p.v_cache + off, bytes, bar, stream_policy);
        }
    } else {
#pragma unroll
        for (int s = 0; s < Sh::kMaxIds; ++s) {
            if (s * bs >= nv)
                break;
            if (!ok[s])
                continue;
            const uint32_t bytes = uint32_t(min(bs, nv - s * bs)) * D * 2;
            const size_t off = (size_t(ids[s]) * p.num_heads + cur.h) * head_stride;
            const uint32_t sub = uint32_t(s) * bs * D * 2;
            bulk_copy_g2s_hint(kdst + sub, p.k_cache + off, bytes, bar, stream_policy);
            bulk_copy_g2s_hint(vdst + sub, p.v_cache + off, bytes, bar, stream_policy);
        }
    }
}

// Merge the partial results of a (sequence, head) whose tiles were split
// between workers w_first..w_last, in worker order, and write out.  One pass:
// each contribution rescales the running sums to the running maximum, so all
// loads are independent.  Lanes with r == 0 each handle 8 dims.
template <int D>
__device__ __forceinline__ void merge_partials(const DecodeParams &p, uint4 *out_row, int c,
                                               long long u_start, long long w_first,
                                               long long w_last, long long total,
                                               long long workers)
{
    float gmax = -INFINITY, den = 0.f;
    float num[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (long long w = w_first; w <= w_last; ++w) {
        const size_t q = size_t(w) * 2 + (u_start <= range_start(w, total, workers) ? 0 : 1);
        const float mw = __ldcg(p.ws_ml + q * 2), lw = __ldcg(p.ws_ml + q * 2 + 1);
        const float4 *po = reinterpret_cast<const float4 *>(p.ws_o + q * D + 8 * c);
        const float4 x = __ldcg(po), y = __ldcg(po + 1);
        const float m_new = fmaxf(gmax, mw);
        const float a = exp2f(gmax - m_new), f = exp2f(mw - m_new);
        gmax = m_new;
        den = fmaf(den, a, f * lw);
        num[0] = fmaf(num[0], a, f * x.x);
        num[1] = fmaf(num[1], a, f * x.y);
        num[2] = fmaf(num[2], a, f * x.z);
        num[3] = fmaf(num[3], a, f * x.w);
        num[4] = fmaf(num[4], a, f * y.x);
        num[5] = fmaf(num[5], a, f * y.y);
        num[6] = fmaf(num[6], a, f * y.z);
        num[7] = fmaf(num[7], a, f * y.w);
    }
    __half2 o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
        o[k] = __floats2half2_rn(num[2 * k] / den, num[2 * k + 1] / den);
    out_row[c] = *reinterpret_cast<const uint4 *>(o);
}

template <int D, int NW, int S>
__global__ void __launch_bounds__(NW * 32) paged_decode_kernel(const DecodeParams p)
{
    using Sh = DecodeShape<D>;
    using Sm = DecodeSmem<D, NW, S>;
    constexpr int T = Sh::kTokens;
    constexpr int kThreads = Sm::kThreads;
    constexpr int kWarps = NW;

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ long long s_warp_sum[kWarps];
    __shared__ long long s_total;
    __shared__ int s_start_b[NW];
    __shared__ long long s_start_cum[NW];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.num_heads, B = p.num_seqs;
    if (blockDim.x != kThreads) {  // launched with the wrong shape: do nothing
        if (tid == 0 && blockIdx.x == 0)
            raise_device_error(kErrTimeout);
        return;
    }

    // Inputs may come from the previous kernel in the stream: read none before
    // it has finished.  The next kernel may start launching meanwhile.
    grid_dependency_wait();
    allow_dependent_launch();

    // Bring the small inputs every worker looks up (context lengths, block
    // tables, q) into L2 while the scan below runs; the CTAs split the lines.
    {
        const size_t g = size_t(blockIdx.x) * kThreads + tid, stride = size_t(gridDim.x) * kThreads;
        const size_t table_lines = (size_t(B) * p.max_blocks_per_seq * 4 + 127) / 128;
        const size_t q_lines = (size_t(B) * H * D * 2 + 127) / 128;
        const size_t len_lines = (size_t(B) * 4 + 127) / 128;
        for (size_t i = g; i < table_lines + q_lines + len_lines; i += stride) {
            if (i < table_lines)
                prefetch_l2(reinterpret_cast<const char *>(p.block_tables) + i * 128);
            else if (i < table_lines + q_lines)
                prefetch_l2(reinterpret_cast<const char *>(p.q) + (i - table_lines) * 128);
            else
                prefetch_l2(reinterpret_cast<const char *>(p.context_lens) + (i - table_lines - q_lines) * 128);
        }
    }

    // ---- 1. total tile count (and zero outputs of empty sequences) --------
    long long mine = 0, first_chunk = 0;
    for (int b = tid; b < B; b += kThreads) {
        const int raw = p.context_lens[b];
        const int len = clamp_len(raw, p.max_context_len);
        if (raw != len && blockIdx.x == 0)
            raise_device_error(kErrContextLen);
        const long long t = (long long)((len + T - 1) / T) * H;
        if (b == tid)
            first_chunk = t;
        mine += t;
        if (len == 0 && b % gridDim.x == blockIdx.x) {
            uint4 *o = reinterpret_cast<uint4 *>(p.out + size_t(b) * H * D);
            for (int e = 0; e < H * D / 8; ++e)
                o[e] = make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        mine += __shfl_xor_sync(kFullMask, mine, off);
    if (lane == 0)
        s_warp_sum[warp] = mine;
    __syncthreads();
    if (tid == 0) {
        long long t = 0;
        for (int w = 0; w < kWarps; ++w)
            t += s_warp_sum[w];
        s_total = t;
    }
    __syncthreads();
    const long long total = s_total;
    const long long workers = min((long long)gridDim.x * NW, total);

    // ---- 2. locate the sequence holding each worker's first tile ----------
    long long carry = 0;
    for (int base = 0; base < B; base += kThreads) {
        const int b = base + tid;
        long long t = 0;
        if (base == 0)
            t = first_chunk;
        else if (b < B)
            t = (long long)((clamp_len(p.context_lens[b], p.max_context_len) + T - 1) / T) * H;
        long long incl = t;  // inclusive scan within the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long y = __shfl_up_sync(kFullMask, incl, off);
            if (lane >= off)
                incl += y;
        }
        __syncthreads();  // s_warp_sum reuse
        if (lane == 31)
            s_warp_sum[warp] = incl;
        __syncthreads();
        long long before = carry;
        for (int w = 0; w < warp; ++w)
            before += s_warp_sum[w];
        const long long excl = before + incl - t;
        if (t > 0) {
            for (int w = 0; w < NW; ++w) {
                const long long wg = (long long)blockIdx.x * NW + w;
                if (wg < workers) {
                    const long long wlo = range_start(wg, total, workers);
                    if (excl <= wlo && wlo < excl + t) {
                        s_start_b[w] = b;
                        s_start_cum[w] = excl;
                    }
                }
            }
        }
        for (int w = 0; w < kWarps; ++w)
            carry += s_warp_sum[w];
    }

    // ---- 3. barriers ------------------------------------------------------
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Sm::kTiles);
    TileMeta *metas = reinterpret_cast<TileMeta *>(smem + Sm::kTiles + Sm::kBars);
    if (tid < NW * S)
        mbar_init(smem_u32(&full[tid]), 1);
    fence_mbar_init();
    __syncthreads();

    const long long gw = (long long)blockIdx.x * NW + warp;
    if (gw >= workers)
        return;
    const long long lo = range_start(gw, total, workers);
    const long long hi = range_start(gw + 1, total, workers);
    const int ntiles = int(hi - lo);
    unsigned char *my_buf = smem + size_t(warp) * S * Sm::kStageBytes;
    const uint32_t my_bar = smem_u32(&full[warp * S]);
    TileMeta *my_meta = metas + warp * S;
    const int r = lane / Sh::kChunks, c = lane % Sh::kChunks;

    // ---- 4. fill the ring: lane s walks to this warp's s-th tile and loads
    // its block ids, so the first S lookups are in flight together; lane 0
    // issues the copies.
    TileCursor prod;
    prod.b = s_start_b[warp];
    prod.len = clamp_len(p.context_lens[prod.b], p.max_context_len);
    prod.nt = (prod.len + T - 1) / T;
    {
        const long long off = lo - s_start_cum[warp];
        prod.h = int(off / prod.nt);
        prod.i = int(off % prod.nt);
    }
    prod.k = lo;
    const int first = min(S, ntiles);
    const uint64_t policy = l2_policy_evict_first();
    int ids[Sh::kMaxIds];
    {
        TileCursor mc = prod;
        for (int s = 0; s < first - 1; ++s)
            if (s < lane)
                mc.template advance<T>(p);
        if (lane < first)
            load_tile_ids<D>(p, mc, ids);
        __syncwarp();
        for (int s = 0; s < first; ++s) {
            TileCursor cs;
            cs.k = __shfl_sync(kFullMask, mc.k, s);
            cs.b = __shfl_sync(kFullMask, mc.b, s);
            cs.h = __shfl_sync(kFullMask, mc.h, s);
            cs.i = __shfl_sync(kFullMask, mc.i, s);
            cs.len = __shfl_sync(kFullMask, mc.len, s);
            cs.nt = __shfl_sync(kFullMask, mc.nt, s);
            int ids_s[Sh::kMaxIds];
#pragma unroll
            for (int e = 0; e < Sh::kMaxIds; ++e)
                ids_s[e] = __shfl_sync(kFullMask, ids[e], s);
            if (lane == 0)
                issue_tile<D>(p, cs, ids_s, cs.i == 0 || cs.k == lo,
                              my_buf + size_t(s) * Sm::kStageBytes, my_bar + 8 * s, my_meta + s,
                              policy);
            if (s == first - 1)
                prod = cs;
        }
    }
    int issued = first;
    if (issued < ntiles) {
        prod.template advance<T>(p);
        load_tile_ids<D>(p, prod, ids);
    }

    // ---- 5. stream --------------------------------------------------------
    uint4 qh = make_uint4(0, 0, 0, 0);
    float m = -INFINITY, l_part = 0.f;
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        acc[k] = 0.f;
    int seg_i0 = 0;
    for (int j = 0; j < ntiles; ++j) {
        const int stage = j % S;
        const bool ok = mbar_wait_bounded(my_bar + 8 * stage, uint32_t(j / S) & 1u);
        if (!__all_sync(kFullMask, ok)) {
            // Record the failure and let every copy already in flight land
            // before the CTA's shared memory is released.
            if (lane == 0)
                raise_device_error(kErrTimeout);
            for (int jj = j; jj < issued; ++jj)
                mbar_wait_bounded(my_bar + 8 * (jj % S), uint32_t(jj / S) & 1u);
            return;
        }
        const TileMeta mt = my_meta[stage];
        const int nt = (mt.len + T - 1) / T;
        const int nv = min(T, mt.len - mt.i * T);
        const unsigned char *buf = my_buf + size_t(stage) * Sm::kStageBytes;
        if (mt.i == 0 || mt.k == lo) {  // first tile of a segment: fresh state, new q
            qh = reinterpret_cast<const uint4 *>(buf + 2 * kTileBytes)[c];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                acc[k] = 0.f;
            m = -INFINITY;
            l_part = 0.f;
            seg_i0 = mt.i;
        }
        const uint4 *ks = reinterpret_cast<const uint4 *>(buf);
        const uint4 *vs = ks + kTileBytes / 16;
        if (nv == T)
            consume_tile<D, true>(ks, vs, nv, r, c, qh, p.qk_scale_log2, m, l_part, acc);
        else
            consume_tile<D, false>(ks, vs, nv, r, c, qh, p.qk_scale_log2, m, l_part, acc);
        __syncwarp();
        if (issued < ntiles) {  // refill the stage just consumed
            if (lane == 0) {
                fence_proxy_async_smem();
                issue_tile<D>(p, prod, ids, prod.i == 0 || prod.k == lo,
                              my_buf + size_t(stage) * Sm::kStageBytes, my_bar + 8 * stage,
                              my_meta + stage, policy);
            }
            if (++issued < ntiles) {
                prod.template advance<T>(p);
                load_tile_ids<D>(p, prod, ids);
            }
        }
        if (!(mt.i == nt - 1 || mt.k == hi - 1))
            continue;

        // ---- end of a segment: finish this (sequence, head) or publish it
        float l = l_part;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
            l += __shfl_xor_sync(kFullMask, l, off);
#pragma unroll
        for (int off = Sh::kChunks; off < 32; off <<= 1)
#pragma unroll
            for (int k = 0; k < 8; ++k)
                acc[k] += __shfl_xor_sync(kFullMask, acc[k], off);
        const size_t unit = size_t(mt.b) * H + mt.h;
        uint4 *out_row = reinterpret_cast<uint4 *>(p.out + unit * D);
        if (seg_i0 == 0 && mt.i == nt - 1) {
            if (r == 0) {
                __half2 o[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    o[k] = __floats2half2_rn(acc[2 * k] / l, acc[2 * k + 1] / l);
                out_row[c] = *reinterpret_cast<const uint4 *>(o);
            }
            continue;
        }
        const long long u_start = mt.k - mt.i;      // global index of the unit's tile 0
        const int slot = u_start <= lo ? 0 : 1;     // first or last segment of this worker
        const size_t pidx = size_t(gw) * 2 + slot;
        if (r == 0) {
            float4 *po = reinterpret_cast<float4 *>(p.ws_o + pidx * D + 8 * c);
            po[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            po[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        if (lane == 0) {
            p.ws_ml[pidx * 2 + 0] = m;
            p.ws_ml[pidx * 2 + 1] = l;
        }
        __threadfence();
        __syncwarp();
        const long long w_first = worker_of(u_start, total, workers);
        const long long w_last = worker_of(u_start + nt - 1, total, workers);
        unsigned last = 0;
        if (lane == 0) {
            const unsigned n = unsigned(w_last - w_first);  // contributors - 1
            last = atomicInc(&p.ws_count[unit], n) == n;
        }
        if (!__shfl_sync(kFullMask, last, 0))
            continue;
        __threadfence();
        if (r == 0)
            merge_partials<D>(p, out_row, c, u_start, w_first, w_last, total, workers);
    }
}

} // namespace pa
