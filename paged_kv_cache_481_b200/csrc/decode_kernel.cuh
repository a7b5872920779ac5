// Paged single-token decode attention for sm_100a.
//
// What it computes (comfyai.app "6.4 PagedAttention", 6.4.1; polomodov.tech
// "vLLM and PagedAttention", slides 9-10; brentwoodlivery.com 5.3.18 on the
// attention arithmetic being unchanged by paging): for sequence b, head h and
// t < L_b, K_t / V_t are row t % bs of physical block block_tables[b][t / bs];
// out = softmax(scale * q.K) V.
//
// How (one CTA per (context partition, head, sequence)):
//   * the partition's slice of the block table is staged in shared memory
//     first, so the block-id -> address step never sits behind a global load
//     inside the stream loop;
//   * each warp owns every NW-th tile of the partition (a tile is 4 KB of K
//     and 4 KB of V: 16 tokens at D = 128, 32 at D = 64; within one (block,
//     head) those rows are contiguous in HBM) and keeps its own S-stage ring
//     of shared-memory buffers filled by 1-D bulk copies (the TMA engine),
//     one mbarrier per stage; only the valid rows of a partial block are
//     fetched;
//   * QK: lanes split a row into 16-byte chunks; per-row partial dot products
//     are combined with a transposing shuffle reduction (8 shuffles for 16
//     rows), scores kept in the log2 domain (scale * log2 e folded into q);
//   * online softmax per warp (running max m, running sum l, fp32 acc over
//     the lane's 8 dims), then the NW warps are merged in shared memory;
//   * a sequence with one partition writes fp16 out directly; otherwise each
//     partition stores (m, l, o[D]) in the workspace and the last CTA of the
//     (sequence, head) to finish — found with a self-resetting atomic ticket —
//     merges all partitions in partition order (deterministic) and writes
//     out.  No second kernel launch.
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

constexpr int kTileBytes = 4096;     // one K (or V) tile in shared memory
constexpr int kMaxTableSlice = 256;  // block-table entries staged per partition

struct DecodeParams {
    __half *out;
    const __half *q;
    const __half *k_cache;
    const __half *v_cache;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *ws_o;         // [B*H, max_parts, D] un-normalised partial outputs
    float *ws_ml;        // [B*H, max_parts, 2] (running max in log2 units, sum)
    unsigned *ws_count;  // [B*H] merge tickets, zero between calls
    int max_blocks_per_seq;
    int max_context_len;
    int num_heads;
    int block_size;
    int num_blocks;
    int partition_size;  // tokens per partition, multiple of the tile and of block_size
    int max_parts;
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
    static_assert(kChunks * kRowsPerStep == 32, "a warp covers whole rows");
    static_assert(kLogChunks >= kLogIters, "reduction keeps one row per lane group");
};

__device__ __forceinline__ float2 h2f(uint32_t bits)
{
    __half2 h = *reinterpret_cast<const __half2 *>(&bits);
    return __half22float2(h);
}

__device__ __forceinline__ float dot8(const float (&q)[8], const uint4 &u)
{
    const float2 a = h2f(u.x), b = h2f(u.y), c = h2f(u.z), d = h2f(u.w);
    float s0 = q[0] * a.x;
    float s1 = q[1] * a.y;
    s0 = fmaf(q[2], b.x, s0);
    s1 = fmaf(q[3], b.y, s1);
    s0 = fmaf(q[4], c.x, s0);
    s1 = fmaf(q[5], c.y, s1);
    s0 = fmaf(q[6], d.x, s0);
    s1 = fmaf(q[7], d.y, s1);
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
                                             int valid_rows, int r, int c, const float (&qf)[8],
                                             float &m, float &l_part, float (&acc)[8])
{
    using S = DecodeShape<D>;
    float v[S::kIters];
#pragma unroll
    for (int i = 0; i < S::kIters; ++i)
        v[i] = dot8(qf, ks[(i * S::kRowsPerStep + r) * S::kChunks + c]);

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
    float s = v[0];
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

template <int D, int NW, int S>
struct DecodeSmem {
    static constexpr int kTileElems = kTileBytes / 2;
    static constexpr size_t kTileRegion = size_t(NW) * S * 2 * kTileBytes;
    static constexpr size_t kBytes = kTileRegion + size_t(NW) * S * sizeof(uint64_t);
};

// Issue the bulk copies of warp `warp`'s j-th tile of the partition into
// stage j % S of its ring (called by one lane).  Only the rows below the
// context length are fetched; ids marked bad (-1) are skipped, with the
// barrier told the reduced byte count.
template <int D, int NW, int S>
__device__ __forceinline__ void issue_tile(const DecodeParams &p, const int *s_table, unsigned char *my_buf,
                                           uint32_t my_bar, int j, int warp, int h, int t_begin,
                                           int t_end, int blk_begin)
{
    using Sh = DecodeShape<D>;
    const int bs = p.block_size;
    const size_t head_stride = size_t(bs) * D;  // elements between heads of a block
    const int stage = j % S;
    const int t0 = t_begin + (warp + j * NW) * Sh::kTokens;
    const int nv = min(Sh::kTokens, t_end - t0);
    const uint32_t kdst = smem_u32(my_buf + size_t(stage) * 2 * kTileBytes);
    const uint32_t vdst = kdst + kTileBytes;
    const uint32_t bar = my_bar + 8 * stage;
    if (bs >= Sh::kTokens) {
        const int id = s_table[t0 / bs - blk_begin];
        const uint32_t bytes = id >= 0 ? uint32_t(nv) * D * 2 : 0u;
        mbar_arrive_expect_tx(bar, 2 * bytes);
        if (bytes) {
            const size_t off = (size_t(id) * p.num_heads + h) * head_stride + size_t(t0 % bs) * D;
            bulk_copy_g2s(kdst, p.k_cache + off, bytes, bar);
            bulk_copy_g2s(vdst, p.v_cache + off, bytes, bar);
        }
    } else {
        const int nsub = (nv + bs - 1) / bs;
        uint32_t total = 0;
        for (int s = 0; s < nsub; ++s)
            if (s_table[t0 / bs + s - blk_begin] >= 0)
                total += uint32_t(min(bs, nv - s * bs)) * D * 2;
        mbar_arrive_expect_tx(bar, 2 * total);
        for (int s = 0; s < nsub; ++s) {
            const int id = s_table[t0 / bs + s - blk_begin];
            if (id < 0)
                continue;
            const uint32_t bytes = uint32_t(min(bs, nv - s * bs)) * D * 2;
            const size_t off = (size_t(id) * p.num_heads + h) * head_stride;
            const uint32_t sub = uint32_t(s) * bs * D * 2;
            bulk_copy_g2s(kdst + sub, p.k_cache + off, bytes, bar);
            bulk_copy_g2s(vdst + sub, p.v_cache + off, bytes, bar);
        }
    }
}

template <int D, int NW, int S>
__global__ void __launch_bounds__(NW * 32) paged_decode_kernel(const DecodeParams p)
{
    using Sh = DecodeShape<D>;
    using Sm = DecodeSmem<D, NW, S>;
    static_assert(NW * 32 >= D, "one thread per output dim in the merge");

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int s_table[kMaxTableSlice];
    __shared__ float s_red_m[NW], s_red_l[NW];
    __shared__ __align__(16) float s_red_acc[NW][D];
    __shared__ int s_is_last;

    const int part = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int H = p.num_heads, bs = p.block_size;
    const int tid = threadIdx.x;

    int L = p.context_lens[b];
    if (L < 0 || L > p.max_context_len) {
        if (part == 0 && h == 0 && tid == 0)
            raise_device_error(1u << 1);
        L = L < 0 ? 0 : p.max_context_len;
    }
    const size_t unit = size_t(b) * H + h;
    __half *out_row = p.out + unit * D;
    if (L == 0) {
        if (part == 0)
            for (int t = tid; t < D; t += NW * 32)
                out_row[t] = __float2half_rn(0.f);
        return;
    }
    const int P = p.partition_size;
    const int nparts = (L + P - 1) / P;
    if (part >= nparts)
        return;
    const int t_begin = part * P;
    const int t_end = min(L, t_begin + P);
    const int ntiles = (t_end - t_begin + Sh::kTokens - 1) / Sh::kTokens;

    // Stage this partition's block-table slice; bad ids are recorded and
    // never dereferenced.
    const int blk_begin = t_begin / bs;
    const int nblk = (t_end - 1) / bs - blk_begin + 1;
    const int32_t *trow = p.block_tables + size_t(b) * p.max_blocks_per_seq + blk_begin;
    for (int i = tid; i < nblk; i += NW * 32) {
        int id = trow[i];
        if (unsigned(id) >= unsigned(p.num_blocks)) {
            raise_device_error(1u << 0);
            id = -1;
        }
        s_table[i] = id;
    }
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Sm::kTileRegion);
    if (tid == 0) {
        for (int i = 0; i < NW * S; ++i)
            mbar_init(smem_u32(&bars[i]), 1);
        fence_mbar_init();
    }
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    const int r = lane / Sh::kChunks, c = lane % Sh::kChunks;

    float qf[8];
    {
        const uint4 qv = reinterpret_cast<const uint4 *>(p.q + unit * D)[c];
        const float2 a = h2f(qv.x), bb = h2f(qv.y), cc = h2f(qv.z), dd = h2f(qv.w);
        qf[0] = a.x; qf[1] = a.y; qf[2] = bb.x; qf[3] = bb.y;
        qf[4] = cc.x; qf[5] = cc.y; qf[6] = dd.x; qf[7] = dd.y;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            qf[k] *= p.qk_scale_log2;
    }

    const int my_tiles = ntiles > warp ? (ntiles - 1 - warp) / NW + 1 : 0;
    unsigned char *my_buf = smem + size_t(warp) * S * 2 * kTileBytes;
    const uint32_t my_bar = smem_u32(&bars[warp * S]);
    if (lane == 0) {
        const int first = my_tiles < S ? my_tiles : S;
        for (int j = 0; j < first; ++j)
            issue_tile<D, NW, S>(p, s_table, my_buf, my_bar, j, warp, h, t_begin, t_end, blk_begin);
    }

    float m = -INFINITY, l_part = 0.f;
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        acc[k] = 0.f;

    int j = 0;
    bool aborted = false;
    for (; j < my_tiles; ++j) {
        const int stage = j % S;
        const bool ok = mbar_wait_bounded(my_bar + 8 * stage, uint32_t(j / S) & 1u);
        if (!__all_sync(kFullMask, ok)) {
            aborted = true;
            break;
        }
        const int t0 = t_begin + (warp + j * NW) * Sh::kTokens;
        const int nv = min(Sh::kTokens, t_end - t0);
        const uint4 *ks = reinterpret_cast<const uint4 *>(my_buf + size_t(stage) * 2 * kTileBytes);
        const uint4 *vs = ks + kTileBytes / 16;
        if (nv == Sh::kTokens)
            consume_tile<D, true>(ks, vs, nv, r, c, qf, m, l_part, acc);
        else
            consume_tile<D, false>(ks, vs, nv, r, c, qf, m, l_part, acc);
        __syncwarp();
        if (lane == 0 && j + S < my_tiles) {
            fence_proxy_async_smem();
            issue_tile<D, NW, S>(p, s_table, my_buf, my_bar, j + S, warp, h, t_begin, t_end,
                                 blk_begin);
        }
    }
    if (aborted) {
        // Record the failure and let every copy already in flight land before
        // the CTA's shared memory is released.
        if (lane == 0)
            raise_device_error(1u << 4);
        const int last = min(j + S, my_tiles);
        for (int jj = j; jj < last; ++jj)
            mbar_wait_bounded(my_bar + 8 * (jj % S), uint32_t(jj / S) & 1u);
    }

    // Warp totals: l over all lanes, acc across the row groups.
    float l = l_part;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        l += __shfl_xor_sync(kFullMask, l, off);
#pragma unroll
    for (int off = Sh::kChunks; off < 32; off <<= 1)
#pragma unroll
        for (int k = 0; k < 8; ++k)
            acc[k] += __shfl_xor_sync(kFullMask, acc[k], off);
    if (r == 0) {
        float4 *dst = reinterpret_cast<float4 *>(&s_red_acc[warp][8 * c]);
        dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
    if (lane == 0) {
        s_red_m[warp] = m;
        s_red_l[warp] = l;
    }
    __syncthreads();

    // Merge the warps (a warp with no tile has m = -inf and contributes 0).
    float o = 0.f, lsum = 0.f, mmax = -INFINITY;
    if (tid < D) {
#pragma unroll
        for (int w = 0; w < NW; ++w)
            mmax = fmaxf(mmax, s_red_m[w]);
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float f = exp2f(s_red_m[w] - mmax);
            o = fmaf(f, s_red_acc[w][tid], o);
            lsum = fmaf(f, s_red_l[w], lsum);
        }
    }
    if (nparts == 1) {
        if (tid < D)
            out_row[tid] = __float2half_rn(o / lsum);
        return;
    }

    // Split-K: publish this partition, then the last CTA of the (b, h) merges.
    const size_t slot = unit * p.max_parts + part;
    if (tid < D) {
        p.ws_o[slot * D + tid] = o;
        if (tid == 0) {
            p.ws_ml[slot * 2 + 0] = mmax;
            p.ws_ml[slot * 2 + 1] = lsum;
        }
        __threadfence();
    }
    __syncthreads();
    if (tid == 0) {
        const unsigned ticket = atomicInc(&p.ws_count[unit], unsigned(nparts - 1));
        s_is_last = ticket == unsigned(nparts - 1);
    }
    __syncthreads();
    if (!s_is_last)
        return;
    __threadfence();
    if (tid < D) {
        const float *ml = p.ws_ml + unit * p.max_parts * 2;
        const float *po = p.ws_o + unit * p.max_parts * D;
        float gmax = -INFINITY;
        for (int q = 0; q < nparts; ++q)
            gmax = fmaxf(gmax, __ldcg(ml + 2 * q));
        float num = 0.f, den = 0.f;
        for (int q = 0; q < nparts; ++q) {
            const float f = exp2f(__ldcg(ml + 2 * q) - gmax);
            num = fmaf(f, __ldcg(po + size_t(q) * D + tid), num);
            den = fmaf(f, __ldcg(ml + 2 * q + 1), den);
        }
        out_row[tid] = __float2half_rn(num / den);
    }
}

} // namespace pa
