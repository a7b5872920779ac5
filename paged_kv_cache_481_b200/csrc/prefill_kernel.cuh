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
// How: one CTA per (128 new tokens, head, sequence).  Warps 0-3 own one
// query row each per thread (TMEM lane = row); warp 4 drives the copies and
// the matrix multiplies.  For each 128-token tile of the context:
//   * TMA tensor loads bring K and V rows, (block, head) run by run, into
//     128-byte-swizzled shared-memory tiles (two 64-column halves each);
//   * tcgen05.mma computes S = Q K^T (both operands K-major) into TMEM;
//   * the row threads read S back (tcgen05.ld), apply the causal mask and the
//     online softmax in the log2 domain, and write P as fp16 into a swizzled
//     shared tile (rows of V past the context end are zeroed so 0 * garbage
//     cannot reach the output);
//   * tcgen05.mma computes P V (V as an N-major operand) into TMEM, and the
//     row threads fold it into their fp32 output row: o = o * alpha + P V.
// Every mbarrier wait is bounded; a wait that runs out records
// PA_DEVERR_TIMEOUT and the CTA stops after the current tile.
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
    float qk_scale_log2;              // softmax scale * log2(e)
    unsigned int *error_word;         // PA_DEVERR_* bits
};

__device__ __forceinline__ void prefill_error(const PrefillParams &p, unsigned int bits)
{
    atomicOr(p.error_word, bits);
}

constexpr int kPM = 128;              // query rows per CTA (MMA M)
constexpr int kPN = 128;              // context tokens per tile (MMA N of Q K^T)
constexpr int kPD = 128;              // head dim handled here
constexpr uint32_t kSub = 128 * 128;  // bytes of one [128 rows x 64 fp16] swizzled half tile
constexpr uint32_t kOffK = 2 * kSub, kOffV = 4 * kSub, kOffP = 6 * kSub;
constexpr uint32_t kPrefillSmem = 8 * kSub + 1024;  // + slack to align to 1024
constexpr int kPrefillThreads = 160;
constexpr uint32_t kTmemCols = 256;   // S at column 0, P V at column 128

__global__ void __launch_bounds__(kPrefillThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const PrefillParams p)
{
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bar_q, bar_kv, bar_s, bar_o;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool ctrl = tid == 4 * 32;
    const bool row_thread = tid < kPM;

    grid_dependency_wait();
    allow_dependent_launch();

    const int q_first = p.query_start_loc[b];
    const int n = p.query_start_loc[b + 1] - q_first;
    int L = p.context_lens[b];
    if (L < 0 || L > p.max_context_len) {
        if (tid == 0 && qt == 0 && h == 0)
            prefill_error(p, PA_DEVERR_CONTEXT_LEN);
        L = max(0, min(L, p.max_context_len));
    }
    if (n <= 0 || qt * kPM >= n)
        return;
    if (n > L) {  // more new tokens than the context holds: nothing sensible to do
        if (tid == 0 && qt == 0 && h == 0)
            prefill_error(p, PA_DEVERR_CONTEXT_LEN);
        return;
    }
    const int row0 = qt * kPM;              // first new token of this tile
    const int rows = min(kPM, n - row0);    // new tokens in this tile
    const int pos0 = L - n + row0;          // position of row 0
    const int ntiles = (pos0 + rows - 1) / kPN + 1;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sQ = (raw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sQ - raw);
    const uint32_t bq = smem_u32(&bar_q), bkv = smem_u32(&bar_kv), bs_ = smem_u32(&bar_s),
                   bo = smem_u32(&bar_o);
    if (tid == 0) {
        mbar_init(bq, 1);
        mbar_init(bkv, 1);
        mbar_init(bs_, 1);
        mbar_init(bo, 1);
        s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 4)
        tmem_alloc(smem_u32(&s_tmem), kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = s_tmem;
    const uint32_t tS = tmem, tO = tmem + kPN;

    const int H = p.num_heads, bsz = p.block_size;
    const int box_rows = bsz < kPN ? bsz : kPN;
    const int32_t *trow = p.block_tables + size_t(b) * p.max_blocks_per_seq;
    constexpr uint32_t kIdescS = idesc_f16_f32(kPM, kPN, false);
    constexpr uint32_t kIdescO = idesc_f16_f32(kPM, kPD, true);

    if (ctrl) {
        mbar_arrive_expect_tx(bq, 2 * kSub);
        tma_load_2d(sQ, &tm_q, h * kPD, q_first + row0, bq);
        tma_load_2d(sQ + kSub, &tm_q, h * kPD + 64, q_first + row0, bq);
    }

    float o[kPD];
#pragma unroll
    for (int d = 0; d < kPD; ++d)
        o[d] = 0.f;
    float m = -INFINITY, l = 0.f;
    const int my_pos = pos0 + tid;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;  // this warp's TMEM lanes

    for (int j = 0; j < ntiles; ++j) {
        const int t0 = j * kPN;
        const int valid = min(kPN, L - t0);   // context tokens in this tile
        const uint32_t par = uint32_t(j) & 1u;

        // ---- K, V of tile j, then S = Q K^T --------------------------------
        if (ctrl) {
            uint32_t bytes = 0;
            for (int i = 0; i * box_rows < valid; ++i) {
                const int tok = t0 + i * box_rows;
                if (unsigned(trow[tok / bsz]) < unsigned(p.num_blocks))
                    bytes += 4u * uint32_t(box_rows) * 128u;
            }
            mbar_arrive_expect_tx(bkv, bytes);
            for (int i = 0; i * box_rows < valid; ++i) {
                const int tok = t0 + i * box_rows;
                const int id = trow[tok / bsz];
                if (unsigned(id) >= unsigned(p.num_blocks)) {
                    prefill_error(p, PA_DEVERR_BLOCK_ID);
                    continue;
                }
                const int y = (id * H + h) * bsz + tok % bsz;
                const uint32_t off = uint32_t(i * box_rows) * 128u;
                tma_load_2d(sQ + kOffK + off, &tm_k, 0, y, bkv);
                tma_load_2d(sQ + kOffK + kSub + off, &tm_k, 64, y, bkv);
                tma_load_2d(sQ + kOffV + off, &tm_v, 0, y, bkv);
                tma_load_2d(sQ + kOffV + kSub + off, &tm_v, 64, y, bkv);
            }
            const bool ok = (j > 0 || mbar_wait_bounded(bq, 0u)) && mbar_wait_bounded(bkv, par);
            if (!ok) {
                prefill_error(p, PA_DEVERR_TIMEOUT);
                s_abort = 1;
            } else {
                tc_fence_after_sync();
#pragma unroll
                for (int k = 0; k < kPD / 16; ++k) {
                    const uint32_t kb = uint32_t(k >> 2) * kSub, kk = uint32_t(k & 3) * 32u;
                    umma_f16(tS, smem_desc_sw128(sQ + kb + kk, 16, 1024),
                             smem_desc_sw128(sQ + kOffK + kb + kk, 16, 1024), kIdescS, k > 0);
                }
                umma_commit(bs_);
            }
        }

        // ---- softmax of S, P to shared memory ------------------------------
        float alpha = 1.f;
        if (row_thread) {
            if (!mbar_wait_bounded(bs_, par)) {
                prefill_error(p, PA_DEVERR_TIMEOUT);
                s_abort = 1;
            } else {
                tc_fence_after_sync();
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < kPN / 32; ++c) {
                    float s[32];
                    tmem_load32(tS + lane_base + uint32_t(c * 32), s);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int t = t0 + c * 32 + i;
                        const float v = (t > my_pos || t >= L) ? -INFINITY : s[i] * p.qk_scale_log2;
                        mx = fmaxf(mx, v);
                    }
                }
                const float m_new = fmaxf(m, mx);
                alpha = exp2f(m - m_new);
                float lsum = 0.f;
#pragma unroll
                for (int c = 0; c < kPN / 32; ++c) {
                    float s[32];
                    tmem_load32(tS + lane_base + uint32_t(c * 32), s);
#pragma unroll
                    for (int g = 0; g < 4; ++g) {  // 8 tokens -> one 16-byte chunk of P
                        __half2 ph[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float pr[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int i = g * 8 + e * 2 + u;
                                const int t = t0 + c * 32 + i;
                                pr[u] = (t > my_pos || t >= L) ? 0.f
                                                               : exp2f(s[i] * p.qk_scale_log2 - m_new);
                            }
                            ph[e] = __floats2half2_rn(pr[0], pr[1]);
                            const float2 back = __half22float2(ph[e]);
                            lsum += back.x + back.y;
                        }
                        const int tok = c * 32 + g * 8;           // first token of the chunk
                        const uint32_t half = uint32_t(tok >> 6) * kSub;
                        const uint32_t chunk = uint32_t((tok & 63) >> 3);
                        *reinterpret_cast<uint4 *>(smem + kOffP + half + uint32_t(tid) * 128u +
                                                   ((chunk ^ (uint32_t(tid) & 7u)) << 4)) =
                            *reinterpret_cast<const uint4 *>(ph);
                    }
                }
                l = l * alpha + lsum;
                m = m_new;
            }
            // V rows past the context end (loaded with the last block, or stale)
            // are zeroed; S having completed, the tile's loads have landed.
            if (!s_abort && tid >= valid) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    *reinterpret_cast<uint4 *>(smem + kOffV + uint32_t(tid) * 128u + c * 16u) =
                        make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(smem + kOffV + kSub + uint32_t(tid) * 128u + c * 16u) =
                        make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async_smem();
        }
        tc_fence_before_sync();
        __syncthreads();
        if (s_abort)
            break;

        // ---- P V -------------------------------------------------------------
        if (ctrl) {
            tc_fence_after_sync();
#pragma unroll
            for (int k = 0; k < kPN / 16; ++k) {
                const uint32_t kb = uint32_t(k >> 2) * kSub, kk = uint32_t(k & 3) * 32u;
                umma_f16(tO, smem_desc_sw128(sQ + kOffP + kb + kk, 16, 1024),
                         smem_desc_sw128(sQ + kOffV + uint32_t(k) * 2048u, kSub, 1024), kIdescO,
                         k > 0);
            }
            umma_commit(bo);
        }
        if (row_thread || ctrl) {
            if (!mbar_wait_bounded(bo, par)) {
                prefill_error(p, PA_DEVERR_TIMEOUT);
                s_abort = 1;
            } else if (row_thread) {
                tc_fence_after_sync();
#pragma unroll
                for (int c = 0; c < kPD / 32; ++c) {
                    float ov[32];
                    tmem_load32(tO + lane_base + uint32_t(c * 32), ov);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        o[c * 32 + i] = fmaf(o[c * 32 + i], alpha, ov[i]);
                }
            }
        }
        tc_fence_before_sync();
        __syncthreads();
        if (s_abort)
            break;
    }

    // ---- epilogue ----------------------------------------------------------
    if (row_thread && !s_abort && tid < rows) {
        const float inv = 1.f / l;
        uint4 *dst = reinterpret_cast<uint4 *>(p.out + (size_t(q_first + row0 + tid) * H + h) * kPD);
#pragma unroll
        for (int c = 0; c < kPD / 8; ++c) {
            __half2 v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                v[e] = __floats2half2_rn(o[c * 8 + 2 * e] * inv, o[c * 8 + 2 * e + 1] * inv);
            dst[c] = *reinterpret_cast<const uint4 *>(v);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after_sync();
        tmem_free(tmem, kTmemCols);
    }
}

} // namespace pa
