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
//   * Storage: fp16 rows, or int8 codes with one affine (s, z) per (token,
//     head) row (brentwoodlivery.com 5.3.18: r_hat = s (q - z)).  For int8 a
//     tile is 32 rows, and the zero point enters once per row:
//       q.K = s (q . c - z sum_d q_d),
//       sum_t w_t V_t = sum_t w_t s_t (1024 + c_t) - sum_t w_t s_t (1024 + z_t).
//     q . c is exact integer arithmetic (dp4a) on the query in 16-bit fixed
//     point (q = s_q q16, s_q = max |q| / 32767, set once per segment), so
//     the only rounding the int8 path adds to the score is q's to 16 bits.
//     For the P.V sum the codes are widened exactly to fp16 as 1024 + c by a
//     byte permute and multiplied by w_t s_t rounded once to fp16 (the same
//     rounded value in both sums, so the bias cancels exactly), with the
//     products and sums in fp32 (mixed-precision FMA).
//   * Fused append (DecodeExtras, fp16): the worker that issues a unit's last
//     tile fetches one row fewer and its warp copies the new token's K / V
//     rows from the input into the stage and into the cache slot (the decode
//     step's cache write, polomodov.tech slide 11, in the same launch).
//   * Optional log-normaliser output (DecodeExtras::lse) so a caller can merge
//     this attention with attention over other parts of the context.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "quant.cuh"

namespace pa {

__device__ unsigned int g_device_error;

__device__ __forceinline__ void raise_device_error(unsigned int bits)
{
    atomicOr(&g_device_error, bits);
}

constexpr unsigned kErrBlockId = 1u << 0;
constexpr unsigned kErrContextLen = 1u << 1;
constexpr unsigned kErrSlot = 1u << 2;
constexpr unsigned kErrTimeout = 1u << 4;

constexpr int kTileBytes = 4096;  // one fp16 K (or V) tile in shared memory
constexpr int kMaxWorkers = 4096; // warps per grid; sizes the workspace

struct DecodeParams {
    __half *out;
    const __half *q;
    const void *k_cache;     // fp16 rows or int8 codes, [NB, H, bs, D]
    const void *v_cache;
    const float *k_params;   // int8 only: [NB, H, bs, 2] (s, z) per row
    const float *v_params;
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

// Optional extras, a separate kernel parameter: adding these fields to
// DecodeParams itself made ptxas allocate the kernel with 80 instead of 117
// registers and ~10 % more instructions.
struct DecodeExtras {
    // Fused append (fp16 cache only; new_slots == nullptr: plain decode).  For
    // a sequence b with new_slots[b] >= 0, position context_lens[b] - 1 is a
    // new token: its K / V rows come from new_k / new_v [B, H, D] (not from
    // the cache) and are also written to the cache at slot new_slots[b].
    const __half *new_k;
    const __half *new_v;
    const int64_t *new_slots;
    // optional [B, H]: log2 of each unit's softmax denominator relative to
    // 2^0, i.e. max + log2(sum) in base-2 units (to merge with other parts)
    float *lse;
    // optional, kLateDepWait instances only: the inputs are written by a
    // kernel that may still be running, which sets *ready non-zero once they
    // are all visible; every CTA waits for it (bounded) before it starts
    const unsigned int *ready;
};

constexpr int ilog2(int x)
{
    return x <= 1 ? 0 : 1 + ilog2(x / 2);
}

// Tile geometry for head_dim D and fp16 (kInt8 = false) or int8 storage.
template <int D, bool kInt8>
struct DecodeShape {
    static constexpr bool kQuant = kInt8;
    static constexpr int kElemBytes = kInt8 ? 1 : 2;
    static constexpr int kRowBytes = D * kElemBytes;
    static constexpr int kTokens = kInt8 ? 32 : kTileBytes / kRowBytes;  // rows per tile
    static constexpr int kTileK = kTokens * kRowBytes;                  // bytes of a K (or V) tile
    static constexpr int kChunks = kRowBytes / 16;                      // 16-byte chunks per row
    static constexpr int kDims = 16 / kElemBytes;                       // dims per chunk
    static constexpr int kRowsPerStep = 32 / kChunks;                   // rows one warp load covers
    static constexpr int kIters = kTokens / kRowsPerStep;               // warp loads per tile
    static constexpr int kLogChunks = ilog2(kChunks);
    static constexpr int kLogIters = ilog2(kIters);
    // after the transposing reduction, kDup adjacent lanes hold the same row
    static constexpr int kDup = 1 << (kLogChunks - kLogIters);
    static constexpr int kParamBytes = kInt8 ? kTokens * 8 : 0;         // (s, z) per row
    static constexpr int kMaxIds = 4;                                   // blocks one tile can span
    static constexpr int kQWords = kDims / 8;                           // uint4 of q per lane
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

template <int D, bool kInt8, int NW, int S>
struct DecodeSmem {
    using Sh = DecodeShape<D, kInt8>;
    // stage: K tile, V tile, K params, V params, q row
    static constexpr size_t kOffV = Sh::kTileK;
    static constexpr size_t kOffKP = 2 * Sh::kTileK;
    static constexpr size_t kOffVP = kOffKP + Sh::kParamBytes;
    static constexpr size_t kOffQ = kOffVP + Sh::kParamBytes;
    static constexpr size_t kStageBytes = kOffQ + D * 2;
    static constexpr size_t kTiles = size_t(NW) * S * kStageBytes;
    static constexpr size_t kBars = size_t(NW) * S * sizeof(uint64_t);
    static constexpr size_t kMeta = size_t(NW) * S * sizeof(TileMeta);
    static constexpr size_t kBytes = kTiles + kBars + kMeta;
    static constexpr int kThreads = NW * 32;
    static_assert(kStageBytes % 16 == 0, "bulk-copy destinations stay 16-byte aligned");
};

__device__ __forceinline__ float2 h2f(uint32_t bits)
{
    __half2 h = *reinterpret_cast<const __half2 *>(&bits);
    return __half22float2(h);
}

// Two int8 codes of a packed word, widened exactly to fp16 as 1024 + code:
// the byte permute builds the halves 0x64cc (exponent of 1024, code in the
// low mantissa bits).  The bias 1024 is removed once per row, through the
// zero point, instead of once per code.
constexpr float kCodeBias = 1024.f;

__device__ __forceinline__ uint32_t codes_to_h2(uint32_t word, uint32_t selector)
{
    return __byte_perm(word, 0x64646464u, selector);
}

// q . k over one 16-byte chunk of 8 fp16 values of K.
__device__ __forceinline__ float dot_chunk(const uint4 (&q)[1], const uint4 &k)
{
    float s0 = fma2_f16_f32(q[0].x, k.x, 0.f);
    float s1 = fma2_f16_f32(q[0].y, k.y, 0.f);
    s0 = fma2_f16_f32(q[0].z, k.z, s0);
    s1 = fma2_f16_f32(q[0].w, k.w, s1);
    return s0 + s1;
}

// q . codes over one 16-byte chunk of 16 int8 codes, exactly, in int32: the
// query in 16-bit fixed point split into a signed high byte and an unsigned
// low byte per dimension (qw[0] = the high bytes of the chunk's 16 dims,
// four per word; qw[1] = the low bytes), q16 . c = 256 (hi . c) + (lo . c).
__device__ __forceinline__ int dot_codes_q16(const uint4 (&qw)[2], const uint4 &k)
{
    int hi = 0, lo = 0;
    asm("dp4a.s32.u32 %0, %2, %3, %0;\n\t"
        "dp4a.s32.u32 %0, %4, %5, %0;\n\t"
        "dp4a.s32.u32 %0, %6, %7, %0;\n\t"
        "dp4a.s32.u32 %0, %8, %9, %0;\n\t"
        "dp4a.u32.u32 %1, %10, %3, %1;\n\t"
        "dp4a.u32.u32 %1, %11, %5, %1;\n\t"
        "dp4a.u32.u32 %1, %12, %7, %1;\n\t"
        "dp4a.u32.u32 %1, %13, %9, %1;"
        : "+r"(hi), "+r"(lo)
        : "r"(qw[0].x), "r"(k.x), "r"(qw[0].y), "r"(k.y), "r"(qw[0].z), "r"(k.z), "r"(qw[0].w), "r"(k.w),
          "r"(qw[1].x), "r"(qw[1].y), "r"(qw[1].z), "r"(qw[1].w));
    return hi * 256 + lo;
}

__device__ __forceinline__ void axpy_h2(float &a0, float &a1, float w, uint32_t h2)
{
    const float2 v = h2f(h2);
    a0 = fmaf(w, v.x, a0);
    a1 = fmaf(w, v.y, a1);
}

// acc += w * chunk (8 fp16 values).
__device__ __forceinline__ void axpy_chunk(float (&acc)[8], float w, const uint4 &u)
{
    axpy_h2(acc[0], acc[1], w, u.x);
    axpy_h2(acc[2], acc[3], w, u.y);
    axpy_h2(acc[4], acc[5], w, u.z);
    axpy_h2(acc[6], acc[7], w, u.w);
}

// acc[2j], acc[2j + 1] += w * (1024 + code) for the 16 codes of a chunk, with
// the weight w in fp16 (both halves of w2) and the products and sums in fp32
// (mixed-precision FMA: no conversion of the codes' fp16 form to fp32).
__device__ __forceinline__ void axpy_codes_f16w(float (&acc)[16], uint32_t w2, const uint4 &u)
{
    const uint32_t words[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t lo = codes_to_h2(words[j], 0x5140u), hi = codes_to_h2(words[j], 0x5342u);
        asm("{\n\t.reg .f16 w0, w1, a0, a1, b0, b1;\n\t"
            "mov.b32 {w0, w1}, %4;\n\t"
            "mov.b32 {a0, a1}, %5;\n\t"
            "mov.b32 {b0, b1}, %6;\n\t"
            "fma.rn.f32.f16 %0, w0, a0, %0;\n\t"
            "fma.rn.f32.f16 %1, w0, a1, %1;\n\t"
            "fma.rn.f32.f16 %2, w0, b0, %2;\n\t"
            "fma.rn.f32.f16 %3, w0, b1, %3;\n\t}"
            : "+f"(acc[4 * j]), "+f"(acc[4 * j + 1]), "+f"(acc[4 * j + 2]), "+f"(acc[4 * j + 3])
            : "r"(w2), "r"(lo), "r"(hi));
    }
}

// Consume one staged tile: scores, online-softmax update and PV accumulate.
// Lane (r, c) = (lane / kChunks, lane % kChunks) handles rows i*kRowsPerStep + r
// and dims [kDims c, kDims (c + 1)).  For int8, kp / vp are the tile's (s, z)
// rows, qh the query in 16-bit fixed point (dot_codes_q16), qsum = sum_d q16_d,
// qk_scale_log2 includes the query's fixed-point scale s_q, and corr
// accumulates sum_t w_t s_t (1024 + z_t).
template <int D, bool kInt8, bool kFull>
__device__ __forceinline__ void consume_tile(const uint4 *__restrict__ ks, const uint4 *__restrict__ vs,
                                             const float2 *__restrict__ kp, const float2 *__restrict__ vp,
                                             int valid_rows, int r, int c,
                                             const uint4 (&qh)[DecodeShape<D, kInt8>::kQWords],
                                             float qsum, float qk_scale_log2, float &m, float &l_part,
                                             float (&acc)[DecodeShape<D, kInt8>::kDims], float &corr)
{
    using S = DecodeShape<D, kInt8>;
    // int8: exact integer partial dot products (query in 16-bit fixed point)
    using Part = typename std::conditional<kInt8, int, float>::type;
    Part v[S::kIters];
#pragma unroll
    for (int i = 0; i < S::kIters; ++i) {
        if constexpr (kInt8)
            v[i] = dot_codes_q16(qh, ks[(i * S::kRowsPerStep + r) * S::kChunks + c]);
        else
            v[i] = dot_chunk(qh, ks[(i * S::kRowsPerStep + r) * S::kChunks + c]);
    }

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
                const Part send = upper ? v[j] : v[j + n / 2];
                const Part keep = upper ? v[j + n / 2] : v[j];
                v[j] = keep + __shfl_xor_sync(kFullMask, send, off);
            }
        } else {
            v[0] += __shfl_xor_sync(kFullMask, v[0], off);
        }
    }
    const int my_row = (c / S::kDup) * S::kRowsPerStep + r;
    float s;
    if constexpr (kInt8) {
        // q . k_t = s_t (q . c_t - z_t sum_d q_d), q = s_q q16; qsum is
        // sum_d q16_d and qk_scale_log2 carries s_q
        const float2 pz = kp[my_row];  // (s, z) of this lane's row
        s = pz.x * fmaf(-pz.y, qsum, float(v[0])) * qk_scale_log2;
    } else {
        s = v[0] * qk_scale_log2;
    }
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
    for (int k = 0; k < S::kDims; ++k)
        acc[k] *= alpha;
    if constexpr (kInt8)
        corr *= alpha;

#pragma unroll
    for (int i = 0; i < S::kIters; ++i) {
        const float wi = __shfl_sync(kFullMask, w, r * S::kChunks + i * S::kDup);
        const int row = i * S::kRowsPerStep + r;
        if (kFull || row < valid_rows) {
            if constexpr (kInt8) {
                // the row's weight times its scale, rounded once to fp16 and
                // used as such by both sums, so the code bias cancels exactly
                const float2 pz = vp[row];
                const __half2 ws2 = __float2half2_rn(wi * pz.x);
                const uint32_t w2 = *reinterpret_cast<const uint32_t *>(&ws2);
                corr = fmaf(__low2float(ws2), pz.y + kCodeBias, corr);
                axpy_codes_f16w(acc, w2, vs[row * S::kChunks + c]);
            } else {
                axpy_chunk(acc, wi, vs[row * S::kChunks + c]);
            }
        }
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
template <class Sh, bool kContig = false>
__device__ __forceinline__ void load_tile_ids(const DecodeParams &p, const TileCursor &cur,
                                              int (&ids)[Sh::kMaxIds])
{
    if constexpr (kContig) {  // no table: addresses follow from the position
#pragma unroll
        for (int s = 0; s < Sh::kMaxIds; ++s)
            ids[s] = 0;
        return;
    }
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

// Copy `rows` rows starting at row `row0` of the (block, head) run into the
// stage: K and V rows, and for int8 their (s, z) pairs (rounded up to an even
// number of rows so every copy is a multiple of 16 bytes; the extra row lies
// inside the same block and is never used).
template <int D, bool kInt8, class Sm>
__device__ __forceinline__ void copy_rows(const DecodeParams &p, size_t row0, int rows, uint32_t dst,
                                          uint32_t dst_row, uint32_t bar, uint64_t policy)
{
    using Sh = DecodeShape<D, kInt8>;
    const uint32_t bytes = uint32_t(rows) * Sh::kRowBytes;
    const char *k = static_cast<const char *>(p.k_cache) + row0 * Sh::kRowBytes;
    const char *v = static_cast<const char *>(p.v_cache) + row0 * Sh::kRowBytes;
    bulk_copy_g2s_hint(dst + dst_row * Sh::kRowBytes, k, bytes, bar, policy);
    bulk_copy_g2s_hint(dst + Sm::kOffV + dst_row * Sh::kRowBytes, v, bytes, bar, policy);
    if constexpr (kInt8) {
        const uint32_t pbytes = uint32_t((rows + 1) & ~1) * 8u;
        bulk_copy_g2s(dst + Sm::kOffKP + dst_row * 8u, p.k_params + row0 * 2, pbytes, bar);
        bulk_copy_g2s(dst + Sm::kOffVP + dst_row * 8u, p.v_params + row0 * 2, pbytes, bar);
    }
}

template <int D, bool kInt8>
__device__ __forceinline__ uint32_t rows_tx_bytes(int rows)
{
    using Sh = DecodeShape<D, kInt8>;
    uint32_t b = 2u * uint32_t(rows) * Sh::kRowBytes;
    if constexpr (kInt8)
        b += 2u * uint32_t((rows + 1) & ~1) * 8u;
    return b;
}

// Arm the stage's full barrier and issue the bulk copies of the tile under
// the cursor (K rows, V rows, their int8 parameters, and the q row when
// `with_q`).  K and V are read exactly once, so they go through L2 with an
// evict-first policy that keeps the small reused data (block tables, q, split
// partials) resident.
template <int D, bool kInt8, class Sm, bool kContig = false>
__device__ __forceinline__ void issue_tile(const DecodeParams &p, const DecodeExtras &x,
                                           const TileCursor &cur,
                                           const int (&ids)[DecodeShape<D, kInt8>::kMaxIds],
                                           bool with_q, unsigned char *stage_buf, uint32_t bar,
                                           TileMeta *meta, uint64_t stream_policy)
{
    using Sh = DecodeShape<D, kInt8>;
    const int bs = p.block_size;
    const int t0 = cur.i * Sh::kTokens;
    const int nv = min(Sh::kTokens, cur.len - t0);
    meta->b = cur.b;
    meta->h = cur.h;
    meta->i = cur.i;
    meta->len = cur.len;
    meta->k = cur.k;

    const uint32_t dst = smem_u32(stage_buf);
    // the last tile of a unit whose sequence appends a token: its last row
    // comes from the new-token input instead (append_new_row)
    int nf = nv;
    if (x.new_slots && cur.i == cur.nt - 1 && x.new_slots[cur.b] >= 0)
        nf = nv - 1;
    if constexpr (kContig) {
        // contiguous layout [B, H, Lmax, D] (Lmax = block_size): the tile is
        // one run of rows at ((b H + h) Lmax + t0)
        mbar_arrive_expect_tx(bar, (with_q ? uint32_t(D * 2) : 0u) + rows_tx_bytes<D, kInt8>(nf));
        if (with_q)
            bulk_copy_g2s(dst + Sm::kOffQ, p.q + (size_t(cur.b) * p.num_heads + cur.h) * D, D * 2, bar);
        if (nf > 0)
            copy_rows<D, kInt8, Sm>(p, (size_t(cur.b) * p.num_heads + cur.h) * size_t(bs) + size_t(t0), nf,
                                    dst, 0, bar, stream_policy);
        return;
    }
    // an id outside the pool is recorded and its rows are not fetched
    bool ok[Sh::kMaxIds];
#pragma unroll
    for (int s = 0; s < Sh::kMaxIds; ++s)
        ok[s] = unsigned(ids[s]) < unsigned(p.num_blocks);
    uint32_t total = with_q ? uint32_t(D * 2) : 0u;
    bool bad = false;
    if (bs >= Sh::kTokens) {
        if (!ok[0])
            bad = true;
        else if (nf > 0)
            total += rows_tx_bytes<D, kInt8>(nf);
    } else {
#pragma unroll
        for (int s = 0; s < Sh::kMaxIds; ++s) {
            if (s * bs >= nf)
                break;
            if (ok[s])
                total += rows_tx_bytes<D, kInt8>(min(bs, nf - s * bs));
            else
                bad = true;
        }
    }
    if (bad)
        raise_device_error(kErrBlockId);
    mbar_arrive_expect_tx(bar, total);
    if (with_q)
        bulk_copy_g2s(dst + Sm::kOffQ, p.q + (size_t(cur.b) * p.num_heads + cur.h) * D, D * 2, bar);
    if (bs >= Sh::kTokens) {
        if (ok[0] && nf > 0)
            copy_rows<D, kInt8, Sm>(p, (size_t(ids[0]) * p.num_heads + cur.h) * bs + size_t(t0 % bs),
                                    nf, dst, 0, bar, stream_policy);
    } else {
#pragma unroll
        for (int s = 0; s < Sh::kMaxIds; ++s) {
            if (s * bs >= nf)
                break;
            if (!ok[s])
                continue;
            copy_rows<D, kInt8, Sm>(p, (size_t(ids[s]) * p.num_heads + cur.h) * bs,
                                    min(bs, nf - s * bs), dst, uint32_t(s * bs), bar, stream_policy);
        }
    }
}

// The int8 tile under the cursor, issued by the whole warp: lane 4 s + k
// issues copy k (K codes, V codes, K (s, z), V (s, z)) of the tile's s-th
// block run, lane 16 the q row.  A 32-row int8 tile is two block runs at
// bs 16 (eight copies) and four at bs 8 (sixteen); one lane issuing them in
// turn spent several hundred cycles on each, and lanes issuing side by side
// took the int8 kernel from 80.6 to 82.6 % of the copy peak on the 13B batch
// and from 69.8 to 73.1 % on the serving batch (same box).  Arguments are
// the same in every lane.
template <int D, class Sm>
__device__ __forceinline__ void issue_tile_int8_warp(const DecodeParams &p, const DecodeExtras &x,
                                                     const TileCursor &cur,
                                                     const int (&ids)[DecodeShape<D, true>::kMaxIds],
                                                     bool with_q, unsigned char *stage_buf, uint32_t bar,
                                                     TileMeta *meta, uint64_t stream_policy, int lane)
{
    using Sh = DecodeShape<D, true>;
    const int bs = p.block_size;
    const int t0 = cur.i * Sh::kTokens;
    const int nv = min(Sh::kTokens, cur.len - t0);
    int nf = nv;  // the appended token's row comes from the input (append_new_row_int8)
    if (x.new_slots && cur.i == cur.nt - 1 && x.new_slots[cur.b] >= 0)
        nf = nv - 1;
    const bool one = bs >= Sh::kTokens;  // the tile lies inside one block
    const int nsub = one ? (nf > 0 ? 1 : 0) : (nf + bs - 1) / bs;
    uint32_t total = with_q ? uint32_t(D * 2) : 0u;
    bool bad = false;
#pragma unroll
    for (int s = 0; s < Sh::kMaxIds; ++s) {
        if (s < nsub) {
            if (unsigned(ids[s]) < unsigned(p.num_blocks))
                total += rows_tx_bytes<D, true>(one ? nf : min(bs, nf - s * bs));
            else
                bad = true;  // recorded; that run's rows are not fetched
        }
    }
    if (lane == 0) {
        meta->b = cur.b;
        meta->h = cur.h;
        meta->i = cur.i;
        meta->len = cur.len;
        meta->k = cur.k;
        if (bad)
            raise_device_error(kErrBlockId);
        mbar_arrive_expect_tx(bar, total);
    }
    __syncwarp();
    const uint32_t dst = smem_u32(stage_buf);
    const int s = lane >> 2, kind = lane & 3;
    const int id = s == 0 ? ids[0] : s == 1 ? ids[1] : s == 2 ? ids[2] : ids[3];
    if (lane < 4 * Sh::kMaxIds && s < nsub && unsigned(id) < unsigned(p.num_blocks)) {
        const int rows = one ? nf : min(bs, nf - s * bs);
        const size_t row0 = (size_t(id) * p.num_heads + cur.h) * bs + (one ? size_t(t0 % bs) : size_t(0));
        const uint32_t dst_row = one ? 0u : uint32_t(s * bs);
        fence_proxy_async_smem();
        if (kind == 0) {
            bulk_copy_g2s_hint(dst + dst_row * Sh::kRowBytes,
                               static_cast<const char *>(p.k_cache) + row0 * Sh::kRowBytes,
                               uint32_t(rows) * Sh::kRowBytes, bar, stream_policy);
        } else if (kind == 1) {
            bulk_copy_g2s_hint(dst + Sm::kOffV + dst_row * Sh::kRowBytes,
                               static_cast<const char *>(p.v_cache) + row0 * Sh::kRowBytes,
                               uint32_t(rows) * Sh::kRowBytes, bar, stream_policy);
        } else {
            const uint32_t pbytes = uint32_t((rows + 1) & ~1) * 8u;
            bulk_copy_g2s(dst + (kind == 2 ? Sm::kOffKP : Sm::kOffVP) + dst_row * 8u,
                          (kind == 2 ? p.k_params : p.v_params) + row0 * 2, pbytes, bar);
        }
    }
    if (with_q && lane == 16) {
        fence_proxy_async_smem();
        bulk_copy_g2s(dst + Sm::kOffQ, p.q + (size_t(cur.b) * p.num_heads + cur.h) * D, D * 2, bar);
    }
}

// Fused append, whole warp, right after the tile under the cursor was issued:
// if it is the last tile of its unit and the sequence appends a token, put
// the new K / V rows (position len - 1) into the stage from the new-token
// input and write them to the cache slot (polomodov.tech "vLLM and
// PagedAttention", slide 11: the new token goes into the next free slot).
// The slot must be the one the block table gives that position; otherwise
// PA_DEVERR_SLOT is recorded (and a slot outside the pool is not written).
template <int D, class Sm>
__device__ __forceinline__ void append_new_row(const DecodeParams &p, const DecodeExtras &x,
                                               const TileCursor &cur, unsigned char *stage_buf,
                                               int lane)
{
    using Sh = DecodeShape<D, false>;
    if (cur.i != cur.nt - 1)
        return;
    const int64_t slot = x.new_slots[cur.b];
    if (slot < 0)
        return;
    constexpr int kChunks = D * 2 / 16;  // 16-byte chunks of one row
    const int bs = p.block_size;
    const int pos = cur.len - 1;
    const int r = pos - cur.i * Sh::kTokens;  // the row's place in the stage
    const bool in_pool = slot < int64_t(p.num_blocks) * bs;
    if (lane == 0) {
        const int id = p.block_tables[size_t(cur.b) * p.max_blocks_per_seq + pos / bs];
        if (!in_pool || slot != int64_t(id) * bs + pos % bs)
            raise_device_error(kErrSlot);
    }
    if (lane < 2 * kChunks) {
        const bool is_v = lane >= kChunks;
        const int c = lane % kChunks;
        const size_t src_row = size_t(cur.b) * p.num_heads + cur.h;
        const uint4 val = __ldg(reinterpret_cast<const uint4 *>((is_v ? x.new_v : x.new_k) + src_row * D) + c);
        *reinterpret_cast<uint4 *>(stage_buf + (is_v ? Sm::kOffV : 0u) + uint32_t(r) * Sh::kRowBytes +
                                   uint32_t(c) * 16u) = val;
        if (in_pool) {
            const size_t row = (size_t(slot / bs) * p.num_heads + cur.h) * bs + size_t(slot % bs);
            uint4 *cache = reinterpret_cast<uint4 *>(const_cast<void *>(is_v ? p.v_cache : p.k_cache));
            cache[row * kChunks + c] = val;
        }
    }
    fence_proxy_async_smem();  // before a later bulk copy overwrites the stage
    __syncwarp();
}

// The same for the int8 cache, whole warp, once the tile's copies have
// landed (the (s, z) copy of the other rows is rounded up to an even row
// count, so it may cover this row's place in the stage): the new K and V
// rows are quantized exactly as the int8 cache write does
// (quantize_row_warp), their codes and (s, z) put into the stage and written
// to the cache slot.
template <int D, class Sm>
__device__ __forceinline__ void append_new_row_int8(const DecodeParams &p, const DecodeExtras &x,
                                                    const TileMeta &mt, unsigned char *stage_buf,
                                                    int lane)
{
    using Sh = DecodeShape<D, true>;
    constexpr int E = D / 32;  // values per lane
    const int64_t slot = x.new_slots[mt.b];
    if (slot < 0)
        return;
    const int bs = p.block_size;
    const int pos = mt.len - 1;
    const int r = pos - mt.i * Sh::kTokens;  // the row's place in the stage
    const bool in_pool = slot < int64_t(p.num_blocks) * bs;
    if (lane == 0) {
        const int id = p.block_tables[size_t(mt.b) * p.max_blocks_per_seq + pos / bs];
        if (!in_pool || slot != int64_t(id) * bs + pos % bs)
            raise_device_error(kErrSlot);
    }
    const size_t src_row = size_t(mt.b) * p.num_heads + mt.h;
    const size_t row = in_pool ? (size_t(slot / bs) * p.num_heads + mt.h) * bs + size_t(slot % bs) : 0;
#pragma unroll
    for (int kv = 0; kv < 2; ++kv) {
        const __half *src = (kv ? x.new_v : x.new_k) + src_row * D + lane * E;
        float v[E];
#pragma unroll
        for (int e = 0; e < E; ++e)
            v[e] = __half2float(src[e]);
        float sc, z;
        const uint32_t packed = quantize_row_warp<E>(v, sc, z);
        unsigned char *codes = stage_buf + (kv ? Sm::kOffV : 0u) + uint32_t(r) * Sh::kRowBytes +
                               uint32_t(lane * E);
        uint8_t *cache = static_cast<uint8_t *>(const_cast<void *>(kv ? p.v_cache : p.k_cache)) +
                         row * D + lane * E;
        if constexpr (E == 4) {
            *reinterpret_cast<uint32_t *>(codes) = packed;
            if (in_pool)
                *reinterpret_cast<uint32_t *>(cache) = packed;
        } else {
            *reinterpret_cast<uint16_t *>(codes) = uint16_t(packed);
            if (in_pool)
                *reinterpret_cast<uint16_t *>(cache) = uint16_t(packed);
        }
        if (lane == 0) {
            *reinterpret_cast<float2 *>(stage_buf + (kv ? Sm::kOffVP : Sm::kOffKP) + uint32_t(r) * 8u) =
                make_float2(sc, z);
            if (in_pool)
                reinterpret_cast<float2 *>(const_cast<float *>(kv ? p.v_params : p.k_params))[row] =
                    make_float2(sc, z);
        }
    }
    fence_proxy_async_smem();  // before a later bulk copy overwrites the stage
    __syncwarp();
}

// Merge the partial results of a (sequence, head) whose tiles were split
// between workers w_first..w_last, in worker order, and write out.  One pass:
// each contribution rescales the running sums to the running maximum, so all
// loads are independent.  Lanes with r == 0 each handle kDims dims.
template <int D, int kDims>
__device__ __forceinline__ void merge_partials(const DecodeParams &p, const DecodeExtras &x,
                                               uint4 *out_row, int c,
                                               long long u_start, long long w_first,
                                               long long w_last, long long total,
                                               long long workers)
{
    float gmax = -INFINITY, den = 0.f;
    float num[kDims];
#pragma unroll
    for (int k = 0; k < kDims; ++k)
        num[k] = 0.f;
    for (long long w = w_first; w <= w_last; ++w) {
        const size_t q = size_t(w) * 2 + (u_start <= range_start(w, total, workers) ? 0 : 1);
        const float mw = __ldcg(p.ws_ml + q * 2), lw = __ldcg(p.ws_ml + q * 2 + 1);
        const float4 *po = reinterpret_cast<const float4 *>(p.ws_o + q * D + kDims * c);
        const float m_new = fmaxf(gmax, mw);
        const float a = exp2f(gmax - m_new), f = exp2f(mw - m_new);
        gmax = m_new;
        den = fmaf(den, a, f * lw);
#pragma unroll
        for (int k = 0; k < kDims / 4; ++k) {
            const float4 x = __ldcg(po + k);
            num[4 * k + 0] = fmaf(num[4 * k + 0], a, f * x.x);
            num[4 * k + 1] = fmaf(num[4 * k + 1], a, f * x.y);
            num[4 * k + 2] = fmaf(num[4 * k + 2], a, f * x.z);
            num[4 * k + 3] = fmaf(num[4 * k + 3], a, f * x.w);
        }
    }
    __half2 o[kDims / 2];
#pragma unroll
    for (int k = 0; k < kDims / 2; ++k)
        o[k] = __floats2half2_rn(num[2 * k] / den, num[2 * k + 1] / den);
#pragma unroll
    for (int k = 0; k < kDims / 8; ++k)
        out_row[(kDims / 8) * c + k] = reinterpret_cast<const uint4 *>(o)[k];
    if (x.lse && c == 0)
        x.lse[(reinterpret_cast<const __half *>(out_row) - p.out) / D] = gmax + log2f(den);
}

template <int D, bool kInt8, int NW, int S, bool kContig>
__device__ __forceinline__ void paged_decode_body(const DecodeParams &p, const DecodeExtras &x)
{
    using Sh = DecodeShape<D, kInt8>;
    using Sm = DecodeSmem<D, kInt8, NW, S>;
    constexpr int T = Sh::kTokens;
    constexpr int kThreads = Sm::kThreads;
    constexpr int kWarps = NW;
    constexpr int kDims = Sh::kDims;

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

    // Bring the small inputs every worker looks up (context lengths, block
    // tables, q) into L2 while the scan below runs; the CTAs split the lines.
    {
        const size_t g = size_t(blockIdx.x) * kThreads + tid, stride = size_t(gridDim.x) * kThreads;
        const size_t table_lines = kContig ? 0 : (size_t(B) * p.max_blocks_per_seq * 4 + 127) / 128;
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
    // int8 tiles: the whole warp issues the copies (issue_tile_int8_warp)
    constexpr bool warp_issue = kInt8;
    int ids[Sh::kMaxIds];
    {
        TileCursor mc = prod;
        for (int s = 0; s < first - 1; ++s)
            if (s < lane)
                mc.template advance<T>(p);
        if (lane < first)
            load_tile_ids<Sh, kContig>(p, mc, ids);
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
            if constexpr (warp_issue && !kContig)
                issue_tile_int8_warp<D, Sm>(p, x, cs, ids_s, cs.i == 0 || cs.k == lo,
                                            my_buf + size_t(s) * Sm::kStageBytes, my_bar + 8 * s,
                                            my_meta + s, policy, lane);
            else if (lane == 0)
                issue_tile<D, kInt8, Sm, kContig>(p, x, cs, ids_s, cs.i == 0 || cs.k == lo,
                                         my_buf + size_t(s) * Sm::kStageBytes, my_bar + 8 * s,
                                         my_meta + s, policy);
            if constexpr (!kInt8)
                if (x.new_slots)
                    append_new_row<D, Sm>(p, x, cs, my_buf + size_t(s) * Sm::kStageBytes, lane);
            if (s == first - 1)
                prod = cs;
        }
    }
    int issued = first;
    if (issued < ntiles) {
        prod.template advance<T>(p);
        load_tile_ids<Sh, kContig>(p, prod, ids);
    }

    // ---- 5. stream --------------------------------------------------------
    uint4 qh[Sh::kQWords];
#pragma unroll
    for (int k = 0; k < Sh::kQWords; ++k)
        qh[k] = make_uint4(0, 0, 0, 0);
    float qsum = 0.f, qscale = p.qk_scale_log2;
    float m = -INFINITY, l_part = 0.f, corr = 0.f;
    float acc[kDims];
#pragma unroll
    for (int k = 0; k < kDims; ++k)
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
        if constexpr (kInt8)
            if (x.new_slots && mt.i == nt - 1)
                append_new_row_int8<D, Sm>(p, x, mt, my_buf + size_t(stage) * Sm::kStageBytes, lane);
        const unsigned char *buf = my_buf + size_t(stage) * Sm::kStageBytes;
        if (mt.i == 0 || mt.k == lo) {  // first tile of a segment: fresh state, new q
            const uint4 *qs = reinterpret_cast<const uint4 *>(buf + Sm::kOffQ);
#pragma unroll
            for (int k = 0; k < Sh::kQWords; ++k)
                qh[k] = qs[Sh::kQWords * c + k];
            if constexpr (kInt8) {
                // the query row in 16-bit fixed point: q_d = s_q q16_d with
                // s_q = max_d |q_d| / 32767, q16 split into a signed high
                // byte and an unsigned low byte (dot_codes_q16)
                float qf[16];
                float amax = 0.f;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const uint32_t w4[4] = {qh[k].x, qh[k].y, qh[k].z, qh[k].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = h2f(w4[e]);
                        qf[8 * k + 2 * e] = f.x;
                        qf[8 * k + 2 * e + 1] = f.y;
                        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
                    }
                }
#pragma unroll
                for (int off = Sh::kChunks >> 1; off >= 1; off >>= 1)
                    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, off));
                const float inv = amax > 0.f ? 32767.f / amax : 0.f;
                int isum = 0;
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t hb = 0, lb = 0;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int q16 = __float2int_rn(qf[4 * w + e] * inv);
                        isum += q16;
                        hb |= uint32_t((q16 >> 8) & 0xff) << (8 * e);
                        lb |= uint32_t(q16 & 0xff) << (8 * e);
                    }
                    hw[w] = hb;
                    lw[w] = lb;
                }
                qh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                qh[1] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
#pragma unroll
                for (int off = Sh::kChunks >> 1; off >= 1; off >>= 1)
                    isum += __shfl_xor_sync(kFullMask, isum, off);
                qsum = float(isum);
                qscale = (amax / 32767.f) * p.qk_scale_log2;
            }
#pragma unroll
            for (int k = 0; k < kDims; ++k)
                acc[k] = 0.f;
            m = -INFINITY;
            l_part = 0.f;
            corr = 0.f;
            seg_i0 = mt.i;
        }
        const uint4 *ks = reinterpret_cast<const uint4 *>(buf);
        const uint4 *vs = reinterpret_cast<const uint4 *>(buf + Sm::kOffV);
        const float2 *kp = reinterpret_cast<const float2 *>(buf + Sm::kOffKP);
        const float2 *vp = reinterpret_cast<const float2 *>(buf + Sm::kOffVP);
        if (nv == T)
            consume_tile<D, kInt8, true>(ks, vs, kp, vp, nv, r, c, qh, qsum, qscale, m, l_part,
                                         acc, corr);
        else
            consume_tile<D, kInt8, false>(ks, vs, kp, vp, nv, r, c, qh, qsum, qscale, m, l_part,
                                          acc, corr);
        __syncwarp();
        if (issued < ntiles) {  // refill the stage just consumed
            if constexpr (warp_issue && !kContig) {
                issue_tile_int8_warp<D, Sm>(p, x, prod, ids, prod.i == 0 || prod.k == lo,
                                            my_buf + size_t(stage) * Sm::kStageBytes, my_bar + 8 * stage,
                                            my_meta + stage, policy, lane);
            } else if (lane == 0) {
                fence_proxy_async_smem();
                issue_tile<D, kInt8, Sm, kContig>(p, x, prod, ids, prod.i == 0 || prod.k == lo,
                                         my_buf + size_t(stage) * Sm::kStageBytes,
                                         my_bar + 8 * stage, my_meta + stage, policy);
            }
            if constexpr (!kInt8)
                if (x.new_slots)
                    append_new_row<D, Sm>(p, x, prod, my_buf + size_t(stage) * Sm::kStageBytes, lane);
            if (++issued < ntiles) {
                prod.template advance<T>(p);
                load_tile_ids<Sh, kContig>(p, prod, ids);
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
        for (int off = Sh::kChunks; off < 32; off <<= 1) {
#pragma unroll
            for (int k = 0; k < kDims; ++k)
                acc[k] += __shfl_xor_sync(kFullMask, acc[k], off);
            if constexpr (kInt8)
                corr += __shfl_xor_sync(kFullMask, corr, off);
        }
        if constexpr (kInt8) {
#pragma unroll
            for (int k = 0; k < kDims; ++k)
                acc[k] -= corr;
        }
        const size_t unit = size_t(mt.b) * H + mt.h;
        uint4 *out_row = reinterpret_cast<uint4 *>(p.out + unit * D);
        if (seg_i0 == 0 && mt.i == nt - 1) {
            if (r == 0) {
                __half2 o[kDims / 2];
#pragma unroll
                for (int k = 0; k < kDims / 2; ++k)
                    o[k] = __floats2half2_rn(acc[2 * k] / l, acc[2 * k + 1] / l);
#pragma unroll
                for (int k = 0; k < kDims / 8; ++k)
                    out_row[(kDims / 8) * c + k] = reinterpret_cast<const uint4 *>(o)[k];
            }
            if (x.lse && lane == 0)
                x.lse[unit] = m + log2f(l);
            continue;
        }
        const long long u_start = mt.k - mt.i;      // global index of the unit's tile 0
        const int slot = u_start <= lo ? 0 : 1;     // first or last segment of this worker
        const size_t pidx = size_t(gw) * 2 + slot;
        if (r == 0) {
            float4 *po = reinterpret_cast<float4 *>(p.ws_o + pidx * D + kDims * c);
#pragma unroll
            for (int k = 0; k < kDims / 4; ++k)
                po[k] = make_float4(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3]);
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
            merge_partials<D, kDims>(p, x, out_row, c, u_start, w_first, w_last, total, workers);
    }
}

// kLateDepWait = false: inputs may come from the previous kernel in the
// stream, so none is read before it has finished; the next kernel may start
// launching meanwhile.  kLateDepWait = true: the caller guarantees the
// inputs are ready -- they were written two launches back and the previous
// kernel only starts this one after it has itself waited for them, or
// x.ready is set and the kernel that writes them raises that flag -- so the
// work starts at once, running beside the previous kernel, and the wait for
// that kernel comes at the end: this grid then completes only after
// everything before it, and the next kernel that waits for this grid sees
// all of it.
// kContig: the cache is contiguous per (sequence, head), [B, H, Lmax, D]
// with Lmax in block_size, and no block table is read (the baseline that
// measures what the paged layout's indirection costs).
template <int D, bool kInt8, int NW, int S, bool kLateDepWait = false, bool kContig = false>
__global__ void __launch_bounds__(NW * 32) paged_decode_kernel(const DecodeParams p, const DecodeExtras x)
{
    if (!kLateDepWait)
        grid_dependency_wait();
    allow_dependent_launch();
    if constexpr (kLateDepWait) {
        if (x.ready) {
            if (threadIdx.x == 0) {
                const volatile unsigned int *flag = x.ready;
                bool ok = *flag != 0u;
                if (!ok) {
                    const uint64_t t0 = global_timer_ns();
                    while (!(ok = *flag != 0u) && global_timer_ns() - t0 < kWaitLimitNs)
                        __nanosleep(64);
                }
                if (!ok)
                    raise_device_error(kErrTimeout);
                __threadfence();
            }
            __syncthreads();
        }
    }
    paged_decode_body<D, kInt8, NW, S, kContig>(p, x);
    if (kLateDepWait && threadIdx.x == 0)
        grid_dependency_wait();
}

} // namespace pa
