// Host-side helpers shared by the library's translation units: argument
// checks, the launch with programmatic stream serialisation, and the device
// error word's address.
#pragma once

#include <cuda_runtime.h>

#include "../../include/pa.h"

#include <cstddef>
#include <cstdint>

namespace pa_host {

// Device address of the library's device error word (the PA_DEVERR_* bits)
// on the current device; nullptr if it cannot be looked up.
unsigned int *device_error_word();

// pa_decode that also writes each (sequence, head)'s softmax log-normaliser
// lse = max + log2(sum) in base-2 units ([num_seqs, num_heads] fp32), so the
// result can be merged with attention over other parts of the context.
// max_ctas > 0 caps the persistent grid (to share the GPU with the kernel
// launched before it); late_dep_wait: see paged_decode_kernel's kLateDepWait.
pa_status decode_with_lse(void *out, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *context_lens, int max_context_len, int num_seqs,
                          int num_heads, int head_dim, int block_size, int num_blocks, float scale,
                          void *workspace, size_t workspace_bytes, float *lse, pa_stream_t stream,
                          int max_ctas = 0, bool late_dep_wait = false,
                          const unsigned int *ready = nullptr);

// CTAs of the fp16, head-dim-128 decode kernel that fit on one SM (0 on error).
int decode_ctas_per_sm();

// Byte offset of the merge tickets (one unsigned per (sequence, head), zero
// between calls) inside pa_decode's workspace for these sizes.
size_t decode_ticket_offset(int num_seqs, int num_heads, int head_dim);

} // namespace pa_host

namespace {

using pa_host::device_error_word;

constexpr int kMaxDevices = 64;

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool supported_head_dim(int d)
{
    return d == 64 || d == 128;
}

bool supported_block_size(int bs)
{
    return bs == 8 || bs == 16 || bs == 32 || bs == 64 || bs == 128;
}

size_t align256(size_t x)
{
    return (x + 255) & ~size_t(255);
}

// Launch with programmatic stream serialisation: the grid may begin while the
// previous kernel in the stream drains; every kernel here waits on
// griddepcontrol.wait before it touches memory, so ordering is unchanged.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

} // namespace
