"""Thin ctypes binding over libpa.so with the C ABI's names.

Argument marshalling only: shapes are read off the tensors, raw device
pointers and sizes are passed to the C functions declared in include/pa.h,
and a non-OK status raises ``PAError``.  Every step of the path runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and loading
fails loudly when libpa.so is missing.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpa.so")

(PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_WORKSPACE,
 PA_ERR_OUT_OF_BLOCKS) = range(6)
PA_DEVERR_BLOCK_ID = 1
PA_DEVERR_CONTEXT_LEN = 2
PA_DEVERR_SLOT = 4
PA_DEVERR_COPY_PAIR = 8
PA_DEVERR_TIMEOUT = 16

# every symbol include/pa.h declares
EXPORTED = ("pa_reshape_and_cache", "pa_decode_workspace_size", "pa_decode_workspace_init",
            "pa_decode", "pa_copy_blocks", "pa_status_string",
            "pa_get_last_device_error", "pa_decode_no_alloc", "pa_selftest_bounded_wait",
            "pa_bm_create", "pa_bm_destroy", "pa_bm_num_free", "pa_bm_refcount",
            "pa_bm_add_sequence", "pa_bm_fork", "pa_bm_free_sequence", "pa_bm_append_slots",
            "pa_bm_block_tables", "pa_reshape_and_cache_int8", "pa_decode_int8",
            "pa_decode_append_int8",
            "pa_copy_blocks_raw", "pa_prefill", "pa_swap_blocks", "pa_bm_create_with_swap",
            "pa_bm_num_free_cpu", "pa_bm_cpu_refcount", "pa_bm_is_swapped", "pa_bm_swap_out",
            "pa_bm_swap_in", "pa_decode_append", "pa_decode_grouped_workspace_size",
            "pa_decode_grouped", "pa_decode_contiguous")

_lock = threading.Lock()
_lib = None


class PAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def load(path: str | None = None):
    """Load libpa.so (once).  Raises if the library is absent."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"libpa.so not built at {p}: run "
                               "`python -m paged_kv_cache_481_b200.build`")
        lib = ctypes.CDLL(p)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.pa_reshape_and_cache.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]
        lib.pa_reshape_and_cache.restype = i32
        lib.pa_decode_workspace_size.argtypes = [i32, i32, i32, i32]
        lib.pa_decode_workspace_size.restype = sz
        lib.pa_decode_workspace_init.argtypes = [vp, sz, vp]
        lib.pa_decode_workspace_init.restype = i32
        lib.pa_decode.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32,
                                  ctypes.c_float, vp, sz, vp]
        lib.pa_decode.restype = i32
        lib.pa_decode_no_alloc.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32,
                                           i32, ctypes.c_float, vp]
        lib.pa_decode_no_alloc.restype = i32
        lib.pa_selftest_bounded_wait.argtypes = [ctypes.c_uint, vp]
        lib.pa_selftest_bounded_wait.restype = i32
        i64, p64, p32 = ctypes.c_int64, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32)
        lib.pa_bm_create.argtypes = [i32, i32]
        lib.pa_bm_create.restype = vp
        lib.pa_bm_destroy.argtypes = [vp]
        lib.pa_bm_destroy.restype = None
        lib.pa_bm_num_free.argtypes = [vp]
        lib.pa_bm_num_free.restype = i32
        lib.pa_bm_refcount.argtypes = [vp, i32]
        lib.pa_bm_refcount.restype = i32
        lib.pa_bm_add_sequence.argtypes = [vp, i64, i32]
        lib.pa_bm_add_sequence.restype = i32
        lib.pa_bm_fork.argtypes = [vp, i64, i64]
        lib.pa_bm_fork.restype = i32
        lib.pa_bm_free_sequence.argtypes = [vp, i64]
        lib.pa_bm_free_sequence.restype = i32
        lib.pa_bm_append_slots.argtypes = [vp, vp, i32, vp, vp, ctypes.POINTER(ctypes.c_int)]
        lib.pa_bm_append_slots.restype = i32
        lib.pa_bm_block_tables.argtypes = [vp, vp, i32, vp, i32, vp]
        lib.pa_bm_block_tables.restype = i32
        lib.pa_reshape_and_cache_int8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                                  i32, vp]
        lib.pa_reshape_and_cache_int8.restype = i32
        lib.pa_decode_int8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32,
                                       i32, i32, ctypes.c_float, vp, sz, vp]
        lib.pa_decode_int8.restype = i32
        lib.pa_copy_blocks_raw.argtypes = [vp, sz, vp, i32, i32, vp]
        lib.pa_copy_blocks_raw.restype = i32
        lib.pa_decode_grouped_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
        lib.pa_decode_contiguous.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                             ctypes.c_float, vp, sz, vp]
        lib.pa_decode_contiguous.restype = i32
        lib.pa_decode_grouped_workspace_size.restype = sz
        lib.pa_decode_grouped.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, vp, vp, i32, i32, i32,
                                          i32, i32, i32, i32, ctypes.c_float, vp, sz, vp]
        lib.pa_decode_grouped.restype = i32
        lib.pa_decode_append.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32,
                                         i32, i32, ctypes.c_float, vp, sz, vp]
        lib.pa_decode_append.restype = i32
        lib.pa_decode_append_int8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, i32,
                                              i32, i32, i32, i32, i32, ctypes.c_float, vp, sz, vp]
        lib.pa_decode_append_int8.restype = i32
        lib.pa_swap_blocks.argtypes = [vp, vp, sz, vp, i32, i32, i32, vp]
        lib.pa_swap_blocks.restype = i32
        lib.pa_bm_create_with_swap.argtypes = [i32, i32, i32]
        lib.pa_bm_create_with_swap.restype = vp
        lib.pa_bm_num_free_cpu.argtypes = [vp]
        lib.pa_bm_num_free_cpu.restype = i32
        lib.pa_bm_cpu_refcount.argtypes = [vp, i32]
        lib.pa_bm_cpu_refcount.restype = i32
        lib.pa_bm_is_swapped.argtypes = [vp, i64]
        lib.pa_bm_is_swapped.restype = i32
        for f in (lib.pa_bm_swap_out, lib.pa_bm_swap_in):
            f.argtypes = [vp, vp, i32, vp, i32, ctypes.POINTER(ctypes.c_int)]
            f.restype = i32
        lib.pa_prefill.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, vp, i32, i32, i32, i32, i32,
                                   i32, i32, ctypes.c_float, vp]
        lib.pa_prefill.restype = i32
        lib.pa_copy_blocks.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp]
        lib.pa_copy_blocks.restype = i32
        lib.pa_status_string.argtypes = [i32]
        lib.pa_status_string.restype = ctypes.c_char_p
        lib.pa_get_last_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        lib.pa_get_last_device_error.restype = i32
        if path is None:
            _lib = lib
        return lib


def status_string(status: int) -> str:
    return load().pa_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != PA_OK:
        raise PAError(status, what)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if isinstance(stream, torch.cuda.Stream)
                           else int(stream))


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(None)
    if not t.is_cuda:
        raise ValueError("libpa takes device tensors")
    _on_current_device(t)
    if not t.is_contiguous():
        raise ValueError("libpa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _on_current_device(t: torch.Tensor):
    """The library launches on the current device and keeps per-device state
    (error word, static scratch, scheduling counters) for it, so a tensor that
    lives on another GPU would hand its kernels a foreign pointer."""
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"tensor on cuda:{t.device.index} but the current device is "
                         f"cuda:{cur}; call under torch.cuda.device({t.device.index})")


def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None):
    """Write each token's K/V row at its slot (negative slots skipped)."""
    n, h, d = key.shape
    nb, hk, bs, dk = k_cache.shape
    assert key.dtype == value.dtype == k_cache.dtype == v_cache.dtype == torch.float16
    assert slot_mapping.dtype == torch.int64 and slot_mapping.numel() == n
    assert (hk, dk) == (h, d) and value.shape == key.shape and v_cache.shape == k_cache.shape
    _check(load().pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(slot_mapping), n, h, d, bs, nb, _stream(stream)),
           "pa_reshape_and_cache")


def pa_decode_workspace_size(num_seqs, num_heads, head_dim, max_context_len) -> int:
    return int(load().pa_decode_workspace_size(num_seqs, num_heads, head_dim, max_context_len))


def pa_decode_workspace_init(workspace: torch.Tensor, stream=None):
    _check(load().pa_decode_workspace_init(_ptr(workspace), workspace.numel()
                                           * workspace.element_size(), _stream(stream)),
           "pa_decode_workspace_init")


def new_workspace(num_seqs, num_heads, head_dim, max_context_len, device=None) -> torch.Tensor:
    """Allocate (through torch) and initialise a decode workspace."""
    n = pa_decode_workspace_size(num_seqs, num_heads, head_dim, max_context_len)
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    pa_decode_workspace_init(ws)
    return ws


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len,
              scale, workspace, stream=None):
    """Paged decode attention: out[b, h] = softmax(scale q.K) V over the
    sequence's blocks.  max_context_len is a host-side bound on context_lens."""
    b, h, d = q.shape
    nb, hk, bs, dk = k_cache.shape
    assert q.dtype == out.dtype == k_cache.dtype == v_cache.dtype == torch.float16
    assert out.shape == q.shape and (hk, dk) == (h, d) and v_cache.shape == k_cache.shape
    assert block_tables.dtype == torch.int32 and block_tables.dim() == 2
    assert context_lens.dtype == torch.int32 and context_lens.numel() == b
    _check(load().pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                            _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                            int(max_context_len), b, h, d, bs, nb, float(scale),
                            _ptr(workspace), workspace.numel() * workspace.element_size(),
                            _stream(stream)),
           "pa_decode")


def pa_decode_append(out, q, key, value, k_cache, v_cache, slot_mapping, block_tables,
                     context_lens, max_context_len, scale, workspace, stream=None):
    """The decode step's cache write and the paged decode in one launch: for
    each sequence b with slot_mapping[b] >= 0, key[b] / value[b] are its new
    token (position context_lens[b] - 1), written to that slot and used by
    the attention."""
    b, h, d = q.shape
    nb, hk, bs, dk = k_cache.shape
    assert q.dtype == out.dtype == key.dtype == value.dtype == k_cache.dtype == torch.float16
    assert out.shape == q.shape == key.shape == value.shape and (hk, dk) == (h, d)
    assert v_cache.shape == k_cache.shape
    assert slot_mapping.dtype == torch.int64 and slot_mapping.numel() == b
    assert block_tables.dtype == torch.int32 and block_tables.dim() == 2
    assert context_lens.dtype == torch.int32 and context_lens.numel() == b
    _check(load().pa_decode_append(_ptr(out), _ptr(q), _ptr(key), _ptr(value), _ptr(k_cache),
                                   _ptr(v_cache), _ptr(slot_mapping), _ptr(block_tables),
                                   block_tables.shape[1], _ptr(context_lens), int(max_context_len),
                                   b, h, d, bs, nb, float(scale), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "pa_decode_append")


def pa_decode_append_int8(out, q, key, value, k_codes, v_codes, k_params, v_params, slot_mapping,
                          block_tables, context_lens, max_context_len, scale, workspace,
                          stream=None):
    """pa_decode_append over the int8 cache: each new K/V row is quantized
    into its slot and the decode sees it, in one launch."""
    b, h, d = q.shape
    nb, hk, bs, dk = k_codes.shape
    assert q.dtype == out.dtype == key.dtype == value.dtype == torch.float16
    assert k_codes.dtype == v_codes.dtype == torch.uint8 and v_codes.shape == k_codes.shape
    assert out.shape == q.shape == key.shape == value.shape and (hk, dk) == (h, d)
    assert k_params.shape == v_params.shape == (nb, h, bs, 2)
    assert k_params.dtype == v_params.dtype == torch.float32
    assert slot_mapping.dtype == torch.int64 and slot_mapping.numel() == b
    assert block_tables.dtype == torch.int32 and block_tables.dim() == 2
    assert context_lens.dtype == torch.int32 and context_lens.numel() == b
    _check(load().pa_decode_append_int8(_ptr(out), _ptr(q), _ptr(key), _ptr(value), _ptr(k_codes),
                                        _ptr(v_codes), _ptr(k_params), _ptr(v_params),
                                        _ptr(slot_mapping), _ptr(block_tables),
                                        block_tables.shape[1], _ptr(context_lens),
                                        int(max_context_len), b, h, d, bs, nb, float(scale),
                                        _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)),
           "pa_decode_append_int8")


def new_grouped_workspace(num_seqs, num_groups, num_heads, head_dim, max_context_len,
                          max_blocks_per_seq, device="cuda"):
    """Workspace for pa_decode_grouped, zero-filled as its first use requires."""
    n = load().pa_decode_grouped_workspace_size(num_seqs, num_groups, num_heads, head_dim,
                                                max_context_len, max_blocks_per_seq)
    return torch.zeros(max(int(n), 16), dtype=torch.uint8, device=device)


def pa_decode_grouped(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len,
                      group_start, prefix_lens, max_group_size, scale, workspace, stream=None):
    """Decode of sequence groups sharing a block prefix: the prefix read once
    per (group, head) and scored for the whole group on the tensor cores,
    each member's tail scored alone, the parts merged.  Same result as
    pa_decode."""
    b, h, d = q.shape
    nb, hk, bs, dk = k_cache.shape
    assert q.dtype == out.dtype == k_cache.dtype == v_cache.dtype == torch.float16
    assert out.shape == q.shape and (hk, dk) == (h, d) and v_cache.shape == k_cache.shape
    assert block_tables.dtype == context_lens.dtype == group_start.dtype == torch.int32
    assert prefix_lens.dtype == torch.int32
    g = prefix_lens.numel()
    assert group_start.numel() == g + 1
    _check(load().pa_decode_grouped(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                                    int(max_context_len), _ptr(group_start), _ptr(prefix_lens), g,
                                    int(max_group_size), b, h, d, bs, nb, float(scale),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)),
           "pa_decode_grouped")


def pa_decode_contiguous(out, q, k, v, context_lens, max_context_len, scale, workspace,
                         stream=None):
    """The contiguous-cache baseline: decode over K / V [B, H, Lmax, D] laid
    out contiguously per (sequence, head), no block table."""
    b, h, d = q.shape
    bk, hk, lmax, dk = k.shape
    assert q.dtype == out.dtype == k.dtype == v.dtype == torch.float16
    assert out.shape == q.shape and (bk, hk, dk) == (b, h, d) and v.shape == k.shape
    assert context_lens.dtype == torch.int32
    _check(load().pa_decode_contiguous(_ptr(out), _ptr(q), _ptr(k), _ptr(v), _ptr(context_lens),
                                       int(max_context_len), lmax, b, h, d, float(scale),
                                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream)),
           "pa_decode_contiguous")


def pa_decode_no_alloc(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len,
                       scale, stream=None):
    """pa_decode with the library's static device scratch instead of a
    workspace, for callers that cannot allocate device memory at decode time
    (e.g. when the KV block pool has taken the free HBM).  Raises PAError
    (PA_ERR_WORKSPACE) for sizes past the 8 MiB scratch.  Calls sharing a
    device must not overlap on the GPU."""
    b, h, d = q.shape
    nb, hk, bs, dk = k_cache.shape
    assert q.dtype == out.dtype == k_cache.dtype == v_cache.dtype == torch.float16
    assert out.shape == q.shape and (hk, dk) == (h, d) and v_cache.shape == k_cache.shape
    assert block_tables.dtype == torch.int32 and block_tables.dim() == 2
    assert context_lens.dtype == torch.int32 and context_lens.numel() == b
    _check(load().pa_decode_no_alloc(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                     _ptr(block_tables), block_tables.shape[1],
                                     _ptr(context_lens), int(max_context_len), b, h, d, bs, nb,
                                     float(scale), _stream(stream)),
           "pa_decode_no_alloc")


def pa_copy_blocks(k_cache, v_cache, block_mapping, stream=None):
    """Copy whole blocks src -> dst for each (src, dst) row of block_mapping."""
    nb, h, bs, d = k_cache.shape
    assert block_mapping.dtype == torch.int64
    pairs = block_mapping.numel() // 2
    _check(load().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_mapping) if pairs
                                 else ctypes.c_void_p(None), pairs, h, d, bs, nb,
                                 _stream(stream)),
           "pa_copy_blocks")


def pa_selftest_bounded_wait(limit_us: int, stream=None):
    """Launch the bounded-wait self-test (a wait nothing completes)."""
    _check(load().pa_selftest_bounded_wait(int(limit_us), _stream(stream)),
           "pa_selftest_bounded_wait")


def pa_reshape_and_cache_int8(key, value, k_codes, v_codes, k_params, v_params, slot_mapping,
                              stream=None):
    """Quantize each token's K/V rows (8-bit affine, per row) into its slot."""
    n, h, d = key.shape
    nb, hk, bs, dk = k_codes.shape
    assert key.dtype == value.dtype == torch.float16 and k_codes.dtype == v_codes.dtype == torch.uint8
    assert k_params.dtype == v_params.dtype == torch.float32 and k_params.shape == (nb, h, bs, 2)
    assert slot_mapping.dtype == torch.int64 and slot_mapping.numel() == n and (hk, dk) == (h, d)
    _check(load().pa_reshape_and_cache_int8(_ptr(key), _ptr(value), _ptr(k_codes), _ptr(v_codes),
                                            _ptr(k_params), _ptr(v_params), _ptr(slot_mapping),
                                            n, h, d, bs, nb, _stream(stream)),
           "pa_reshape_and_cache_int8")


def pa_decode_int8(out, q, k_codes, v_codes, k_params, v_params, block_tables, context_lens,
                   max_context_len, scale, workspace, stream=None):
    """pa_decode over the int8 cache (dequantized rows s (q - z))."""
    b, h, d = q.shape
    nb, hk, bs, dk = k_codes.shape
    assert q.dtype == out.dtype == torch.float16 and k_codes.dtype == torch.uint8
    assert out.shape == q.shape and (hk, dk) == (h, d) and k_params.shape == (nb, h, bs, 2)
    assert block_tables.dtype == torch.int32 and context_lens.dtype == torch.int32
    _check(load().pa_decode_int8(_ptr(out), _ptr(q), _ptr(k_codes), _ptr(v_codes), _ptr(k_params),
                                 _ptr(v_params), _ptr(block_tables), block_tables.shape[1],
                                 _ptr(context_lens), int(max_context_len), b, h, d, bs, nb,
                                 float(scale), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "pa_decode_int8")


def pa_copy_blocks_raw(cache, block_mapping, stream=None):
    """Copy whole blocks (dim 0 of `cache`) src -> dst for each mapping row."""
    nb = cache.shape[0]
    block_bytes = cache[0].numel() * cache.element_size()
    pairs = block_mapping.numel() // 2
    _check(load().pa_copy_blocks_raw(_ptr(cache), block_bytes,
                                     _ptr(block_mapping) if pairs else ctypes.c_void_p(None),
                                     pairs, nb, _stream(stream)),
           "pa_copy_blocks_raw")


def _ptr_addressable(t: torch.Tensor) -> ctypes.c_void_p:
    """Device tensor, or page-locked host tensor the device can address."""
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError("pa_swap_blocks takes device or pinned host tensors")
    if t.is_cuda:
        _on_current_device(t)
    if not t.is_contiguous():
        raise ValueError("libpa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def pa_swap_blocks(src, dst, block_mapping, stream=None):
    """Copy whole blocks (dim 0) of pool `src` into pool `dst`, one of them
    typically pinned host memory: block_mapping[i] = (src block, dst block)."""
    assert src.dtype == dst.dtype and src.shape[1:] == dst.shape[1:]
    assert block_mapping.dtype == torch.int64
    block_bytes = src[0].numel() * src.element_size()
    pairs = block_mapping.numel() // 2
    _check(load().pa_swap_blocks(_ptr_addressable(src), _ptr_addressable(dst), block_bytes,
                                 _ptr_addressable(block_mapping) if pairs else ctypes.c_void_p(None),
                                 pairs, src.shape[0], dst.shape[0], _stream(stream)),
           "pa_swap_blocks")


def pa_prefill(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len,
               query_start_loc, max_query_len, scale, stream=None):
    """Causal multi-query attention of each sequence's new tokens (the last
    n_b of its context) over its paged cache, on the tensor cores."""
    t, h, d = q.shape
    nb, hk, bs, dk = k_cache.shape
    assert q.dtype == out.dtype == k_cache.dtype == v_cache.dtype == torch.float16
    assert out.shape == q.shape and (hk, dk) == (h, d) and v_cache.shape == k_cache.shape
    assert block_tables.dtype == context_lens.dtype == query_start_loc.dtype == torch.int32
    b = context_lens.numel()
    assert query_start_loc.numel() == b + 1
    _check(load().pa_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                             block_tables.shape[1], _ptr(context_lens), int(max_context_len),
                             _ptr(query_start_loc), t, int(max_query_len), b, h, d, bs, nb,
                             float(scale), _stream(stream)),
           "pa_prefill")


def pa_get_last_device_error() -> int:
    code = ctypes.c_uint(0)
    _check(load().pa_get_last_device_error(ctypes.byref(code)), "pa_get_last_device_error")
    return int(code.value)


class BlockManager:
    """Host KV block manager (C++ in libpa): shared free pool, reference
    counts, slot allocation per decode step, copy-on-write decisions and
    swapping of sequence groups to a host pool of num_cpu_blocks blocks."""

    def __init__(self, num_blocks: int, block_size: int, num_cpu_blocks: int = 0):
        self._lib = load()
        self._h = self._lib.pa_bm_create_with_swap(num_blocks, num_cpu_blocks, block_size)
        if not self._h:
            raise PAError(PA_ERR_INVALID_ARG, "pa_bm_create_with_swap")
        self.num_blocks, self.block_size = num_blocks, block_size
        self.num_cpu_blocks = num_cpu_blocks

    def close(self):
        if self._h:
            self._lib.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def num_free(self) -> int:
        return int(self._lib.pa_bm_num_free(self._h))

    def refcount(self, block: int) -> int:
        return int(self._lib.pa_bm_refcount(self._h, int(block)))

    def num_free_cpu(self) -> int:
        return int(self._lib.pa_bm_num_free_cpu(self._h))

    def cpu_refcount(self, block: int) -> int:
        return int(self._lib.pa_bm_cpu_refcount(self._h, int(block)))

    def is_swapped(self, seq: int) -> int:
        return int(self._lib.pa_bm_is_swapped(self._h, int(seq)))

    def _move(self, fn, name, seqs):
        import numpy as np
        ids = np.ascontiguousarray(seqs, dtype=np.int64)
        cap = max(1, self.num_blocks + self.num_cpu_blocks)
        pairs = np.empty((cap, 2), dtype=np.int64)
        npairs = ctypes.c_int(0)
        _check(fn(self._h, ids.ctypes.data, ids.shape[0], pairs.ctypes.data, cap,
                  ctypes.byref(npairs)), name)
        return pairs[:npairs.value].copy()

    def swap_out(self, seqs):
        """Move a sequence group to the host pool; (device, host) block pairs."""
        return self._move(self._lib.pa_bm_swap_out, "pa_bm_swap_out", seqs)

    def swap_in(self, seqs):
        """Move a swapped group back to the device; (host, device) block pairs."""
        return self._move(self._lib.pa_bm_swap_in, "pa_bm_swap_in", seqs)

    def add_sequence(self, seq: int, prompt_len: int):
        _check(self._lib.pa_bm_add_sequence(self._h, int(seq), int(prompt_len)), "pa_bm_add_sequence")

    def fork(self, parent: int, child: int):
        _check(self._lib.pa_bm_fork(self._h, int(parent), int(child)), "pa_bm_fork")

    def free_sequence(self, seq: int):
        _check(self._lib.pa_bm_free_sequence(self._h, int(seq)), "pa_bm_free_sequence")

    def append_slots(self, seqs):
        """Reserve each sequence's next slot.  Returns (slots int64 [n],
        cow_pairs int64 [p, 2])."""
        import numpy as np
        ids = np.ascontiguousarray(seqs, dtype=np.int64)
        n = ids.shape[0]
        slots = np.empty(n, dtype=np.int64)
        pairs = np.empty((max(n, 1), 2), dtype=np.int64)
        npairs = ctypes.c_int(0)
        _check(self._lib.pa_bm_append_slots(self._h, ids.ctypes.data, n, slots.ctypes.data,
                                            pairs.ctypes.data, ctypes.byref(npairs)),
               "pa_bm_append_slots")
        return slots, pairs[:npairs.value].copy()

    def block_tables(self, seqs, max_blocks: int):
        """(block_tables int32 [n, max_blocks] padded with -1, context_lens int32 [n])."""
        import numpy as np
        ids = np.ascontiguousarray(seqs, dtype=np.int64)
        n = ids.shape[0]
        tables = np.empty((n, max_blocks), dtype=np.int32)
        lens = np.empty(n, dtype=np.int32)
        _check(self._lib.pa_bm_block_tables(self._h, ids.ctypes.data, n, tables.ctypes.data,
                                            int(max_blocks), lens.ctypes.data),
               "pa_bm_block_tables")
        return tables, lens

