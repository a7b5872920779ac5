"""Plain fp64 CPU oracle for the PagedAttention decode path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports, links or runs anything here, and nothing here imports the product.

The arithmetic lives in ``pa_oracle.c`` (plain C, double precision, OpenMP over
(sequence, head)); this module compiles it with gcc on first use and marshals
numpy arrays through ctypes.  fp16 arrays are passed as their uint16 bit
patterns and widened exactly inside the C code.

Passages followed (page title, section):
  * comfyai.app "6.4 PagedAttention", 6.4.1 Mechanism and 6.4.2-6.4.3
    (blocks, block table, sharing, copy-on-write);
  * brentwoodlivery.com "5.3.18 LLM serving, vLLM, quantized inference"
    (KV size formula 2*B*S*L*d_model*p; attention math unchanged by paging);
  * polomodov.tech "vLLM and PagedAttention", slides 5, 9, 10, 11, 13, 15.

Every function is pinned by ``tests/test_oracle_pins.py`` to values the pages
print, closed forms, library routines or invariants; no function here is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK, ERR_ARG, ERR_RANGE = 0, 1, 2


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into oracle/liboracle.so with gcc (-O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-pthread", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        # PA_ORACLE_LIB points the tests' mutation check at a deliberately
        # broken copy of this oracle; normal use builds and loads pa_oracle.c.
        lib = ctypes.CDLL(os.environ.get("PA_ORACLE_LIB") or build())
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_kv_cache_bytes.argtypes = [i64, i64, i64, i64, i64]
        lib.oracle_kv_cache_bytes.restype = i64
        lib.oracle_reshape_and_cache.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32]
        lib.oracle_reshape_and_cache.restype = i32
        lib.oracle_copy_blocks.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32]
        lib.oracle_copy_blocks.restype = i32
        lib.oracle_paged_decode.argtypes = [vp, vp, i64, vp, vp, vp, vp, i32, vp,
                                            i32, i32, i32, i32, i32, ctypes.c_double]
        lib.oracle_paged_decode.restype = i32
        lib.oracle_quantize_rows.argtypes = [vp, i32, i32, i32, vp, vp]
        lib.oracle_quantize_rows.restype = i32
        lib.oracle_reshape_and_cache_int8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                                      i32, i32]
        lib.oracle_reshape_and_cache_int8.restype = i32
        lib.oracle_paged_decode_int8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32,
                                                 i32, i32, i32, ctypes.c_double]
        lib.oracle_paged_decode_int8.restype = i32
        lib.oracle_paged_prefill.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32,
                                             i32, ctypes.c_double]
        lib.oracle_paged_prefill.restype = i32
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = i32
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _bits(a) -> np.ndarray:
    """fp16 array (numpy float16 or uint16 bit patterns) -> contiguous uint16."""
    a = np.asarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected fp16/uint16 array, got {a.dtype}")
    return np.ascontiguousarray(a)


def _check(rc: int, what: str):
    if rc != OK:
        raise OracleError(f"{what}: oracle returned {rc}")


def half_to_double(bits) -> float:
    """Exact IEEE binary16 -> double of one 16-bit pattern."""
    return _load().oracle_half_to_double(int(bits) & 0xFFFF)


def kv_cache_bytes(batch: int, seq_len: int, layers: int, d_model: int,
                   bytes_per_elem: int) -> int:
    """KV cache bytes = 2 * B * S * L * d_model * p (brentwoodlivery.com 5.3.18)."""
    return int(_load().oracle_kv_cache_bytes(batch, seq_len, layers, d_model,
                                             bytes_per_elem))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, block_size):
    """Return new (k_cache, v_cache) after writing each token at its slot.

    key/value [N, H, D] fp16; caches [NB, H, bs, D] fp16; slot_mapping [N]
    int64, negative = skip.  Inputs are not modified."""
    key, value = _bits(key), _bits(value)
    kc, vc = _bits(k_cache).copy(), _bits(v_cache).copy()
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    n, h, d = key.shape
    nb = kc.shape[0]
    assert kc.shape == (nb, h, block_size, d) and vc.shape == kc.shape
    assert value.shape == key.shape and slots.shape == (n,)
    rc = _load().oracle_reshape_and_cache(_ptr(key), _ptr(value), _ptr(kc), _ptr(vc),
                                          _ptr(slots), n, h, d, block_size, nb)
    _check(rc, "reshape_and_cache")
    return kc.view(np.float16), vc.view(np.float16)


def copy_blocks(k_cache, v_cache, block_mapping):
    """Return new (k_cache, v_cache) with block dst := block src for each pair."""
    kc, vc = _bits(k_cache).copy(), _bits(v_cache).copy()
    mapping = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    nb, h, bs, d = kc.shape
    rc = _load().oracle_copy_blocks(_ptr(kc), _ptr(vc), _ptr(mapping), mapping.shape[0],
                                    h, d, bs, nb)
    _check(rc, "copy_blocks")
    return kc.view(np.float16), vc.view(np.float16)


def swap_blocks(src_pool, dst_pool, block_mapping):
    """polomodov.tech slide 15 (a preempted request comes back by swapping):
    return a copy of dst_pool in which block dst of each (src, dst) pair holds
    src_pool's block src, byte for byte.  Pools are arrays whose first axis
    indexes blocks."""
    src = np.asarray(src_pool)
    out = np.array(dst_pool, copy=True)
    assert src.dtype == out.dtype and src.shape[1:] == out.shape[1:]
    for s, d in np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2):
        if not (0 <= s < src.shape[0] and 0 <= d < out.shape[0]):
            raise ValueError("swap pair outside the pools")
        out[d] = src[s]
    return out


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale,
                 return_probs: bool = False):
    """fp64 paged decode attention.

    q [B, H, D] fp16; caches [NB, H, bs, D] fp16; block_tables [B, MB] int32;
    context_lens [B] int32.  Returns out [B, H, D] float64 and, if asked, the
    softmax weights [B, H, max(context_lens)] float64 (zero past each length).
    """
    q = _bits(q)
    kc, vc = _bits(k_cache), _bits(v_cache)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    b, h, d = q.shape
    nb, hk, bs, dk = kc.shape
    assert (hk, dk) == (h, d) and vc.shape == kc.shape
    assert tables.ndim == 2 and tables.shape[0] == b and lens.shape == (b,)
    out = np.zeros((b, h, d), dtype=np.float64)
    probs = None
    stride = 0
    if return_probs:
        stride = max(int(lens.max()) if b else 0, 1)
        probs = np.zeros((b, h, stride), dtype=np.float64)
    rc = _load().oracle_paged_decode(_ptr(out), _ptr(probs), stride, _ptr(q), _ptr(kc),
                                     _ptr(vc), _ptr(tables), tables.shape[1], _ptr(lens),
                                     b, h, d, bs, nb, float(scale))
    _check(rc, "paged_decode")
    return (out, probs) if return_probs else out


# ---------------------------------------------------------------- int8 KV

def quantize_rows(x, bits: int = 8):
    """Affine quantization of each row of x ([n, D] fp16), brentwoodlivery.com
    5.3.18: returns (codes uint8 [n, D], params float32 [n, 2] = (s, z))."""
    x = _bits(x)
    n, d = x.shape
    codes = np.zeros((n, d), dtype=np.uint8)
    params = np.zeros((n, 2), dtype=np.float32)
    _check(_load().oracle_quantize_rows(_ptr(x), n, d, bits, _ptr(codes), _ptr(params)),
           "quantize_rows")
    return codes, params


def dequantize(codes, params):
    """r_hat = s (q - z), in float64."""
    p = np.asarray(params, dtype=np.float64)
    return p[..., 0:1] * (np.asarray(codes, dtype=np.float64) - p[..., 1:2])


def reshape_and_cache_int8(key, value, k_codes, v_codes, k_params, v_params, slot_mapping,
                           block_size):
    """Return new (k_codes, v_codes, k_params, v_params) after quantizing each
    token's rows into its slot (negative slots skipped).  Inputs unchanged."""
    key, value = _bits(key), _bits(value)
    kc, vc = np.ascontiguousarray(k_codes, np.uint8).copy(), np.ascontiguousarray(v_codes, np.uint8).copy()
    kp, vp_ = np.ascontiguousarray(k_params, np.float32).copy(), np.ascontiguousarray(v_params, np.float32).copy()
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    n, h, d = key.shape
    nb = kc.shape[0]
    assert kc.shape == (nb, h, block_size, d) and kp.shape == (nb, h, block_size, 2)
    rc = _load().oracle_reshape_and_cache_int8(_ptr(key), _ptr(value), _ptr(kc), _ptr(vc),
                                               _ptr(kp), _ptr(vp_), _ptr(slots), n, h, d,
                                               block_size, nb)
    _check(rc, "reshape_and_cache_int8")
    return kc, vc, kp, vp_


def paged_decode_int8(q, k_codes, v_codes, k_params, v_params, block_tables, context_lens, scale):
    """fp64 paged decode over the dequantized int8 cache: out [B, H, D] float64."""
    q = _bits(q)
    kc, vc = np.ascontiguousarray(k_codes, np.uint8), np.ascontiguousarray(v_codes, np.uint8)
    kp, vp_ = np.ascontiguousarray(k_params, np.float32), np.ascontiguousarray(v_params, np.float32)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    b, h, d = q.shape
    nb, hk, bs, dk = kc.shape
    assert (hk, dk) == (h, d) and kp.shape == (nb, h, bs, 2)
    out = np.zeros((b, h, d), dtype=np.float64)
    rc = _load().oracle_paged_decode_int8(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(kp),
                                          _ptr(vp_), _ptr(tables), tables.shape[1], _ptr(lens),
                                          b, h, d, bs, nb, float(scale))
    _check(rc, "paged_decode_int8")
    return out


def paged_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale):
    """fp64 multi-query (chunked prefill) paged attention.  q [T, H, D] fp16
    holds each sequence's new tokens (rows query_start_loc[b] ..
    query_start_loc[b+1]); token i of sequence b is at position
    context_lens[b] - n_b + i and attends to cached positions <= its own.
    Returns out [T, H, D] float64."""
    q = _bits(q)
    kc, vc = _bits(k_cache), _bits(v_cache)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
    t, h, d = q.shape
    nb, hk, bs, dk = kc.shape
    assert (hk, dk) == (h, d) and vc.shape == kc.shape and qsl[-1] == t
    out = np.zeros((t, h, d), dtype=np.float64)
    rc = _load().oracle_paged_prefill(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(tables),
                                      tables.shape[1], _ptr(lens), _ptr(qsl), len(lens), h, d, bs,
                                      nb, float(scale))
    _check(rc, "paged_prefill")
    return out

