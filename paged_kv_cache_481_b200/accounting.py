"""Algorithmic byte counts used by the benchmark's throughput and roofline.

Bytes are what the operation must move at minimum, counted from exact token
counts (not rounded to blocks); block tables, context lengths and split-K
partials are implementation overhead and are not counted.
"""
from __future__ import annotations

import numpy as np

FP16_BYTES = 2


def kv_bytes_per_token(num_heads: int, head_dim: int, elem_bytes: int = FP16_BYTES) -> int:
    """K and V bytes one token occupies in one layer's cache: 2 * H * D * s."""
    return 2 * num_heads * head_dim * elem_bytes


def decode_bytes(context_lens, num_heads: int, head_dim: int,
                 elem_bytes: int = FP16_BYTES) -> int:
    """K + V read for every context token, plus q read and out written, over
    all (sequence, head): sum_b H * (2 * L_b * D * s + 2 * D * s)."""
    lens = np.asarray(context_lens, dtype=np.int64)
    per_head = 2 * lens * head_dim * elem_bytes + 2 * head_dim * elem_bytes
    return int(num_heads * per_head.sum())


def decode_unique_bytes(block_tables, context_lens, num_heads: int, head_dim: int,
                        block_size: int, elem_bytes: int = FP16_BYTES) -> int:
    """Like decode_bytes but counting each physical (block, row) once: the
    bytes DRAM must deliver when aliased blocks are shared between sequences."""
    rows = {}
    tables = np.asarray(block_tables)
    for b, length in enumerate(np.asarray(context_lens)):
        length = int(length)
        nblk = (length + block_size - 1) // block_size
        for i in range(nblk):
            used = min(block_size, length - i * block_size)
            p = int(tables[b, i])
            rows[p] = max(rows.get(p, 0), used)
    kv = sum(rows.values()) * kv_bytes_per_token(num_heads, head_dim, elem_bytes)
    qo = len(np.asarray(context_lens)) * num_heads * 2 * head_dim * elem_bytes
    return int(kv + qo)


def cache_write_bytes(num_valid_tokens: int, num_heads: int, head_dim: int,
                      elem_bytes: int = FP16_BYTES) -> int:
    """K and V rows read from the new-token buffers and written to the pool."""
    return 2 * num_valid_tokens * kv_bytes_per_token(num_heads, head_dim, elem_bytes)


def copy_blocks_bytes(num_pairs: int, num_heads: int, head_dim: int, block_size: int,
                      elem_bytes: int = FP16_BYTES) -> int:
    """Whole K and V blocks read from src and written to dst."""
    return 2 * num_pairs * block_size * kv_bytes_per_token(num_heads, head_dim, elem_bytes)


def decode_bytes_int8(context_lens, num_heads: int, head_dim: int) -> int:
    """Int8 cache: per context token and head, K and V codes (D bytes each)
    and their (s, z) float pairs (8 bytes each), plus q read and out written
    in fp16."""
    lens = np.asarray(context_lens, dtype=np.int64)
    per_head = lens * 2 * (head_dim + 8) + 2 * head_dim * FP16_BYTES
    return int(num_heads * per_head.sum())

