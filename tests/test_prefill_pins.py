"""Pins for the multi-query (chunked prefill) oracle: library causal
attention on the contiguous sequences (torch float64 scaled_dot_product_attention
with is_causal, or with the explicit mask of a chunk that continues a cached
context), and the decode oracle for one-token chunks."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_cache_481_b200 import workloads


def _complete(wl):
    return oracle.reshape_and_cache(wl.new_key.numpy(), wl.new_value.numpy(), wl.k_cache.numpy(),
                                    wl.v_cache.numpy(), wl.slot_mapping, wl.block_size)


def _queries(lens, n_new, h, d, seed):
    g = torch.Generator().manual_seed(seed)
    qsl = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    q = torch.randn((int(qsl[-1]), h, d), generator=g).half()
    return q, qsl


@pytest.mark.parametrize("seed,d,bs,lens,frac", [
    (1, 64, 16, [1, 17, 40], 1.0),      # whole prompts
    (2, 128, 16, [130, 33, 5], 0.5),     # chunks continuing a cached context
    (3, 128, 8, [64, 9, 100], 0.25),
    (4, 64, 32, [50, 200], 0.1),
])
def test_prefill_equals_masked_library_attention(seed, d, bs, lens, frac):
    wl = workloads.make_random(seed, lens, num_heads=3, head_dim=d, block_size=bs, pool_factor=2.0)
    kc, vc = _complete(wl)
    n_new = [max(1, int(round(frac * x))) for x in lens]
    q, qsl = _queries(lens, n_new, 3, d, seed + 100)
    out = oracle.paged_prefill(q.numpy(), kc, vc, wl.block_tables, wl.context_lens, qsl, wl.scale)
    for b, (length, n) in enumerate(zip(lens, n_new)):
        k = wl.logical_k[b].double().unsqueeze(0)          # [1, H, L, D]
        v = wl.logical_v[b].double().unsqueeze(0)
        qb = q[qsl[b]:qsl[b + 1]].double().permute(1, 0, 2).unsqueeze(0)   # [1, H, n, D]
        if n == length:
            ref = F.scaled_dot_product_attention(qb, k, v, is_causal=True, scale=wl.scale)
        else:
            pos = np.arange(length - n, length)[:, None]
            mask = torch.from_numpy(np.arange(length)[None, :] <= pos)
            ref = F.scaled_dot_product_attention(qb, k, v, attn_mask=mask, scale=wl.scale)
        got = out[qsl[b]:qsl[b + 1]]
        np.testing.assert_allclose(got, ref[0].permute(1, 0, 2).numpy(), rtol=1e-11, atol=1e-12)


def test_one_token_chunks_are_decode():
    wl = workloads.make_random(5, [1, 30, 77], num_heads=2, head_dim=64, block_size=16)
    kc, vc = _complete(wl)
    qsl = np.arange(4, dtype=np.int32)
    dec = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables, wl.context_lens, wl.scale)
    pre = oracle.paged_prefill(wl.q.numpy(), kc, vc, wl.block_tables, wl.context_lens, qsl, wl.scale)
    assert np.array_equal(dec, pre)


def test_prefill_rejects_more_queries_than_context():
    wl = workloads.make_random(6, [4], num_heads=1, head_dim=64, block_size=16)
    kc, vc = _complete(wl)
    q = np.zeros((5, 1, 64), np.float16)
    with pytest.raises(oracle.OracleError):
        oracle.paged_prefill(q, kc, vc, wl.block_tables, wl.context_lens, [0, 5], wl.scale)
