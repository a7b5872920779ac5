"""Pins for the fp64 CPU oracle: each test ties it to something other than
itself — a value the pages print, a closed form, a library routine (numpy's
binary16 decoding, torch's float64 scaled_dot_product_attention and softmax),
or an invariant the pages state.  They are chosen so that a plausible slip in
the oracle (a dropped scale, a wrong sign, a transposed index, an off-by-one
length, a bad fp16 decode) fails at least one of them."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_cache_481_b200 import accounting, workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _sdpa(q_row, k_logical, v_logical, scale):
    """Library attention in float64 on a contiguous [L, D] copy."""
    q = torch.as_tensor(np.asarray(q_row, dtype=np.float64)).view(1, 1, 1, -1)
    k = k_logical.double().view(1, 1, *k_logical.shape)
    v = v_logical.double().view(1, 1, *v_logical.shape)
    return F.scaled_dot_product_attention(q, k, v, scale=scale).view(-1).numpy()


def _complete_pool(wl):
    """Run the oracle's cache write so the pool holds every context token."""
    return oracle.reshape_and_cache(wl.new_key.numpy(), wl.new_value.numpy(),
                                    wl.k_cache.numpy(), wl.v_cache.numpy(),
                                    wl.slot_mapping, wl.block_size)


# ---------------------------------------------------------------- fp16 decode

def test_half_to_double_matches_numpy_on_every_bit_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    ours = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zero survives
    assert math.copysign(1.0, oracle.half_to_double(0x8000)) == -1.0


# ------------------------------------------------------ sizes the pages print

def test_kv_size_per_token_is_800_kib():
    g = _golden("kv_sizes.json")["per_token"]
    n = oracle.kv_cache_bytes(g["batch"], g["seq_len"], g["layers"], g["d_model"],
                              g["bytes_per_elem"])
    assert n == 2 * 5120 * 40 * 2 == 819200
    assert n / 1024 == g["printed_value"]


def test_kv_size_2048_token_request():
    g = _golden("kv_sizes.json")["request_2048"]
    n = oracle.kv_cache_bytes(g["batch"], g["seq_len"], g["layers"], g["d_model"],
                              g["bytes_per_elem"])
    assert n == 1677721600
    # the two pages print the same byte count once in GiB and once in GB
    assert round(n / 2**30, 1) == g["printed_gib_1dp"]
    assert round(n / 1e9, 1) == g["printed_gb_1dp"]


def test_kv_size_4096_token_request():
    g = _golden("kv_sizes.json")["request_4096"]
    n = oracle.kv_cache_bytes(g["batch"], g["seq_len"], g["layers"], g["d_model"],
                              g["bytes_per_elem"])
    assert n == 3355443200
    assert float(f"{n:.3g}") == g["printed_bytes_3sf"]
    assert round(n / 2**30, 1) == g["printed_gib_1dp"]


def test_benchmark_byte_accounting_reproduces_page_formula():
    # one layer of a 13B model: 40 heads x 128 = d_model 5120
    per_layer = accounting.kv_bytes_per_token(num_heads=40, head_dim=128)
    assert per_layer * 40 == oracle.kv_cache_bytes(1, 1, 40, 5120, 2)
    lens = np.array([2048])
    kv_only = accounting.decode_bytes(lens, 40, 128) - 40 * 2 * 128 * 2
    assert kv_only * 40 == oracle.kv_cache_bytes(1, 2048, 40, 5120, 2)


# --------------------------------------------------- block tables and paging

def _pool_from_table(table, k_logical, v_logical, num_blocks, bs):
    """Place a contiguous [H, L, D] sequence into a NaN-filled pool by writing
    logical block i into physical block table[i] (contiguous -> paged)."""
    h, length, d = k_logical.shape
    kc = np.full((num_blocks, h, bs, d), np.nan, dtype=np.float16)
    vc = np.full_like(kc, np.nan)
    for i, p in enumerate(table):
        lo, hi = i * bs, min((i + 1) * bs, length)
        if p is None or lo >= length:
            continue
        kc[p, :, : hi - lo, :] = k_logical[:, lo:hi, :].numpy()
        vc[p, :, : hi - lo, :] = v_logical[:, lo:hi, :].numpy()
    return kc, vc


@pytest.mark.parametrize("length", [12, 9, 1])
def test_slide10_block_table_gathers_in_logical_order(length):
    table = _golden("block_tables.json")["slide10_table"]["logical_to_physical"]
    bs, h, d, nb = 4, 3, 8, 8
    g = torch.Generator().manual_seed(10 + length)
    k = torch.randn(h, length, d, generator=g).half()
    v = torch.randn(h, length, d, generator=g).half()
    q = torch.randn(1, h, d, generator=g).half()
    kc, vc = _pool_from_table(table, k, v, nb, bs)
    row = np.array([-1 if p is None else p for p in table], dtype=np.int32)[None]
    out = oracle.paged_decode(q.numpy(), kc, vc, row, np.array([length], np.int32), 0.37)
    for hh in range(h):
        ref = _sdpa(q[0, hh].double().numpy(), k[hh], v[hh], 0.37)
        np.testing.assert_allclose(out[0, hh], ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("seed,d,bs,lens", [
    (1, 64, 16, [1, 17, 33, 50]),
    (2, 128, 16, [16, 31, 100, 257]),
    (3, 64, 8, [7, 8, 9, 64]),
    (4, 128, 32, [5, 96, 130]),
    (5, 64, 64, [63, 64, 65, 200]),
    (6, 128, 128, [129, 3, 384]),
])
def test_paged_equals_contiguous_sdpa_under_random_placement(seed, d, bs, lens):
    wl = workloads.make_random(seed, lens, num_heads=3, head_dim=d, block_size=bs,
                               pool_factor=2.0)
    kc, vc = _complete_pool(wl)
    out = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables, wl.context_lens,
                              wl.scale)
    for b in range(wl.num_seqs):
        for h in range(wl.num_heads):
            ref = _sdpa(wl.q[b, h].double().numpy(), wl.logical_k[b][h],
                        wl.logical_v[b][h], wl.scale)
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-11, atol=1e-13)


def test_result_independent_of_physical_permutation():
    wl = workloads.make_random(7, [40, 77, 5], num_heads=2, head_dim=64, block_size=16,
                               pool_factor=3.0)
    kc, vc = _complete_pool(wl)
    base = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables, wl.context_lens,
                               wl.scale)
    rng = np.random.default_rng(0)
    perm = rng.permutation(wl.num_blocks)          # new physical id of each block
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    tables2 = np.where(wl.block_tables >= 0, perm[np.maximum(wl.block_tables, 0)], -1)
    moved = oracle.paged_decode(wl.q.numpy(), kc2, vc2, tables2.astype(np.int32),
                                wl.context_lens, wl.scale)
    assert np.array_equal(base, moved)


# ------------------------------------------------------------ softmax facts

def test_softmax_weights_sum_to_one_and_match_library_softmax():
    wl = workloads.make_random(8, [3, 50, 129], num_heads=2, head_dim=128, block_size=16)
    kc, vc = _complete_pool(wl)
    out, probs = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables,
                                     wl.context_lens, wl.scale, return_probs=True)
    for b, length in enumerate(wl.context_lens):
        for h in range(wl.num_heads):
            p = probs[b, h, :length]
            assert abs(p.sum() - 1.0) < 1e-12
            s = (wl.logical_k[b][h].double() @ wl.q[b, h].double()) * wl.scale
            np.testing.assert_allclose(p, torch.softmax(s, 0).numpy(), rtol=1e-12,
                                       atol=1e-15)
            assert np.all(probs[b, h, length:] == 0)


def test_single_token_context_returns_v0_exactly():
    wl = workloads.make_random(9, [1, 1], num_heads=4, head_dim=64, block_size=16)
    kc, vc = _complete_pool(wl)
    out = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables, wl.context_lens,
                              wl.scale)
    for b in range(2):
        assert np.array_equal(out[b], wl.logical_v[b][:, 0].double().numpy())


def test_zero_query_gives_mean_of_values():
    wl = workloads.make_random(10, [37, 64], num_heads=2, head_dim=64, block_size=16)
    kc, vc = _complete_pool(wl)
    q0 = np.zeros(wl.q.shape, dtype=np.float16)
    out = oracle.paged_decode(q0, kc, vc, wl.block_tables, wl.context_lens, wl.scale)
    for b in range(2):
        np.testing.assert_allclose(out[b], wl.logical_v[b].double().mean(dim=1).numpy(),
                                   rtol=1e-13, atol=1e-15)


def test_equal_keys_give_mean_of_values():
    wl = workloads.make_random(11, [45], num_heads=2, head_dim=64, block_size=16)
    kc, vc = _complete_pool(wl)
    used = wl.block_tables[0][wl.block_tables[0] >= 0]
    kc[used] = np.float16(0.25)                    # every key identical
    out = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables, wl.context_lens,
                              wl.scale)
    np.testing.assert_allclose(out[0], wl.logical_v[0].double().mean(dim=1).numpy(),
                               rtol=1e-13, atol=1e-15)


def test_dominant_key_selects_its_value():
    wl = workloads.make_random(12, [40], num_heads=1, head_dim=64, block_size=16)
    kc, vc = _complete_pool(wl)
    q = np.ones(wl.q.shape, dtype=np.float16)
    t = 23
    p = wl.block_tables[0][t // 16]
    kc[p, 0, t % 16, :] = np.float16(8.0)          # score 8 * 64 / 8 = 64 above ~N(0,1)
    out = oracle.paged_decode(q, kc, vc, wl.block_tables, wl.context_lens, wl.scale)
    np.testing.assert_allclose(out[0, 0], wl.logical_v[0][0, t].double().numpy(),
                               rtol=0, atol=1e-12)


def test_two_token_closed_form_logistic():
    # out = sigma(s0 - s1) V0 + sigma(s1 - s0) V1 with s_t = scale * q.K_t
    bs, d = 16, 64
    g = torch.Generator().manual_seed(13)
    k = torch.randn(1, 2, d, generator=g).half()
    v = torch.randn(1, 2, d, generator=g).half()
    q = torch.randn(1, 1, d, generator=g).half()
    kc, vc = _pool_from_table([2], k, v, 4, bs)
    for scale in (0.125, 1.0, 0.02):
        out = oracle.paged_decode(q.numpy(), kc, vc, np.array([[2]], np.int32),
                                  np.array([2], np.int32), scale)
        qd = q[0, 0].double()
        s0 = scale * float(qd @ k[0, 0].double())
        s1 = scale * float(qd @ k[0, 1].double())
        a = 1.0 / (1.0 + math.exp(s1 - s0))
        ref = a * v[0, 0].double().numpy() + (1.0 - a) * v[0, 1].double().numpy()
        np.testing.assert_allclose(out[0, 0], ref, rtol=1e-13, atol=1e-15)


def test_empty_context_gives_zeros():
    wl = workloads.make_random(14, [5], num_heads=2, head_dim=64, block_size=16)
    kc, vc = _complete_pool(wl)
    out = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables,
                              np.array([0], np.int32), wl.scale)
    assert np.array_equal(out, np.zeros_like(out))


# ------------------------------------------------------------- cache write

def test_cache_write_completes_the_sequence_and_touches_nothing_else():
    wl = workloads.make_workload(1, keep_logical=True)
    kc0, vc0 = wl.k_cache.numpy(), wl.v_cache.numpy()
    kc, vc = _complete_pool(wl)
    # exactly N x H rows of D elements changed, in each cache
    changed = np.any(kc.view(np.uint16) != kc0.view(np.uint16), axis=-1)
    assert changed.sum() == wl.num_seqs * wl.num_heads
    changed_v = np.any(vc.view(np.uint16) != vc0.view(np.uint16), axis=-1)
    assert changed_v.sum() == wl.num_seqs * wl.num_heads
    # and the decode now equals attention over the full logical sequence
    out = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables, wl.context_lens,
                              wl.scale)
    for b in range(wl.num_seqs):
        for h in range(wl.num_heads):
            ref = _sdpa(wl.q[b, h].double().numpy(), wl.logical_k[b][h],
                        wl.logical_v[b][h], wl.scale)
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-11, atol=1e-13)


def test_cache_write_without_it_the_canary_shows():
    wl = workloads.make_workload(1)
    out = oracle.paged_decode(wl.q.numpy(), wl.k_cache.numpy(), wl.v_cache.numpy(),
                              wl.block_tables, wl.context_lens, wl.scale)
    assert np.isnan(out).all()


def test_cache_write_skips_negative_slots():
    wl = workloads.make_workload(1)
    slots = wl.slot_mapping.copy()
    slots[1] = -1
    kc, vc = oracle.reshape_and_cache(wl.new_key.numpy(), wl.new_value.numpy(),
                                      wl.k_cache.numpy(), wl.v_cache.numpy(), slots, 16)
    changed = np.any(kc.view(np.uint16) != wl.k_cache.numpy().view(np.uint16), axis=-1)
    assert changed.sum() == (wl.num_seqs - 1) * wl.num_heads
    out = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert np.isnan(out[1]).all() and not np.isnan(np.delete(out, 1, axis=0)).any()


def test_cache_write_rejects_slot_past_pool():
    wl = workloads.make_workload(1)
    slots = wl.slot_mapping.copy()
    slots[0] = wl.num_blocks * wl.block_size
    with pytest.raises(oracle.OracleError):
        oracle.reshape_and_cache(wl.new_key.numpy(), wl.new_value.numpy(),
                                 wl.k_cache.numpy(), wl.v_cache.numpy(), slots, 16)


def test_decode_rejects_block_id_past_pool():
    wl = workloads.make_workload(1)
    kc, vc = _complete_pool(wl)
    tables = wl.block_tables.copy()
    tables[3, 0] = wl.num_blocks
    with pytest.raises(oracle.OracleError):
        oracle.paged_decode(wl.q.numpy(), kc, vc, tables, wl.context_lens, wl.scale)


# --------------------------------------------------------- copy-on-write

def test_cow_example_from_parallel_sampling():
    ex = _golden("block_tables.json")["cow_parallel_sampling"]
    bs, h, d, nb = 4, 2, 16, 4
    g = torch.Generator().manual_seed(15)
    k = torch.randn(h, 7, d, generator=g).half()   # 7 tokens: blocks 0 (full), 1 (3 rows)
    v = torch.randn(h, 7, d, generator=g).half()
    q = torch.randn(2, h, d, generator=g).half()
    kc, vc = _pool_from_table(ex["shared_before"]["A1"], k, v, nb, bs)
    before = oracle.paged_decode(q.numpy(), kc, vc,
                                 np.array([ex["shared_before"]["A1"],
                                           ex["shared_before"]["A2"]], np.int32),
                                 np.array([7, 7], np.int32), 0.25)
    kc2, vc2 = oracle.copy_blocks(kc, vc, [[ex["copy"]["src"], ex["copy"]["dst"]]])
    assert np.array_equal(kc2[3].view(np.uint16), kc2[1].view(np.uint16))
    assert np.array_equal(vc2[3].view(np.uint16), vc2[1].view(np.uint16))
    for p in (0, 1, 2):                           # every other block unchanged
        assert np.array_equal(kc2[p].view(np.uint16), kc[p].view(np.uint16))
    after = oracle.paged_decode(q.numpy(), kc2, vc2,
                                np.array([ex["after"]["A1"], ex["after"]["A2"]], np.int32),
                                np.array([7, 7], np.int32), 0.25)
    assert np.array_equal(before, after)


def test_shared_prefix_aliasing_equals_private_copies():
    wl = workloads.make_shared_prefix(num_groups=2, group_size=3, prefix_len=64,
                                      num_heads=2, head_dim=64, block_size=16,
                                      keep_logical=True)
    kc, vc = _complete_pool(wl)
    alias = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.alias_block_tables,
                                wl.context_lens, wl.scale)
    kc2, vc2 = oracle.copy_blocks(kc, vc, wl.copy_pairs)
    cow = oracle.paged_decode(wl.q.numpy(), kc2, vc2, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert np.array_equal(alias, cow)
    for b in range(wl.num_seqs):
        ref = _sdpa(wl.q[b, 1].double().numpy(), wl.logical_k[b][1], wl.logical_v[b][1],
                    wl.scale)
        np.testing.assert_allclose(cow[b, 1], ref, rtol=1e-11, atol=1e-13)
    # before the copy the private blocks are canary: the CoW tables see NaN
    stale = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables, wl.context_lens,
                                wl.scale)
    assert np.isnan(stale).all()


def test_copy_blocks_rejects_bad_ids():
    wl = workloads.make_workload(1)
    with pytest.raises(oracle.OracleError):
        oracle.copy_blocks(wl.k_cache.numpy(), wl.v_cache.numpy(), [[0, wl.num_blocks]])
