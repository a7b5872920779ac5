"""GPU parity of the int8 KV cache (brentwoodlivery.com 5.3.18, affine
8-bit per (token, head) row): the quantizing cache write must produce the
oracle's codes and (s, z) bit for bit (both decide in fp32), and the decode
over the int8 cache must match the oracle's fp64 decode of the dequantized
rows within max-abs 2e-3."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_481_b200 import binding, build, workloads

from gpu_helpers import ATOL, max_abs_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    binding.load()
    torch.cuda.init()


def _empty_int8(wl, device="cuda"):
    nb, h, bs, d = wl.num_blocks, wl.num_heads, wl.block_size, wl.head_dim
    codes = [torch.zeros((nb, h, bs, d), dtype=torch.uint8, device=device) for _ in range(2)]
    params = [torch.zeros((nb, h, bs, 2), dtype=torch.float32, device=device) for _ in range(2)]
    return codes + params


def _gpu_int8_pool(wl, seqs=None):
    keys, values, slots = workloads.all_token_writes(wl, seqs)
    kc, vc, kp, vp = _empty_int8(wl)
    binding.pa_reshape_and_cache_int8(keys.cuda(), values.cuda(), kc, vc, kp, vp,
                                      torch.from_numpy(slots).cuda())
    return (kc, vc, kp, vp), (keys, values, slots)


def _oracle_int8_pool(wl, keys, values, slots):
    kc, vc, kp, vp = (x.cpu().numpy() for x in _empty_int8(wl, device="cpu"))
    return oracle.reshape_and_cache_int8(keys.cpu().numpy(), values.cpu().numpy(), kc, vc, kp, vp,
                                         slots, wl.block_size)


def _decode(wl, pool, tables=None, lens=None, mcl=None):
    kc, vc, kp, vp = pool
    q = wl.q.cuda()
    out = torch.empty_like(q)
    tables = torch.from_numpy(np.ascontiguousarray(wl.block_tables if tables is None else tables)).cuda()
    lens = torch.from_numpy(wl.context_lens if lens is None else lens).cuda()
    mcl = wl.max_context_len if mcl is None else mcl
    ws = binding.new_workspace(wl.num_seqs, wl.num_heads, wl.head_dim, mcl)
    binding.pa_decode_int8(out, q, kc, vc, kp, vp, tables, lens, mcl, wl.scale, ws)
    return out


CASES = [
    (201, 128, 16, [1, 2, 31, 32, 33, 500, 1100]),
    (202, 128, 8, [7, 9, 64, 300]),
    (203, 128, 32, [31, 33, 700]),
    (204, 128, 64, [65, 128, 900]),
    (205, 128, 128, [1, 129, 1030]),
    (206, 64, 16, [1, 17, 50, 640]),
    (207, 64, 8, [3, 33, 520]),
    (208, 64, 128, [129, 600]),
]


@pytest.mark.parametrize("seed,d,bs,lens", CASES)
def test_int8_write_is_bit_exact_and_decode_matches(seed, d, bs, lens):
    wl = workloads.make_random(seed, lens, num_heads=5, head_dim=d, block_size=bs,
                               keep_logical=False, keep_tokens=True, pool_factor=2.0)
    pool, (keys, values, slots) = _gpu_int8_pool(wl)
    ref_pool = _oracle_int8_pool(wl, keys, values, slots)
    for got, want in zip(pool, ref_pool):
        assert np.array_equal(got.cpu().numpy().view(np.uint8), np.asarray(want).view(np.uint8))
    out = _decode(wl, pool)
    ref = oracle.paged_decode_int8(wl.q.numpy(), *ref_pool, wl.block_tables, wl.context_lens,
                                   wl.scale)
    assert max_abs_err(out, ref) <= ATOL
    assert binding.pa_get_last_device_error() == 0


def test_int8_write_edge_rows():
    """Constant rows, zero rows, large offsets and huge magnitudes quantize
    identically on both sides; negative slots are skipped."""
    h, d, bs, nb = 3, 128, 16, 4
    g = torch.Generator().manual_seed(7)
    rows = torch.randn((6, h, d), generator=g)
    rows[0] = 0.0
    rows[1] = 0.75
    rows[2] = rows[2] * 1e-3 + 100.0
    rows[3] = rows[3] * 3000.0
    rows[4, 0] = -65504.0
    keys = rows.half()
    values = (rows * -0.5).half()         # stays finite (codes of inf/NaN rows are unspecified)
    assert torch.isfinite(keys.float()).all() and torch.isfinite(values.float()).all()
    slots = np.array([0, 5, -1, 17, 33, 63], np.int64)
    kc, vc, kp, vp = (torch.zeros((nb, h, bs, d), dtype=torch.uint8, device="cuda"),
                      torch.zeros((nb, h, bs, d), dtype=torch.uint8, device="cuda"),
                      torch.zeros((nb, h, bs, 2), dtype=torch.float32, device="cuda"),
                      torch.zeros((nb, h, bs, 2), dtype=torch.float32, device="cuda"))
    binding.pa_reshape_and_cache_int8(keys.cuda(), values.cuda(), kc, vc, kp, vp,
                                      torch.from_numpy(slots).cuda())
    ref = oracle.reshape_and_cache_int8(keys.numpy(), values.numpy(),
                                        np.zeros((nb, h, bs, d), np.uint8),
                                        np.zeros((nb, h, bs, d), np.uint8),
                                        np.zeros((nb, h, bs, 2), np.float32),
                                        np.zeros((nb, h, bs, 2), np.float32), slots, bs)
    for got, want in zip((kc, vc, kp, vp), ref):
        assert np.array_equal(got.cpu().numpy().view(np.uint8), want.view(np.uint8))
    # the constant row dequantizes exactly
    assert np.array_equal(oracle.dequantize(ref[0][0, :, 5], ref[2][0, :, 5]),
                          np.full((h, d), 0.75))


def test_int8_copy_on_write_with_raw_block_copies():
    wl = workloads.make_shared_prefix(num_groups=2, group_size=3, prefix_len=64, num_heads=4,
                                      head_dim=128, block_size=16, device="cuda")
    # write every context token of the aliased layout (shared prefix blocks once per group)
    keys, values, slots = [], [], []
    prefix, bs = 64, 16
    for s in range(wl.num_seqs):
        length = int(wl.context_lens[s])
        for t in range(length):
            if t < prefix and s % 3:   # prefix rows come from the group's first member
                continue
            slots.append(int(wl.alias_block_tables[s, t // bs]) * bs + t % bs)
    # values: fresh random rows per written slot
    g = torch.Generator(device="cuda").manual_seed(3)
    n = len(slots)
    keys = torch.randn((n, 4, 128), generator=g, device="cuda").half()
    values = torch.randn((n, 4, 128), generator=g, device="cuda").half()
    slots = np.array(slots, np.int64)
    kc, vc, kp, vp = _empty_int8(wl)
    binding.pa_reshape_and_cache_int8(keys, values, kc, vc, kp, vp, torch.from_numpy(slots).cuda())
    alias = _decode(wl, (kc, vc, kp, vp), tables=wl.alias_block_tables)
    pairs = torch.from_numpy(wl.copy_pairs).cuda()
    for cache in (kc, vc, kp, vp):
        binding.pa_copy_blocks_raw(cache, pairs)
    cow = _decode(wl, (kc, vc, kp, vp))
    assert torch.equal(alias.view(torch.int16), cow.view(torch.int16))
    rk, rv, rkp, rvp = oracle.reshape_and_cache_int8(
        keys.cpu().numpy(), values.cpu().numpy(), *(x.cpu().numpy() for x in _empty_int8(wl, "cpu")),
        slots, bs)
    for arr in (rk, rv, rkp, rvp):
        arr[wl.copy_pairs[:, 1]] = arr[wl.copy_pairs[:, 0]]
    for got, want in zip((kc, vc, kp, vp), (rk, rv, rkp, rvp)):
        assert np.array_equal(got.cpu().numpy().view(np.uint8), want.view(np.uint8))
    ref = oracle.paged_decode_int8(wl.q.cpu().numpy(), rk, rv, rkp, rvp, wl.block_tables,
                                   wl.context_lens, wl.scale)
    assert max_abs_err(cow, ref) <= ATOL


@pytest.mark.slow
def test_int8_llama13b_decode_config_full():
    wl = workloads.make_workload(2, device="cuda", keep_tokens=True)
    pool, (keys, values, slots) = _gpu_int8_pool(wl)
    ref_pool = _oracle_int8_pool(wl, keys, values, slots)
    for got, want in zip(pool, ref_pool):
        assert np.array_equal(got.cpu().numpy().view(np.uint8), np.asarray(want).view(np.uint8))
    out = _decode(wl, pool)
    ref = oracle.paged_decode_int8(wl.q.cpu().numpy(), *ref_pool, wl.block_tables,
                                   wl.context_lens, wl.scale)
    assert max_abs_err(out, ref) <= ATOL
    assert binding.pa_get_last_device_error() == 0


def _pool_without_newest(wl, skip_slots):
    """int8 pool holding every context token except those written to
    `skip_slots` (the rows the fused call appends)."""
    keys, values, slots = workloads.all_token_writes(wl)
    keep = torch.from_numpy(~np.isin(slots, skip_slots))
    kc, vc, kp, vp = _empty_int8(wl)
    binding.pa_reshape_and_cache_int8(keys[keep.to(keys.device)].cuda(),
                                      values[keep.to(values.device)].cuda(), kc, vc, kp, vp,
                                      torch.from_numpy(slots[keep.numpy()]).cuda())
    return (kc, vc, kp, vp), (keys, values, slots)


def _fused_int8(wl, pool, slots):
    kc, vc, kp, vp = pool
    q = wl.q.cuda()
    out = torch.empty_like(q)
    ws = binding.new_workspace(wl.num_seqs, wl.num_heads, wl.head_dim, wl.max_context_len)
    binding.pa_decode_append_int8(out, q, wl.new_key.cuda(), wl.new_value.cuda(), kc, vc, kp, vp,
                                  slots, torch.from_numpy(np.ascontiguousarray(wl.block_tables)).cuda(),
                                  torch.from_numpy(wl.context_lens).cuda(), wl.max_context_len,
                                  wl.scale, ws)
    torch.cuda.synchronize()
    return out


def _same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


@pytest.mark.parametrize("seed,d,bs,lens", CASES)
def test_int8_fused_append_equals_write_then_decode(seed, d, bs, lens):
    """pa_decode_append_int8 quantizes each sequence's newest row into its
    slot and decodes with it: the same cache bits and output bits as
    pa_reshape_and_cache_int8 of every token followed by pa_decode_int8, and
    the oracle's int8 write + decode within the tolerance."""
    wl = workloads.make_random(seed, lens, num_heads=5, head_dim=d, block_size=bs,
                               keep_logical=False, keep_tokens=True, pool_factor=2.0)
    pool, (keys, values, slots) = _pool_without_newest(wl, wl.slot_mapping)
    out = _fused_int8(wl, pool, torch.from_numpy(wl.slot_mapping).cuda())
    assert binding.pa_get_last_device_error() == 0
    full, _ = _gpu_int8_pool(wl)
    out2 = _decode(wl, full)
    assert _same_bits(out, out2)
    for got, want in zip(pool, full):
        assert _same_bits(got, want)
    ref_pool = _oracle_int8_pool(wl, keys, values, slots)
    ref = oracle.paged_decode_int8(wl.q.numpy(), *ref_pool, wl.block_tables, wl.context_lens,
                                   wl.scale)
    assert max_abs_err(out, ref) <= ATOL


def test_int8_fused_append_mixed_batch_and_bad_slot():
    """Half the sequences append nothing (slot -1; their newest row is in the
    cache already); then a slot that is not position L - 1's is reported."""
    wl = workloads.make_random(209, [40, 1, 95, 33, 64, 200], num_heads=3, head_dim=128,
                               block_size=16, keep_logical=False, keep_tokens=True, pool_factor=2.0)
    slots = wl.slot_mapping.copy()
    slots[::2] = -1
    pool, _ = _pool_without_newest(wl, wl.slot_mapping[1::2])
    out = _fused_int8(wl, pool, torch.from_numpy(slots).cuda())
    assert binding.pa_get_last_device_error() == 0
    full, _ = _gpu_int8_pool(wl)
    assert _same_bits(out, _decode(wl, full))
    for got, want in zip(pool, full):
        assert _same_bits(got, want)
    bad = wl.slot_mapping.copy()
    bad[2] -= 1                       # the slot of position L - 2
    _fused_int8(wl, pool, torch.from_numpy(bad).cuda())
    assert binding.pa_get_last_device_error() == binding.PA_DEVERR_SLOT


@pytest.mark.slow
def test_int8_fused_append_llama13b_full():
    wl = workloads.make_workload(2, device="cuda", keep_tokens=True)
    pool, (keys, values, slots) = _pool_without_newest(wl, wl.slot_mapping)
    out = _fused_int8(wl, pool, torch.from_numpy(wl.slot_mapping).cuda())
    assert binding.pa_get_last_device_error() == 0
    ref_pool = _oracle_int8_pool(wl, keys, values, slots)
    for got, want in zip(pool, ref_pool):
        assert np.array_equal(got.cpu().numpy().view(np.uint8), np.asarray(want).view(np.uint8))
    ref = oracle.paged_decode_int8(wl.q.cpu().numpy(), *ref_pool, wl.block_tables,
                                   wl.context_lens, wl.scale)
    assert max_abs_err(out, ref) <= ATOL
