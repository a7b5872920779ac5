"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle on
the same seeded inputs.  Cache write and block copy must be bit-exact;
attention outputs within max-abs 2e-3 (fp32 accumulation, fp16 output)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_481_b200 import binding, build, workloads

from gpu_helpers import (ATOL, gpu_decode, gpu_write_and_decode, max_abs_err,
                         oracle_write_and_decode, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    binding.load()
    torch.cuda.init()


@pytest.fixture(autouse=True)
def _clean_error_word():
    binding.pa_get_last_device_error()
    yield


def _bits(t):
    return t.cpu().numpy().view(np.uint16)


def _assert_no_device_error():
    assert binding.pa_get_last_device_error() == 0


# ------------------------------------------------------------ tiny config

def test_tiny_config_write_is_bit_exact_and_decode_matches():
    wl = workloads.make_workload(1)
    out, kc, vc = gpu_write_and_decode(wl)
    ref, okc, ovc = oracle_write_and_decode(wl)
    assert np.array_equal(_bits(kc), okc.view(np.uint16))
    assert np.array_equal(_bits(vc), ovc.view(np.uint16))
    assert max_abs_err(out, ref) <= ATOL
    # context length 1: the weight is exactly 1, so out is V_0 bit for bit
    assert np.array_equal(_bits(out[0]), wl.new_value[0].numpy().view(np.uint16))
    _assert_no_device_error()


@pytest.mark.parametrize("seed", [11, 21])
def test_tiny_config_second_draws(seed):
    wl = workloads.make_workload(1, seed=seed)
    out, _, _ = gpu_write_and_decode(wl)
    ref, _, _ = oracle_write_and_decode(wl)
    assert max_abs_err(out, ref) <= ATOL


# ------------------------------------------- shapes, block sizes, partitions

CASES = [
    # (seed, head_dim, block_size, lengths): ragged tails, lengths on and next to
    # tile / block / partition boundaries, several partitions
    (101, 128, 16, [1, 2, 15, 16, 17, 511, 512, 513, 1024, 1500]),
    (102, 128, 8, [7, 8, 9, 300, 777, 1025]),
    (103, 128, 32, [31, 33, 64, 1030, 2047]),
    (104, 128, 64, [63, 65, 128, 900, 1600]),
    (105, 128, 128, [1, 127, 129, 513, 2100]),
    (106, 64, 16, [1, 17, 33, 50, 640, 1111]),
    (107, 64, 8, [3, 31, 32, 33, 520]),
    (108, 64, 32, [32, 64, 97, 1300]),
    (109, 64, 64, [5, 700]),
    (110, 64, 128, [129, 1030]),
]


@pytest.mark.parametrize("seed,d,bs,lens", CASES)
def test_random_shapes_match_oracle(seed, d, bs, lens):
    wl = workloads.make_random(seed, lens, num_heads=5, head_dim=d, block_size=bs,
                               keep_logical=False)
    out, kc, vc = gpu_write_and_decode(wl)
    ref, okc, ovc = oracle_write_and_decode(wl)
    assert np.array_equal(_bits(kc), okc.view(np.uint16))
    assert max_abs_err(out, ref) <= ATOL
    _assert_no_device_error()


def test_long_contexts_many_partitions():
    lens = [4096, 4095, 3000, 8192, 6000]
    wl = workloads.make_random(120, lens, num_heads=4, head_dim=128, block_size=16,
                               keep_logical=False)
    out, _, _ = gpu_write_and_decode(wl)
    ref, _, _ = oracle_write_and_decode(wl)
    assert max_abs_err(out, ref) <= ATOL


def test_host_bound_above_actual_lengths():
    wl = workloads.make_random(121, [40, 600], num_heads=3, head_dim=128, block_size=16,
                               pool_factor=2.0, keep_logical=False)
    # widen the tables so a larger host-side bound is legal
    tables = np.full((2, 200), -1, np.int32)
    tables[:, :wl.block_tables.shape[1]] = wl.block_tables
    wl.block_tables = tables
    out, _, _ = gpu_write_and_decode(wl, max_context_len=3000)
    ref, _, _ = oracle_write_and_decode(wl)
    assert max_abs_err(out, ref) <= ATOL
    _assert_no_device_error()


def test_zero_length_context_writes_zeros():
    wl = workloads.make_random(122, [30, 5], num_heads=2, head_dim=64, block_size=16,
                               keep_logical=False)
    t = to_dev(wl)
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slots"])
    t["lens"] = torch.tensor([0, 5], dtype=torch.int32, device="cuda")
    out = gpu_decode(wl, t, max_context_len=30)
    assert torch.count_nonzero(out[0]) == 0
    lens = np.array([0, 5], np.int32)
    kc, vc = oracle.reshape_and_cache(wl.new_key.numpy(), wl.new_value.numpy(),
                                      wl.k_cache.numpy(), wl.v_cache.numpy(), wl.slot_mapping, 16)
    ref = oracle.paged_decode(wl.q.numpy(), kc, vc, wl.block_tables, lens, wl.scale)
    assert max_abs_err(out, ref) <= ATOL


def test_results_are_deterministic_and_workspace_is_reusable():
    wl = workloads.make_random(123, [100, 1800, 2500, 7], num_heads=8, head_dim=128,
                               block_size=16, keep_logical=False)
    t = to_dev(wl)
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slots"])
    ws = binding.new_workspace(wl.num_seqs, wl.num_heads, wl.head_dim, 8192)
    first = gpu_decode(wl, t, workspace=ws)
    for _ in range(5):
        again = gpu_decode(wl, t, workspace=ws)
        assert torch.equal(first.view(torch.int16), again.view(torch.int16))
    # a smaller problem on the same (larger) workspace
    small = workloads.make_random(124, [600, 1200], num_heads=3, head_dim=128, block_size=16,
                                  keep_logical=False)
    ts = to_dev(small)
    out, _, _ = gpu_write_and_decode(small, ts)
    out2 = gpu_decode(small, ts, workspace=ws)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_non_default_stream():
    wl = workloads.make_random(125, [900, 33], num_heads=4, head_dim=128, block_size=16,
                               keep_logical=False)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        t = to_dev(wl)
        out, _, _ = gpu_write_and_decode(wl, t, stream=s)
    s.synchronize()
    ref, _, _ = oracle_write_and_decode(wl)
    assert max_abs_err(out, ref) <= ATOL


# --------------------------------------------------- cache write edge cases

def test_negative_slots_are_skipped():
    wl = workloads.make_workload(1)
    wl.slot_mapping = wl.slot_mapping.copy()
    wl.slot_mapping[2] = -1
    t = to_dev(wl)
    before = _bits(t["k_cache"]).copy()
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slots"])
    kc, vc = oracle.reshape_and_cache(wl.new_key.numpy(), wl.new_value.numpy(),
                                      wl.k_cache.numpy(), wl.v_cache.numpy(), wl.slot_mapping, 16)
    assert np.array_equal(_bits(t["k_cache"]), kc.view(np.uint16))
    assert np.array_equal(_bits(t["v_cache"]), vc.view(np.uint16))
    changed = np.any(_bits(t["k_cache"]) != before, axis=-1).sum()
    assert changed == (wl.num_seqs - 1) * wl.num_heads
    _assert_no_device_error()


def test_padding_tokens_mixed_in_a_write_batch():
    wl = workloads.make_workload(3, num_seqs=24)
    n = wl.num_seqs
    # interleave padding tokens (slot -1) with the real ones
    key = torch.cat([wl.new_key, torch.randn_like(wl.new_key.float()).half()])
    value = torch.cat([wl.new_value, torch.randn_like(wl.new_value.float()).half()])
    slots = np.concatenate([wl.slot_mapping, -np.ones(n, np.int64)])
    perm = np.random.default_rng(0).permutation(2 * n)
    key, value, slots = key[perm], value[perm], slots[perm]
    kc_d, vc_d = wl.k_cache.cuda(), wl.v_cache.cuda()
    binding.pa_reshape_and_cache(key.cuda(), value.cuda(), kc_d, vc_d,
                                 torch.from_numpy(slots).cuda())
    kc, vc = oracle.reshape_and_cache(key.numpy(), value.numpy(), wl.k_cache.numpy(),
                                      wl.v_cache.numpy(), slots, wl.block_size)
    assert np.array_equal(_bits(kc_d), kc.view(np.uint16))
    assert np.array_equal(_bits(vc_d), vc.view(np.uint16))


def test_out_of_range_slot_is_reported_not_written():
    wl = workloads.make_workload(1)
    wl.slot_mapping = wl.slot_mapping.copy()
    wl.slot_mapping[1] = wl.num_blocks * wl.block_size + 5
    t = to_dev(wl)
    before_k = _bits(t["k_cache"]).copy()
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slots"])
    err = binding.pa_get_last_device_error()
    assert err & binding.PA_DEVERR_SLOT
    changed = np.any(_bits(t["k_cache"]) != before_k, axis=-1).sum()
    assert changed == (wl.num_seqs - 1) * wl.num_heads


def test_out_of_range_block_id_is_reported_and_skipped():
    wl = workloads.make_random(126, [40, 700], num_heads=2, head_dim=128, block_size=16,
                               keep_logical=False)
    t = to_dev(wl)
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slots"])
    bad = wl.block_tables.copy()
    bad[1, 3] = wl.num_blocks + 100
    bad[1, 5] = -7
    out = gpu_decode(wl, t, tables=torch.from_numpy(bad).cuda())
    err = binding.pa_get_last_device_error()
    assert err & binding.PA_DEVERR_BLOCK_ID
    ref = oracle.paged_decode(wl.q.numpy()[:1], *oracle.reshape_and_cache(
        wl.new_key.numpy(), wl.new_value.numpy(), wl.k_cache.numpy(), wl.v_cache.numpy(),
        wl.slot_mapping, 16), wl.block_tables[:1], wl.context_lens[:1], wl.scale)
    assert max_abs_err(out[:1], ref) <= ATOL      # the healthy sequence is unaffected


def test_context_len_above_host_bound_is_reported():
    wl = workloads.make_random(127, [50, 60], num_heads=2, head_dim=64, block_size=16,
                               keep_logical=False)
    t = to_dev(wl)
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slots"])
    gpu_decode(wl, t, max_context_len=55)
    assert binding.pa_get_last_device_error() & binding.PA_DEVERR_CONTEXT_LEN


# ----------------------------------------------------------- copy-on-write

def test_copy_blocks_bit_exact_every_block_size():
    for bs in (8, 16, 32, 64, 128):
        wl = workloads.make_random(130 + bs, [300, 500, 90], num_heads=6, head_dim=128,
                                   block_size=bs, pool_factor=3.0, keep_logical=False)
        used = wl.block_tables[wl.block_tables >= 0]
        free = np.setdiff1d(np.arange(wl.num_blocks), used)
        pairs = np.stack([used[:len(free)][:7], free[:7]], axis=1).astype(np.int64)
        kc_d, vc_d = wl.k_cache.cuda(), wl.v_cache.cuda()
        binding.pa_copy_blocks(kc_d, vc_d, torch.from_numpy(pairs).cuda())
        kc, vc = oracle.copy_blocks(wl.k_cache.numpy(), wl.v_cache.numpy(), pairs)
        assert np.array_equal(_bits(kc_d), kc.view(np.uint16))
        assert np.array_equal(_bits(vc_d), vc.view(np.uint16))
    _assert_no_device_error()


def test_bad_copy_pair_is_reported_and_skipped():
    wl = workloads.make_workload(1)
    kc_d, vc_d = wl.k_cache.cuda(), wl.v_cache.cuda()
    pairs = torch.tensor([[0, wl.num_blocks + 3], [1, 2]], dtype=torch.int64, device="cuda")
    binding.pa_copy_blocks(kc_d, vc_d, pairs)
    assert binding.pa_get_last_device_error() & binding.PA_DEVERR_COPY_PAIR
    kc, _ = oracle.copy_blocks(wl.k_cache.numpy(), wl.v_cache.numpy(), [[1, 2]])
    assert np.array_equal(_bits(kc_d), kc.view(np.uint16))


def test_shared_prefix_config_aliased_equals_copied():
    """Config 4: 8 groups x 8 sequences share a 1024-token prefix; the CoW copy
    of the prefix's last block must be bit-exact and decoding through the copy
    must give bit-identical outputs to decoding through the shared block."""
    wl = workloads.make_workload(4, device="cuda")
    t = to_dev(wl)
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slots"])
    alias_tables = torch.from_numpy(wl.alias_block_tables).cuda()
    out_alias = gpu_decode(wl, t, tables=alias_tables)
    binding.pa_copy_blocks(t["k_cache"], t["v_cache"], torch.from_numpy(wl.copy_pairs).cuda())
    out_cow = gpu_decode(wl, t)
    assert torch.equal(out_alias.view(torch.int16), out_cow.view(torch.int16))
    # oracle: the same write, then the copy, then decode through the copies
    okc, ovc = oracle.reshape_and_cache(wl.new_key.cpu().numpy(), wl.new_value.cpu().numpy(),
                                        wl.k_cache.cpu().numpy(), wl.v_cache.cpu().numpy(),
                                        wl.slot_mapping, wl.block_size)
    okc, ovc = oracle.copy_blocks(okc, ovc, wl.copy_pairs)
    assert np.array_equal(_bits(t["k_cache"]), okc.view(np.uint16))
    assert np.array_equal(_bits(t["v_cache"]), ovc.view(np.uint16))
    ref = oracle.paged_decode(wl.q.cpu().numpy(), okc, ovc, wl.block_tables, wl.context_lens,
                              wl.scale)
    err = max_abs_err(out_cow, ref)
    assert err <= ATOL, f"max-abs {err:.3e}"
    _assert_no_device_error()


# --------------------------------------------------------- full-size configs

@pytest.mark.slow
def test_llama13b_decode_config_full():
    wl = workloads.make_workload(2, device="cuda")
    out, kc, vc = gpu_write_and_decode(wl)
    ref, okc, ovc = oracle_write_and_decode(wl)
    assert np.array_equal(_bits(kc), okc.view(np.uint16))
    err = max_abs_err(out, ref)
    assert err <= ATOL, f"max-abs {err:.3e}"
    _assert_no_device_error()


@pytest.mark.slow
def test_serving_batch_config_full():
    wl = workloads.make_workload(3, device="cuda")
    out, kc, vc = gpu_write_and_decode(wl)
    ref, okc, ovc = oracle_write_and_decode(wl)
    assert np.array_equal(_bits(kc), okc.view(np.uint16))
    assert np.array_equal(_bits(vc), ovc.view(np.uint16))
    err = max_abs_err(out, ref)
    assert err <= ATOL, f"max-abs {err:.3e}"
    _assert_no_device_error()


def _sampled_oracle(wl, seqs):
    """Oracle on the blocks the sampled sequences reference, extracted from the
    (pre-write) pool and renumbered; the GPU ran on the full pool."""
    tables = wl.block_tables[seqs]
    ids = np.unique(tables[tables >= 0])
    remap = np.full(wl.num_blocks, -1, np.int64)
    remap[ids] = np.arange(len(ids))
    sub_tables = np.where(tables >= 0, remap[np.maximum(tables, 0)], -1).astype(np.int32)
    idx = torch.from_numpy(ids).to(wl.k_cache.device)
    kc = wl.k_cache.index_select(0, idx).cpu().numpy()
    vc = wl.v_cache.index_select(0, idx).cpu().numpy()
    bs = wl.block_size
    slots = wl.slot_mapping[seqs]
    sub_slots = remap[slots // bs] * bs + slots % bs
    kc, vc = oracle.reshape_and_cache(wl.new_key[seqs].cpu().numpy(),
                                      wl.new_value[seqs].cpu().numpy(), kc, vc, sub_slots, bs)
    return oracle.paged_decode(wl.q[seqs].cpu().numpy(), kc, vc, sub_tables,
                               wl.context_lens[seqs], wl.scale)


@pytest.mark.slow
@pytest.mark.parametrize("bs", [8, 16, 32, 64, 128])
def test_opt66b_heads_block_size_sweep_sampled(bs):
    wl = workloads.make_workload(5, device="cuda", block_size=bs)
    out, _, _ = gpu_write_and_decode(wl)
    rng = np.random.default_rng(bs)
    seqs = np.unique(np.concatenate([rng.choice(wl.num_seqs, 6, replace=False),
                                     [int(np.argmax(wl.context_lens)),
                                      int(np.argmin(wl.context_lens))]]))
    ref = _sampled_oracle(wl, seqs)
    err = max_abs_err(out[torch.from_numpy(seqs).cuda()], ref)
    assert err <= ATOL, f"max-abs {err:.3e}"
    _assert_no_device_error()


# ------------------------------------------------------ failure detection

def test_bounded_wait_gives_up_and_the_context_stays_usable():
    """A wait that nothing completes ends after its limit with
    PA_DEVERR_TIMEOUT in the error word; the next decode still matches."""
    import time
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    binding.pa_selftest_bounded_wait(20000)           # 20 ms
    assert binding.pa_get_last_device_error() == binding.PA_DEVERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 0.015 < elapsed < 5.0
    assert binding.pa_get_last_device_error() == 0     # read clears it
    wl = workloads.make_random(140, [300, 20], num_heads=2, head_dim=128, block_size=16,
                               keep_logical=False)
    out, _, _ = gpu_write_and_decode(wl)
    ref, _, _ = oracle_write_and_decode(wl)
    assert max_abs_err(out, ref) <= ATOL
    _assert_no_device_error()
