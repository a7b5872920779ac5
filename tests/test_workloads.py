"""Host-side checks of the seeded input generators (no GPU)."""
import math

import numpy as np
import pytest

from paged_kv_cache_481_b200 import accounting, workloads


@pytest.mark.parametrize("cfg", [1, 2, 3, 5])
def test_config_lengths_follow_their_recipe(cfg):
    lens = workloads.config_lengths(cfg, cfg)
    if cfg == 1:
        assert lens.tolist() == [1, 17, 33, 50]
    elif cfg == 2:
        assert len(lens) == 32 and lens.min() >= 256 and lens.max() <= 2048
    elif cfg == 3:
        assert len(lens) == 256 and lens.min() >= 1 and lens.max() <= 4096
        assert 300 < np.median(lens) < 800          # lognormal around a median of 512
    else:
        assert len(lens) == 128 and lens.min() >= 1024 and lens.max() <= 4096
    # seeded: the same draw twice
    assert np.array_equal(lens, workloads.config_lengths(cfg, cfg))


def test_append_rule_and_waste_bound():
    """A block is taken only when the previous one is full, so each sequence
    uses ceil(L / bs) blocks and wastes at most bs - 1 slots (polomodov.tech
    slide 11; brentwoodlivery.com 5.3.18 on the maximum waste per request)."""
    wl = workloads.make_workload(1)
    for bs in (8, 16, 32):
        for length, row in zip(wl.context_lens, workloads.make_workload(
                1, block_size=bs).block_tables):
            used = int((row >= 0).sum())
            assert used == math.ceil(length / bs)
            assert used * bs - length <= bs - 1


def test_tables_use_distinct_physical_blocks():
    wl = workloads.make_workload(3, num_seqs=40)
    ids = wl.block_tables[wl.block_tables >= 0]
    assert len(ids) == len(np.unique(ids))
    assert ids.max() < wl.num_blocks
    assert wl.num_blocks >= 1.5 * len(ids) - 1


def test_slots_point_at_the_newest_token():
    wl = workloads.make_workload(1)
    bs = wl.block_size
    for b, length in enumerate(wl.context_lens):
        pos = length - 1
        assert wl.slot_mapping[b] // bs == wl.block_tables[b, pos // bs]
        assert wl.slot_mapping[b] % bs == pos % bs


def test_pool_positions_without_tokens_hold_the_canary():
    wl = workloads.make_workload(1)
    bits = wl.k_cache.numpy().view(np.uint16)
    used = wl.block_tables[wl.block_tables >= 0]
    free = np.setdiff1d(np.arange(wl.num_blocks), used)
    assert (bits[free] == workloads.CANARY_BITS).all()
    # the newest token is not in the pool until the cache write runs
    for b, s in enumerate(wl.slot_mapping):
        assert (bits[s // wl.block_size, :, s % wl.block_size] == workloads.CANARY_BITS).all()


def test_same_values_for_every_block_size():
    a = workloads.make_random(3, [40, 9], 2, 64, 8)
    b = workloads.make_random(3, [40, 9], 2, 64, 32)
    for x, y in zip(a.logical_k, b.logical_k):
        assert np.array_equal(x.numpy(), y.numpy())


def test_shared_prefix_structure():
    wl = workloads.make_shared_prefix(num_groups=2, group_size=3, prefix_len=64,
                                      num_heads=2, head_dim=64)
    n_prefix = 64 // 16
    for s in range(wl.num_seqs):
        g = s // 3
        first = wl.alias_block_tables[g * 3, :n_prefix]
        assert np.array_equal(wl.alias_block_tables[s, :n_prefix], first)
        assert wl.copy_pairs[s, 0] == first[-1]
        assert wl.block_tables[s, n_prefix - 1] == wl.copy_pairs[s, 1]
    assert len(np.unique(wl.copy_pairs[:, 1])) == wl.num_seqs


def test_unique_bytes_count_shared_blocks_once():
    wl = workloads.make_shared_prefix(num_groups=2, group_size=4, prefix_len=64,
                                      num_heads=2, head_dim=64)
    logical = accounting.decode_bytes(wl.context_lens, 2, 64)
    unique = accounting.decode_unique_bytes(wl.alias_block_tables, wl.context_lens, 2, 64, 16)
    shared_rows = 2 * (4 - 1) * 64               # prefix rows read by the 3 other members
    assert logical - unique == shared_rows * accounting.kv_bytes_per_token(2, 64)


def test_sequential_placement_keeps_values_and_makes_blocks_consecutive():
    a = workloads.make_workload(1, keep_logical=True)
    b = workloads.make_workload(1, keep_logical=True, placement="sequential")
    for x, y in zip(a.logical_k, b.logical_k):
        assert np.array_equal(x.numpy(), y.numpy())
    ids = b.block_tables[b.block_tables >= 0]
    assert np.array_equal(ids, np.arange(len(ids)))
