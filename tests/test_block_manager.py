"""Host block manager (C++ in libpa) against the pages' examples and the
plain-Python oracle of oracle/block_manager.py; runs on CPU."""
import json
import os

import numpy as np
import pytest

from oracle.block_manager import BlockManagerOracle, OutOfBlocks
from paged_kv_cache_481_b200 import binding, build

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    binding.load()


def _invariants(bm, oracle_like_tables, num_blocks):
    """Reference count of each block = number of tables holding it; the free
    pool holds exactly the blocks nobody references."""
    counts = np.zeros(num_blocks, dtype=int)
    for t in oracle_like_tables.values():
        for b in t:
            counts[b] += 1
    for b in range(num_blocks):
        assert bm.refcount(b) == counts[b]
    assert bm.num_free() == int((counts == 0).sum())


def test_copy_on_write_example_of_parallel_sampling():
    """comfyai.app 6.4.3: A1 and A2 share physical blocks 0 and 1 after the
    prompt; when A1's new token diverges, A1's logical block 1 moves to a new
    physical block 3 (count 1) and A2 keeps block 1 (count back to 1)."""
    ex = json.load(open(os.path.join(GOLDEN, "block_tables.json")))["cow_parallel_sampling"]
    bm = binding.BlockManager(num_blocks=8, block_size=4)
    bm.add_sequence(1, 7)              # A1: 7 prompt tokens -> blocks 0, 1 (1 has a free slot)
    bm.fork(1, 2)                      # A2 shares both blocks
    tables, _ = bm.block_tables([1, 2], 4)
    assert tables[0, :2].tolist() == ex["shared_before"]["A1"]
    assert tables[1, :2].tolist() == ex["shared_before"]["A2"]
    assert bm.refcount(0) == 2 and bm.refcount(1) == 2
    bm.add_sequence(3, 2)              # another request takes block 2
    slots, pairs = bm.append_slots([1])
    assert pairs.tolist() == [[ex["copy"]["src"], ex["copy"]["dst"]]]
    tables, lens = bm.block_tables([1, 2], 4)
    assert tables[0, :2].tolist() == ex["after"]["A1"]
    assert tables[1, :2].tolist() == ex["after"]["A2"]
    for blk, count in ex["refcount_after"].items():
        assert bm.refcount(int(blk)) == count
    assert slots.tolist() == [3 * 4 + 3]   # position 7 -> block 3, offset 3
    assert lens.tolist() == [8, 7]


def test_new_block_only_when_the_last_is_full():
    """polomodov.tech slide 11: after the prompt, the first decode step
    writes into the free slot, the step after that takes a new block."""
    bm = binding.BlockManager(num_blocks=8, block_size=4)
    bm.add_sequence(7, 7)                       # blocks 0, 1; slot 7 free
    free = bm.num_free()
    s1, p1 = bm.append_slots([7])
    assert s1.tolist() == [1 * 4 + 3] and len(p1) == 0 and bm.num_free() == free
    s2, p2 = bm.append_slots([7])
    assert s2.tolist() == [2 * 4 + 0] and len(p2) == 0 and bm.num_free() == free - 1


def test_both_sharers_writing_in_one_step():
    bm = binding.BlockManager(num_blocks=8, block_size=4)
    bm.add_sequence(1, 5)
    bm.fork(1, 2)
    slots, pairs = bm.append_slots([1, 2])
    # the first writer copies; the second is then the block's only owner
    assert pairs.tolist() == [[1, 2]]
    assert slots.tolist() == [2 * 4 + 1, 1 * 4 + 1]
    assert bm.refcount(1) == 1 and bm.refcount(2) == 1


def test_out_of_blocks_changes_nothing():
    bm = binding.BlockManager(num_blocks=3, block_size=4)
    bm.add_sequence(1, 4)        # block 0 full
    bm.add_sequence(2, 8)        # blocks 1, 2 full
    before = bm.block_tables([1, 2], 3)
    with pytest.raises(binding.PAError) as e:
        bm.append_slots([1, 2])  # both need a fresh block, none left
    assert e.value.status == binding.PA_ERR_OUT_OF_BLOCKS
    after = bm.block_tables([1, 2], 3)
    assert all(np.array_equal(x, y) for x, y in zip(before, after))
    with pytest.raises(binding.PAError):
        bm.add_sequence(3, 1)


def test_errors_for_unknown_or_repeated_sequences():
    bm = binding.BlockManager(num_blocks=4, block_size=4)
    bm.add_sequence(1, 1)
    for call in (lambda: bm.add_sequence(1, 1), lambda: bm.fork(9, 10),
                 lambda: bm.fork(1, 1), lambda: bm.free_sequence(9),
                 lambda: bm.append_slots([1, 1]), lambda: bm.append_slots([5]),
                 lambda: bm.block_tables([1], 0)):
        with pytest.raises(binding.PAError):
            call()


def test_free_returns_blocks_when_the_last_sharer_leaves():
    bm = binding.BlockManager(num_blocks=8, block_size=4)
    bm.add_sequence(1, 9)        # blocks 0, 1, 2
    bm.fork(1, 2)
    bm.free_sequence(1)
    assert bm.num_free() == 5 and bm.refcount(0) == 1
    bm.free_sequence(2)
    assert bm.num_free() == 8
    bm.add_sequence(3, 1)        # the most recently freed block (2, freed last) comes back first
    tables, _ = bm.block_tables([3], 1)
    assert tables[0, 0] == 2


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_match_the_oracle(seed):
    rng = np.random.default_rng(seed)
    nb, bs = int(rng.integers(16, 96)), int(rng.choice([4, 8, 16]))
    bm = binding.BlockManager(nb, bs)
    ref = BlockManagerOracle(nb, bs)
    next_id = 0
    for _ in range(400):
        op = rng.choice(["add", "fork", "step", "free"], p=[0.2, 0.15, 0.5, 0.15])
        live = list(ref.tables)
        if op == "add":
            n = int(rng.integers(0, 3 * bs))
            try:
                ref.add_sequence(next_id, n)
                bm.add_sequence(next_id, n)
            except OutOfBlocks:
                with pytest.raises(binding.PAError):
                    bm.add_sequence(next_id, n)
            next_id += 1
        elif op == "fork" and live:
            parent = int(rng.choice(live))
            ref.fork(parent, next_id)
            bm.fork(parent, next_id)
            next_id += 1
        elif op == "step" and live:
            batch = [int(x) for x in rng.permutation(live)[: int(rng.integers(1, len(live) + 1))]]
            try:
                slots, pairs = ref.append_slots(batch)
            except OutOfBlocks:
                with pytest.raises(binding.PAError):
                    bm.append_slots(batch)
                continue
            s2, p2 = bm.append_slots(batch)
            assert s2.tolist() == slots
            assert [tuple(x) for x in p2.tolist()] == pairs
        elif op == "free" and live:
            victim = int(rng.choice(live))
            ref.free_sequence(victim)
            bm.free_sequence(victim)
        live = list(ref.tables)
        if live:
            mb = max(1, max(len(t) for t in ref.tables.values()))
            tables, lens = bm.block_tables(live, mb)
            for row, (seq, length) in zip(tables, zip(live, lens)):
                want = ref.tables[seq]
                assert row[: len(want)].tolist() == want and (row[len(want):] == -1).all()
                assert length == ref.lens[seq]
                # each table holds ceil(len / bs) blocks: at most bs - 1 slots wasted
                assert len(want) == -(-int(length) // bs)
        _invariants(bm, ref.tables, nb)
