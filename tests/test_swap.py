"""Swap-out / swap-in of sequence groups by the host block manager (C++ in
libpa) against a hand-worked example and the plain-Python oracle; the data
copy of the oracle against its definition.  polomodov.tech "vLLM and
PagedAttention", slide 15: preemption is all-or-nothing and a preempted
request comes back by swapping its blocks (or by recomputation)."""
import numpy as np
import pytest

import oracle
from oracle.block_manager import BlockManagerOracle, OutOfBlocks
from paged_kv_cache_481_b200 import binding, build


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    binding.load()


def _tables(bm, seqs, mb=8):
    t, lens = bm.block_tables(seqs, mb)
    return [row[row >= 0].tolist() for row in t], lens.tolist()


def test_swap_round_trip_worked_example():
    """Pools of 8 device and 8 host blocks, block size 4.
    Request 1 (6 tokens) takes device blocks 0, 1; its sample 2 shares them
    (counts 2); request 3 (5 tokens) takes 2, 3.  Swapping out the group
    {1, 2} maps device 0 -> host 0 and device 1 -> host 1 (counts 2 kept);
    device 0 then 1 go back on the stack, so request 4 (3 tokens) takes 1.
    Swapping the group back in takes device 0, then 4 (the stack is 7 6 5 4
    0 with 0 on top after block 1 left): pairs (0, 0) and (1, 4)."""
    bm = binding.BlockManager(8, 4, num_cpu_blocks=8)
    bm.add_sequence(1, 6)
    bm.fork(1, 2)
    bm.add_sequence(3, 5)
    out = bm.swap_out([1, 2])
    assert out.tolist() == [[0, 0], [1, 1]]
    assert bm.is_swapped(1) == 1 and bm.is_swapped(2) == 1 and bm.is_swapped(3) == 0
    assert bm.cpu_refcount(0) == 2 and bm.cpu_refcount(1) == 2
    assert bm.refcount(0) == 0 and bm.refcount(1) == 0
    assert bm.num_free() == 6 and bm.num_free_cpu() == 6
    bm.add_sequence(4, 3)
    assert _tables(bm, [4])[0] == [[1]]
    back = bm.swap_in([1, 2])
    assert back.tolist() == [[0, 0], [1, 4]]
    assert _tables(bm, [1, 2]) == ([[0, 4], [0, 4]], [6, 6])
    assert bm.refcount(0) == 2 and bm.refcount(4) == 2
    assert bm.num_free_cpu() == 8 and bm.cpu_refcount(0) == 0
    # the group keeps decoding where it stopped: position 6 of block 4 is
    # shared, so the first writer copies it
    slots, pairs = bm.append_slots([1])
    assert pairs.tolist() == [[4, 5]] and slots.tolist() == [5 * 4 + 2]


def test_partial_group_is_refused_and_nothing_changes():
    bm = binding.BlockManager(8, 4, num_cpu_blocks=8)
    bm.add_sequence(1, 6)
    bm.fork(1, 2)
    with pytest.raises(binding.PAError) as e:
        bm.swap_out([1])               # sample 2 still holds blocks 0 and 1
    assert e.value.status == binding.PA_ERR_INVALID_ARG
    assert bm.is_swapped(1) == 0 and bm.num_free_cpu() == 8 and bm.refcount(0) == 2


def test_short_pools_change_nothing():
    bm = binding.BlockManager(4, 4, num_cpu_blocks=1)
    bm.add_sequence(1, 8)              # blocks 0, 1
    with pytest.raises(binding.PAError) as e:
        bm.swap_out([1])               # 2 blocks, 1 host block
    assert e.value.status == binding.PA_ERR_OUT_OF_BLOCKS
    assert _tables(bm, [1]) == ([[0, 1]], [8]) and bm.num_free_cpu() == 1
    bm2 = binding.BlockManager(2, 4, num_cpu_blocks=4)
    bm2.add_sequence(1, 8)             # both device blocks
    bm2.swap_out([1])
    bm2.add_sequence(2, 5)             # device blocks taken again
    with pytest.raises(binding.PAError) as e:
        bm2.swap_in([1])
    assert e.value.status == binding.PA_ERR_OUT_OF_BLOCKS
    assert bm2.is_swapped(1) == 1 and bm2.num_free_cpu() == 2


def test_swapped_sequences_only_free():
    bm = binding.BlockManager(8, 4, num_cpu_blocks=8)
    bm.add_sequence(1, 5)
    bm.swap_out([1])
    for call in (lambda: bm.append_slots([1]), lambda: bm.fork(1, 9),
                 lambda: bm.block_tables([1], 4), lambda: bm.swap_out([1]),
                 lambda: bm.swap_in([7])):
        with pytest.raises(binding.PAError):
            call()
    bm.free_sequence(1)
    assert bm.num_free_cpu() == 8 and bm.num_free() == 8 and bm.is_swapped(1) == -1


def _groups(ref, swapped: bool):
    """Sharing groups (connected through common blocks) among resident or
    swapped sequences of the oracle, each sorted."""
    seqs = [s for s in ref.tables if (s in ref.swapped) == swapped]
    parent = {s: s for s in seqs}

    def find(x):
        while parent[x] != x:
            x = parent[x]
        return x
    owner = {}
    for s in seqs:
        for b in ref.tables[s]:
            if b in owner:
                parent[find(s)] = find(owner[b])
            else:
                owner[b] = s
    out = {}
    for s in seqs:
        out.setdefault(find(s), []).append(s)
    return [sorted(g) for g in out.values()]


@pytest.mark.parametrize("seed", range(5))
def test_random_operations_with_swaps_match_the_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    nb, ncpu, bs = int(rng.integers(16, 64)), int(rng.integers(8, 64)), int(rng.choice([4, 8]))
    bm = binding.BlockManager(nb, bs, num_cpu_blocks=ncpu)
    ref = BlockManagerOracle(nb, bs, num_cpu_blocks=ncpu)
    next_id = 0
    for _ in range(400):
        op = rng.choice(["add", "fork", "step", "free", "out", "in"],
                        p=[0.2, 0.1, 0.4, 0.1, 0.1, 0.1])
        resident = [s for s in ref.tables if s not in ref.swapped]
        if op == "add":
            n = int(rng.integers(0, 3 * bs))
            try:
                ref.add_sequence(next_id, n)
                bm.add_sequence(next_id, n)
            except OutOfBlocks:
                with pytest.raises(binding.PAError):
                    bm.add_sequence(next_id, n)
            next_id += 1
        elif op == "fork" and resident:
            parent = int(rng.choice(resident))
            ref.fork(parent, next_id)
            bm.fork(parent, next_id)
            next_id += 1
        elif op == "step" and resident:
            batch = [int(x) for x in rng.permutation(resident)[: int(rng.integers(1, len(resident) + 1))]]
            try:
                slots, pairs = ref.append_slots(batch)
            except OutOfBlocks:
                with pytest.raises(binding.PAError):
                    bm.append_slots(batch)
                continue
            s2, p2 = bm.append_slots(batch)
            assert s2.tolist() == slots and [tuple(x) for x in p2.tolist()] == pairs
        elif op == "free" and ref.tables:
            victim = int(rng.choice(list(ref.tables)))
            ref.free_sequence(victim)
            bm.free_sequence(victim)
        elif op in ("out", "in"):
            groups = _groups(ref, swapped=(op == "in"))
            if not groups:
                continue
            g = groups[int(rng.integers(len(groups)))]
            g = [int(x) for x in rng.permutation(g)]
            fn_ref = ref.swap_out if op == "out" else ref.swap_in
            fn_bm = bm.swap_out if op == "out" else bm.swap_in
            try:
                want = fn_ref(g)
            except OutOfBlocks:
                with pytest.raises(binding.PAError) as e:
                    fn_bm(g)
                assert e.value.status == binding.PA_ERR_OUT_OF_BLOCKS
                continue
            got = fn_bm(g)
            assert [tuple(x) for x in got.tolist()] == want
        # state: tables of resident sequences, both pools' counts and free sizes
        resident = [s for s in ref.tables if s not in ref.swapped]
        if resident:
            mb = max(1, max(len(ref.tables[s]) for s in resident))
            rows, lens = _tables(bm, resident, mb)
            assert rows == [ref.tables[s] for s in resident]
            assert lens == [ref.lens[s] for s in resident]
        for s in ref.tables:
            assert bm.is_swapped(s) == int(s in ref.swapped)
        for b in range(nb):
            assert bm.refcount(b) == ref.ref[b]
        for b in range(ncpu):
            assert bm.cpu_refcount(b) == ref.cpu_ref[b]
        assert bm.num_free() == len(ref.free) and bm.num_free_cpu() == len(ref.cpu_free)
        # invariants of the oracle itself: count = holders in each pool
        for pool_ref, held in ((ref.ref, [s for s in ref.tables if s not in ref.swapped]),
                               (ref.cpu_ref, list(ref.swapped))):
            counts = np.zeros(len(pool_ref), dtype=int)
            for s in held:
                for b in ref.tables[s]:
                    counts[b] += 1
            assert counts.tolist() == pool_ref


def test_oracle_swap_blocks_moves_whole_blocks_bytewise():
    rng = np.random.default_rng(3)
    src = rng.integers(0, 2 ** 16, size=(5, 2, 4, 8), dtype=np.uint16).view(np.float16)
    dst = np.zeros((3, 2, 4, 8), dtype=np.float16)
    out = oracle.swap_blocks(src, dst, [[4, 0], [1, 2]])
    assert out.view(np.uint16)[0].tolist() == src.view(np.uint16)[4].tolist()
    assert out.view(np.uint16)[2].tolist() == src.view(np.uint16)[1].tolist()
    assert not out[1].any() and not dst.any()   # untouched block; input not modified
    with pytest.raises(ValueError):
        oracle.swap_blocks(src, dst, [[5, 0]])


def test_oracle_manager_on_the_worked_example():
    """The oracle's swap decisions on the same hand-worked example."""
    ref = BlockManagerOracle(8, 4, num_cpu_blocks=8)
    ref.add_sequence(1, 6)
    ref.fork(1, 2)
    ref.add_sequence(3, 5)
    assert ref.swap_out([1, 2]) == [(0, 0), (1, 1)]
    assert ref.cpu_ref[:2] == [2, 2] and ref.ref[:2] == [0, 0]
    ref.add_sequence(4, 3)
    assert ref.tables[4] == [1]
    assert ref.swap_in([1, 2]) == [(0, 0), (1, 4)]
    assert ref.tables[1] == ref.tables[2] == [0, 4] and ref.lens[1] == 6
    with pytest.raises(KeyError):
        ref.swap_out([1])              # sample 2 still shares the blocks
    assert ref.append_slots([1]) == ([5 * 4 + 2], [(4, 5)])
