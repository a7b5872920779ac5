"""Swapping a preempted request group out to pinned host memory and back
(polomodov.tech "vLLM and PagedAttention", slide 15), driven by the host
block manager: the device pool, the host pool and every decode output must
match the oracle path (oracle block manager + oracle copies + oracle decode)
bit for bit on the caches and within 2e-3 on the outputs."""
import numpy as np
import pytest
import torch

import oracle
from oracle.block_manager import BlockManagerOracle
from paged_kv_cache_481_b200 import binding, build

from gpu_helpers import ATOL, max_abs_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    binding.load()
    torch.cuda.init()


def _slots(row, positions, bs):
    return np.array([int(row[p // bs]) * bs + p % bs for p in positions], np.int64)


@pytest.mark.parametrize("seed,bs,d", [(0, 16, 128), (1, 8, 64)])
def test_preempt_swap_out_reuse_swap_in_and_decode(seed, bs, d):
    rng = np.random.default_rng(seed)
    gen = torch.Generator().manual_seed(seed)
    h, nb, ncpu = 4, 24, 16
    scale = 1.0 / np.sqrt(d)
    bm, ref = binding.BlockManager(nb, bs, num_cpu_blocks=ncpu), BlockManagerOracle(nb, bs, ncpu)
    shape = (nb, h, bs, d)
    kc, vc = (torch.randn(shape, generator=gen).half().cuda() for _ in range(2))
    okc, ovc = kc.cpu().numpy().copy(), vc.cpu().numpy().copy()
    hk = torch.zeros((ncpu, h, bs, d), dtype=torch.float16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    ohk, ohv = hk.numpy().copy(), hv.numpy().copy()

    def write(seq, positions):
        nonlocal okc, ovc
        tables, _ = bm.block_tables([seq], 16)
        slots = _slots(tables[0], positions, bs)
        k = torch.randn((len(slots), h, d), generator=gen).half()
        v = torch.randn((len(slots), h, d), generator=gen).half()
        binding.pa_reshape_and_cache(k.cuda(), v.cuda(), kc, vc, torch.from_numpy(slots).cuda())
        okc, ovc = oracle.reshape_and_cache(k.numpy(), v.numpy(), okc, ovc, slots, bs)

    def decode_and_check(seqs):
        tables, lens = bm.block_tables(seqs, 16)
        rt = [ref.tables[s] for s in seqs]
        assert [r[r >= 0].tolist() for r in tables] == rt
        q = torch.randn((len(seqs), h, d), generator=gen).half()
        out = torch.empty_like(q).cuda()
        ws = binding.new_workspace(len(seqs), h, d, int(lens.max()))
        binding.pa_decode(out, q.cuda(), kc, vc, torch.from_numpy(tables).cuda(),
                          torch.from_numpy(lens).cuda(), int(lens.max()), scale, ws)
        want = oracle.paged_decode(q.numpy(), okc, ovc, tables, lens, scale)
        assert max_abs_err(out, want) <= ATOL

    def same_pools():
        torch.cuda.synchronize()
        for dev, want in ((kc, okc), (vc, ovc)):
            assert np.array_equal(dev.cpu().numpy().view(np.uint16), want.view(np.uint16))
        for host, want in ((hk, ohk), (hv, ohv)):
            assert np.array_equal(host.numpy().view(np.uint16), want.view(np.uint16))

    lens0 = {0: int(rng.integers(bs, 4 * bs)), 1: int(rng.integers(1, 3 * bs)),
             2: int(rng.integers(bs, 3 * bs))}
    for s, n in lens0.items():
        bm.add_sequence(s, n)
        ref.add_sequence(s, n)
        write(s, range(n))
    bm.fork(2, 3)
    ref.fork(2, 3)
    decode_and_check([0, 1, 2, 3])

    # preempt the newest request group {2, 3}: device -> host
    pairs = bm.swap_out([2, 3])
    want_pairs = ref.swap_out([2, 3])
    assert [tuple(p) for p in pairs.tolist()] == want_pairs
    m = torch.from_numpy(pairs).cuda()
    binding.pa_swap_blocks(kc, hk, m)
    binding.pa_swap_blocks(vc, hv, m)
    ohk = oracle.swap_blocks(okc, ohk, want_pairs)
    ohv = oracle.swap_blocks(ovc, ohv, want_pairs)
    same_pools()

    # the freed device blocks are reused (and overwritten) by a new request
    bm.add_sequence(4, 3 * bs)
    ref.add_sequence(4, 3 * bs)
    write(4, range(3 * bs))
    decode_and_check([0, 1, 4])

    # bring the group back: host -> device (mapping read from pinned memory)
    pairs = bm.swap_in([3, 2])
    want_pairs = ref.swap_in([3, 2])
    assert [tuple(p) for p in pairs.tolist()] == want_pairs
    m_host = torch.from_numpy(pairs).pin_memory()
    binding.pa_swap_blocks(hk, kc, m_host)
    binding.pa_swap_blocks(hv, vc, m_host)
    okc = oracle.swap_blocks(ohk, okc, want_pairs)
    ovc = oracle.swap_blocks(ohv, ovc, want_pairs)
    same_pools()
    decode_and_check([0, 1, 2, 3, 4])

    # and keeps generating, with copy-on-write between the two samples
    for _ in range(3):
        seqs = [0, 2, 3, 4]
        slots, cow = bm.append_slots(seqs)
        oslots, ocow = ref.append_slots(seqs)
        assert slots.tolist() == oslots and [tuple(p) for p in cow.tolist()] == ocow
        if len(cow):
            binding.pa_copy_blocks(kc, vc, torch.from_numpy(cow).cuda())
            okc, ovc = oracle.copy_blocks(okc, ovc, np.array(ocow, np.int64))
        k = torch.randn((len(seqs), h, d), generator=gen).half()
        v = torch.randn((len(seqs), h, d), generator=gen).half()
        binding.pa_reshape_and_cache(k.cuda(), v.cuda(), kc, vc, torch.from_numpy(slots).cuda())
        okc, ovc = oracle.reshape_and_cache(k.numpy(), v.numpy(), okc, ovc, np.array(oslots), bs)
        decode_and_check(seqs)
    same_pools()
    assert binding.pa_get_last_device_error() == 0


def test_swap_rejects_same_pool_and_reports_bad_pairs():
    pool = torch.zeros((4, 2, 8, 64), dtype=torch.float16, device="cuda")
    host = torch.zeros((2, 2, 8, 64), dtype=torch.float16).pin_memory()
    m = torch.tensor([[0, 0]], dtype=torch.int64, device="cuda")
    with pytest.raises(binding.PAError) as e:
        binding.pa_swap_blocks(pool, pool, m)
    assert e.value.status == binding.PA_ERR_INVALID_ARG
    binding.pa_get_last_device_error()
    bad = torch.tensor([[3, 2]], dtype=torch.int64, device="cuda")   # host pool has 2 blocks
    binding.pa_swap_blocks(pool, host, bad)
    assert binding.pa_get_last_device_error() == binding.PA_DEVERR_COPY_PAIR
    assert not host.any()


def test_swap_refuses_pageable_host_memory():
    import ctypes
    pool = torch.zeros((4, 2, 8, 64), dtype=torch.float16, device="cuda")
    pageable = np.zeros((4, 2, 8, 64), dtype=np.float16)
    m = torch.tensor([[0, 0]], dtype=torch.int64, device="cuda")
    rc = binding.load().pa_swap_blocks(ctypes.c_void_p(pool.data_ptr()),
                                       ctypes.c_void_p(pageable.ctypes.data), pool[0].numel() * 2,
                                       ctypes.c_void_p(m.data_ptr()), 1, 4, 4, None)
    assert rc == binding.PA_ERR_INVALID_ARG
    torch.cuda.synchronize()
