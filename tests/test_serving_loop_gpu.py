"""Several decode iterations driven by the host block manager, the way a
serving engine uses the path (comfyai.app 6.4.2-6.4.3; polomodov.tech slides
11-13): prompts are written into freshly allocated blocks, some sequences are
forked for parallel sampling (shared blocks), and every step reserves one
slot per sequence, copies shared last blocks before writing (copy-on-write),
writes the new K/V and decodes.  The CUDA path (libpa block manager +
kernels) and the oracle path (oracle block manager + oracle kernels) must make
the same decisions and agree on every output."""
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


def _slots_for(tables_row, positions, bs):
    return np.array([int(tables_row[p // bs]) * bs + p % bs for p in positions], np.int64)


@pytest.mark.parametrize("seed,bs,d", [(0, 16, 128), (1, 8, 64), (2, 32, 128)])
def test_decode_iterations_with_forks_and_copy_on_write(seed, bs, d):
    rng = np.random.default_rng(seed)
    gen = torch.Generator().manual_seed(seed)
    h, nb, steps = 4, 96, 6
    scale = 1.0 / np.sqrt(d)
    bm, ref = binding.BlockManager(nb, bs), BlockManagerOracle(nb, bs)
    kc = torch.zeros((nb, h, bs, d), dtype=torch.float16)
    vc = torch.zeros_like(kc)
    kc_dev, vc_dev = kc.cuda(), vc.cuda()
    okc, ovc = kc.numpy().copy(), vc.numpy().copy()
    ws = binding.new_workspace(16, h, d, 4096)

    # prompts
    prompts = {0: int(rng.integers(1, 3 * bs)), 1: int(rng.integers(1, 3 * bs)),
               2: int(rng.integers(1, 3 * bs))}
    for seq, n in prompts.items():
        bm.add_sequence(seq, n)
        ref.add_sequence(seq, n)
        table, _ = bm.block_tables([seq], 8)
        slots = _slots_for(table[0], range(n), bs)
        k = torch.randn((n, h, d), generator=gen).half()
        v = torch.randn((n, h, d), generator=gen).half()
        binding.pa_reshape_and_cache(k.cuda(), v.cuda(), kc_dev, vc_dev,
                                     torch.from_numpy(slots).cuda())
        okc, ovc = oracle.reshape_and_cache(k.numpy(), v.numpy(), okc, ovc, slots, bs)
    # parallel sampling: two samples of sequence 0, one of sequence 2
    for parent, child in ((0, 10), (0, 11), (2, 12)):
        bm.fork(parent, child)
        ref.fork(parent, child)

    copies = 0
    for step in range(steps):
        seqs = sorted(ref.tables)
        slots, pairs = bm.append_slots(seqs)
        oslots, opairs = ref.append_slots(seqs)
        assert slots.tolist() == oslots and [tuple(p) for p in pairs.tolist()] == opairs
        copies += len(opairs)
        if len(pairs):
            binding.pa_copy_blocks(kc_dev, vc_dev, torch.from_numpy(pairs).cuda())
            okc, ovc = oracle.copy_blocks(okc, ovc, np.array(opairs, np.int64))
        n = len(seqs)
        k = torch.randn((n, h, d), generator=gen).half()
        v = torch.randn((n, h, d), generator=gen).half()
        q = torch.randn((n, h, d), generator=gen).half()
        binding.pa_reshape_and_cache(k.cuda(), v.cuda(), kc_dev, vc_dev,
                                     torch.from_numpy(slots).cuda())
        okc, ovc = oracle.reshape_and_cache(k.numpy(), v.numpy(), okc, ovc, np.array(oslots), bs)
        mb = max(len(t) for t in ref.tables.values())
        tables, lens = bm.block_tables(seqs, mb)
        out = torch.empty_like(q).cuda()
        binding.pa_decode(out, q.cuda(), kc_dev, vc_dev, torch.from_numpy(tables).cuda(),
                          torch.from_numpy(lens).cuda(), int(lens.max()), scale, ws)
        want = oracle.paged_decode(q.numpy(), okc, ovc, tables, lens, scale)
        assert max_abs_err(out, want) <= ATOL, f"step {step}"
        # the caches themselves stay bit-identical
        assert np.array_equal(kc_dev.cpu().numpy().view(np.uint16), okc.view(np.uint16))
        assert np.array_equal(vc_dev.cpu().numpy().view(np.uint16), ovc.view(np.uint16))
        if step == 2:  # a sample finishes; its blocks go back to the pool
            bm.free_sequence(11)
            ref.free_sequence(11)
    assert copies >= 1   # the forks did trigger copy-on-write
    assert binding.pa_get_last_device_error() == 0
