"""GPU parity of the tensor-core multi-query (prefill / chunked prefill)
paged attention against the fp64 oracle: every new token's output within
max-abs 2e-3 (fp32 accumulation; the attention weights enter P.V as fp16)."""
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


def _run(seed, lens, n_new, bs, h=4, d=128, growth=0.0):
    wl = workloads.make_random(seed, lens, num_heads=h, head_dim=d, block_size=bs,
                               keep_logical=False, pool_factor=2.0)
    if growth:  # later keys larger: the running max grows from tile to tile
        for b, length in enumerate(wl.context_lens):
            for t in range(int(length) - 1):
                blk, row = int(wl.block_tables[b, t // bs]), t % bs
                wl.k_cache[blk, :, row, :] *= 1.0 + growth * t / length
    kc, vc = wl.k_cache.cuda(), wl.v_cache.cuda()
    binding.pa_reshape_and_cache(wl.new_key.cuda(), wl.new_value.cuda(), kc, vc,
                                 torch.from_numpy(wl.slot_mapping).cuda())
    qsl = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    g = torch.Generator().manual_seed(seed + 7)
    q = torch.randn((int(qsl[-1]), h, d), generator=g).half()
    out = torch.full((int(qsl[-1]), h, d), float("nan"), dtype=torch.float16, device="cuda")
    binding.pa_prefill(out, q.cuda(), kc, vc, torch.from_numpy(wl.block_tables).cuda(),
                       torch.from_numpy(wl.context_lens).cuda(), wl.max_context_len,
                       torch.from_numpy(qsl).cuda(), max(n_new), wl.scale)
    torch.cuda.synchronize()
    okc, ovc = oracle.reshape_and_cache(wl.new_key.numpy(), wl.new_value.numpy(), wl.k_cache.numpy(),
                                        wl.v_cache.numpy(), wl.slot_mapping, bs)
    ref = oracle.paged_prefill(q.numpy(), okc, ovc, wl.block_tables, wl.context_lens, qsl, wl.scale)
    return out, ref


@pytest.mark.parametrize("seed,bs,lens,n_new", [
    (301, 16, [5, 130], [5, 130]),                      # whole prompts, one and two tiles
    (302, 16, [300, 257, 40], [300, 1, 17]),             # mixed: prompt, decode-like, chunk
    (303, 8, [200, 129], [64, 129]),
    (304, 32, [400, 128], [150, 128]),
    (305, 64, [513, 70], [256, 3]),
    (306, 128, [384, 260], [384, 100]),
    (307, 16, [50, 1, 64, 9], [0, 1, 64, 0]),             # sequences with no new tokens
    (308, 8, [700, 129, 256], [3, 128, 255]),            # chunks ending mid-block, bs 8
    (309, 128, [1000, 385], [600, 257]),                  # several items, 128-token blocks
])
def test_prefill_matches_oracle(seed, bs, lens, n_new):
    out, ref = _run(seed, lens, n_new, bs)
    assert not torch.isnan(out).any()
    assert max_abs_err(out, ref) <= ATOL
    assert binding.pa_get_last_device_error() == 0


def test_prefill_long_prompt_many_tiles():
    out, ref = _run(310, [1100, 700], [1100, 333], 16)
    assert max_abs_err(out, ref) <= ATOL


def test_prefill_rejects_other_head_dims():
    with pytest.raises(binding.PAError) as e:
        z = torch.zeros((1, 1, 64), dtype=torch.float16, device="cuda")
        c = torch.zeros((1, 1, 16, 64), dtype=torch.float16, device="cuda")
        i = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
        binding.pa_prefill(z, z, c, c, i, torch.ones(1, dtype=torch.int32, device="cuda"), 1,
                           torch.tensor([0, 1], dtype=torch.int32, device="cuda"), 1, 1.0)
    assert e.value.status == binding.PA_ERR_UNSUPPORTED


def test_prefill_running_max_grows_across_tiles():
    """Scores grow with the key position, so the row max rises by more than
    2^8 between context tiles and the output accumulator is rescaled."""
    out, ref = _run(311, [1000, 600], [700, 600], 16, growth=10.0)
    assert max_abs_err(out, ref) <= ATOL
    assert binding.pa_get_last_device_error() == 0


def test_prefill_many_items_per_persistent_cta():
    """More (query-tile pair, head, sequence) items than SMs, so every
    persistent CTA walks several items back to back (reusing its Q buffers,
    TMEM accumulators and K/V ring), with empty items mixed in."""
    rng = np.random.default_rng(312)
    lens = rng.integers(1, 700, size=24)
    n_new = [int(rng.integers(0, min(int(x), 600) + 1)) for x in lens]
    n_new[3] = int(lens[3])           # one whole prompt
    out, ref = _run(312, lens.tolist(), n_new, 16, h=8)
    assert max_abs_err(out, ref) <= ATOL
    assert binding.pa_get_last_device_error() == 0
