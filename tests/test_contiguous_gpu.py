"""pa_decode_contiguous, the contiguous-cache baseline (polomodov.tech "vLLM
and PagedAttention", slide 19): the same decode over K / V kept contiguous
per (sequence, head), [B, H, Lmax, D], read without a block table.  It must
match the oracle, and -- the tile partition and arithmetic being the same --
give exactly pa_decode's bits over the same values; positions past each
context end hold a NaN canary, so any over-read shows."""
import numpy as np
import pytest
import torch

from paged_kv_cache_481_b200 import binding, build, workloads

from gpu_helpers import ATOL, gpu_write_and_decode, max_abs_err, oracle_write_and_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    binding.load()
    torch.cuda.init()


def contiguous_kv(wl, lmax):
    """[B, H, lmax, D] K and V from the workload's logical tokens (the newest
    token included), NaN past each context end."""
    b, h, d = wl.num_seqs, wl.num_heads, wl.head_dim
    k = torch.full((b, h, lmax, d), float("nan"), dtype=torch.float16)
    v = torch.full((b, h, lmax, d), float("nan"), dtype=torch.float16)
    for i, length in enumerate(wl.context_lens):
        k[i, :, :length] = wl.logical_k[i]
        v[i, :, :length] = wl.logical_v[i]
    return k.cuda(), v.cuda()


@pytest.mark.parametrize("seed,d,bs,lens,extra", [
    (701, 128, 16, [1, 15, 16, 17, 300, 2049, 1024], 0),
    (702, 128, 8, [7, 8, 9, 777, 4100], 5),
    (703, 64, 16, [1, 33, 50, 640, 1111], 16),
    (704, 128, 128, [129, 1000, 3000], 3),
])
def test_contiguous_equals_paged_and_oracle(seed, d, bs, lens, extra):
    wl = workloads.make_random(seed, lens, num_heads=5, head_dim=d, block_size=bs,
                               keep_logical=True)
    lmax = int(max(lens)) + extra
    k, v = contiguous_kv(wl, lmax)
    q = wl.q.cuda()
    lens_d = torch.from_numpy(wl.context_lens).cuda()
    out = torch.empty_like(q)
    ws = binding.new_workspace(wl.num_seqs, wl.num_heads, d, wl.max_context_len)
    binding.pa_decode_contiguous(out, q, k, v, lens_d, wl.max_context_len, wl.scale, ws)
    torch.cuda.synchronize()
    ref, _, _ = oracle_write_and_decode(wl)
    err = max_abs_err(out, ref)
    assert err <= ATOL, f"max-abs {err:.3e}"
    paged, _, _ = gpu_write_and_decode(wl)
    assert torch.equal(out.view(torch.int16), paged.view(torch.int16))
    assert binding.pa_get_last_device_error() == 0


def test_contiguous_zero_length_and_bad_stride():
    wl = workloads.make_random(705, [40, 5], num_heads=2, head_dim=128, block_size=16,
                               keep_logical=True)
    k, v = contiguous_kv(wl, 64)
    lens = torch.tensor([0, 5], dtype=torch.int32, device="cuda")
    out = torch.full_like(wl.q.cuda(), float("nan"))
    ws = binding.new_workspace(2, 2, 128, 40)
    binding.pa_decode_contiguous(out, wl.q.cuda(), k, v, lens, 40, wl.scale, ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[0]) == 0
    assert not torch.isnan(out[1]).any()
    with pytest.raises(binding.PAError):  # the context bound exceeds the stride
        binding.pa_decode_contiguous(out, wl.q.cuda(), k, v, lens, 65, wl.scale, ws)
    assert binding.pa_get_last_device_error() == 0
