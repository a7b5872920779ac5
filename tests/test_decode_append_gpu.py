"""pa_decode_append (the decode step's cache write fused into the paged
decode launch) against the oracle's cache write followed by its decode, and
against the two separate CUDA calls bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_481_b200 import binding, build, workloads

from gpu_helpers import ATOL, gpu_write_and_decode, max_abs_err, oracle_write_and_decode, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    binding.load()
    torch.cuda.init()


def _fused(wl, t, slots=None):
    out = torch.empty_like(t["q"])
    ws = binding.new_workspace(wl.num_seqs, wl.num_heads, wl.head_dim, wl.max_context_len)
    binding.pa_decode_append(out, t["q"], t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                             t["slots"] if slots is None else slots, t["tables"], t["lens"],
                             wl.max_context_len, wl.scale, ws)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("seed,lens,d,bs", [
    (401, [1, 17, 33, 50, 16, 15], 64, 16),
    (402, [200, 1, 129, 300], 128, 16),
    (403, [9, 8, 24, 100], 128, 8),        # last tile spans two blocks
    (404, [64, 65, 500], 128, 32),
    (405, [128, 129, 1000], 128, 128),
])
def test_fused_equals_write_then_decode(seed, lens, d, bs):
    wl = workloads.make_random(seed, lens, num_heads=4, head_dim=d, block_size=bs, pool_factor=2.0)
    t = to_dev(wl)
    out = _fused(wl, t)
    # oracle: cache write of the newest tokens, then decode
    okc, ovc = oracle.reshape_and_cache(wl.new_key.numpy(), wl.new_value.numpy(), wl.k_cache.numpy(),
                                        wl.v_cache.numpy(), wl.slot_mapping, bs)
    ref = oracle.paged_decode(wl.q.numpy(), okc, ovc, wl.block_tables, wl.context_lens, wl.scale)
    assert max_abs_err(out, ref) <= ATOL
    assert np.array_equal(t["k_cache"].cpu().numpy().view(np.uint16), okc.view(np.uint16))
    assert np.array_equal(t["v_cache"].cpu().numpy().view(np.uint16), ovc.view(np.uint16))
    # the two separate CUDA calls give the same bits
    out2, _, _ = gpu_write_and_decode(wl)
    assert torch.equal(out, out2)
    assert binding.pa_get_last_device_error() == 0


def test_fused_mixed_batch_and_no_new_token_rows():
    """A serving-like batch (64 sequences, lognormal lengths); half the
    sequences append nothing (slot -1) and decode their cache as it is."""
    rng = np.random.default_rng(407)
    lens = np.clip(np.round(rng.lognormal(np.log(300), 0.8, size=64)), 1, 2000).astype(int)
    wl = workloads.make_random(407, lens.tolist(), num_heads=8, head_dim=128, block_size=16,
                               pool_factor=1.5)
    t = to_dev(wl)
    slots = t["slots"].clone()
    skip = np.arange(0, wl.num_seqs, 2)
    slots[torch.from_numpy(skip).cuda()] = -1
    # the skipped sequences' newest token is written beforehand, as a cache would hold it
    keep = torch.zeros(wl.num_seqs, dtype=torch.bool)
    keep[skip] = True
    pre_slots = torch.where(keep.cuda(), t["slots"], torch.full_like(t["slots"], -1))
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"], pre_slots)
    out = _fused(wl, t, slots)
    okc, ovc = oracle.reshape_and_cache(wl.new_key.cpu().numpy(), wl.new_value.cpu().numpy(),
                                        wl.k_cache.cpu().numpy(), wl.v_cache.cpu().numpy(),
                                        wl.slot_mapping, wl.block_size)
    ref = oracle.paged_decode(wl.q.cpu().numpy(), okc, ovc, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert max_abs_err(out, ref) <= ATOL
    assert np.array_equal(t["k_cache"].cpu().numpy().view(np.uint16), okc.view(np.uint16))
    assert binding.pa_get_last_device_error() == 0


def test_fused_reports_a_slot_that_is_not_the_last_position():
    wl = workloads.make_random(406, [40, 70], num_heads=2, head_dim=128, block_size=16,
                               pool_factor=2.0)
    t = to_dev(wl)
    binding.pa_get_last_device_error()
    slots = t["slots"].clone()
    slots[1] = slots[1] - 1                 # the slot of position L - 2 instead of L - 1
    _fused(wl, t, slots)
    assert binding.pa_get_last_device_error() == binding.PA_DEVERR_SLOT


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [2, 3])
def test_fused_step_at_full_size(cfg):
    """The benchmarked step itself: pa_decode_append on the 13B decode batch
    (B=32, H=40, D=128, bs=16) and on the serving batch (B=256), against the
    oracle's cache write then decode over every sequence, and bit for bit
    against the two separate calls."""
    wl = workloads.make_workload(cfg, device="cuda")
    t = to_dev(wl)
    out = _fused(wl, t)
    ref, okc, ovc = oracle_write_and_decode(wl)
    assert max_abs_err(out, ref) <= ATOL
    assert np.array_equal(t["k_cache"].cpu().numpy().view(np.uint16), okc.view(np.uint16))
    assert np.array_equal(t["v_cache"].cpu().numpy().view(np.uint16), ovc.view(np.uint16))
    out2, _, _ = gpu_write_and_decode(wl)
    assert torch.equal(out, out2)
    assert binding.pa_get_last_device_error() == 0
