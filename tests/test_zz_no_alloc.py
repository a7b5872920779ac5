"""pa_decode_no_alloc: the decode entry point for callers that cannot allocate
device memory at decode time (a serving engine whose KV block pool already
holds the free HBM, or a loop that must not let cudaMalloc synchronise the
device).  It must give the same results as pa_decode with a caller-supplied
workspace, call after call, while using only the library's static scratch.

Named so that pytest collects it last; it also passes on its own in a fresh
process."""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_481_b200 import binding, build, workloads

from gpu_helpers import ATOL, gpu_decode, max_abs_err, oracle_write_and_decode, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    binding.load()
    torch.cuda.init()


def _written(wl):
    t = to_dev(wl)
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slots"])
    return t


def _no_alloc(wl, t):
    out = torch.full_like(t["q"], float("nan"))
    binding.pa_decode_no_alloc(out, t["q"], t["k_cache"], t["v_cache"], t["tables"], t["lens"],
                               wl.max_context_len, wl.scale)
    return out


def test_matches_workspace_entry_point_on_two_calls_in_a_row():
    # contexts split between workers, so the static scratch holds partial
    # results and merge tickets; the second call sees what the first left
    wl = workloads.make_random(301, [1500, 40, 2049, 700, 1], num_heads=6, head_dim=128,
                               block_size=16, keep_logical=False)
    t = _written(wl)
    ref = gpu_decode(wl, t)
    exact, _, _ = oracle_write_and_decode(wl)
    for _ in range(2):
        out = _no_alloc(wl, t)
        torch.cuda.synchronize()
        err = float((out.float() - ref.float()).abs().max())
        assert err <= ATOL
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        # and against the oracle, so a fault shared by both entry points shows
        assert max_abs_err(out, exact) <= ATOL
    assert binding.pa_get_last_device_error() == 0


def test_second_call_with_other_sizes_and_the_13b_shape():
    first = workloads.make_random(302, [3000, 900], num_heads=3, head_dim=64, block_size=8,
                                  keep_logical=False)
    t1 = _written(first)
    a = _no_alloc(first, t1)
    wl = workloads.make_workload(2, device="cuda")
    t2 = _written(wl)
    b = _no_alloc(wl, t2)
    torch.cuda.synchronize()
    assert binding.pa_get_last_device_error() == 0
    ref_a, ref_b = gpu_decode(first, t1), gpu_decode(wl, t2)
    assert float((a.float() - ref_a.float()).abs().max()) <= ATOL
    assert float((b.float() - ref_b.float()).abs().max()) <= ATOL
    assert torch.equal(a.view(torch.int16), ref_a.view(torch.int16))
    assert torch.equal(b.view(torch.int16), ref_b.view(torch.int16))
    exact_a, _, _ = oracle_write_and_decode(first)
    assert max_abs_err(a, exact_a) <= ATOL
    assert binding.pa_get_last_device_error() == 0


def test_sizes_past_the_static_scratch_are_rejected_before_any_launch():
    lib = binding.load()
    null = ctypes.c_void_p(None)
    # one merge ticket per (sequence, head): 65535 x 64 of them exceed 8 MiB
    assert binding.pa_decode_workspace_size(65535, 64, 128, 16) > 8 << 20
    rc = lib.pa_decode_no_alloc(null, null, null, null, null, 1, null, 16, 65535, 64, 128, 16,
                                1, ctypes.c_float(1.0), null)
    assert rc == binding.PA_ERR_WORKSPACE
    # and through the binding, with real tensors
    b, h, d = 65535, 32, 64
    assert binding.pa_decode_workspace_size(b, h, d, 16) > 8 << 20
    q = torch.zeros((b, h, d), dtype=torch.float16, device="cuda")
    cache = torch.zeros((1, h, 16, d), dtype=torch.float16, device="cuda")
    tables = torch.zeros((b, 1), dtype=torch.int32, device="cuda")
    lens = torch.ones(b, dtype=torch.int32, device="cuda")
    with pytest.raises(binding.PAError) as e:
        binding.pa_decode_no_alloc(torch.empty_like(q), q, cache, cache, tables, lens, 16, 0.1)
    assert e.value.status == binding.PA_ERR_WORKSPACE
