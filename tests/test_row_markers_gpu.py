"""Long contexts whose every row leaves a visible mark on the output.

Paging must leave the attention arithmetic unchanged (brentwoodlivery.com
"5.3.18 ...", "Common mistake: PagedAttention makes the attention math
faster"): every row t < L enters once.  With random N(0, 1) inputs one row
carries weight ~1/L, so at L in the thousands dropping or doubling a row moves
the output by less than the 2e-3 tolerance.  Here the weights are made exactly
uniform (q = 0, or every K row of a head equal, so every score is the same
number and exp2(s - m) = 1 exactly) and V row t of head h is zero except
+-64 in dim (t + h) mod D.  The output is then the mean of V, each dim
counting its own rows: a missing or doubled row moves one dim by 64 / L
>= 7.8e-3 at L <= 8192, well above the tolerance.  The lengths put the
ends of the decode's per-worker ranges inside the contexts."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_481_b200 import binding, build, workloads

from gpu_helpers import ATOL, gpu_write_and_decode, max_abs_err, oracle_write_and_decode, to_dev

pytestmark = pytest.mark.gpu

MARK = 64.0


def marked_workload(seed, lens, num_heads, head_dim, block_size, equal_keys):
    """Workload with marker V rows; q = 0 (equal_keys False) or random q over
    K rows that are equal within each head (equal_keys True)."""
    h, d = num_heads, head_dim
    rng = np.random.default_rng(seed)

    def logical(b, gen):
        length = int(lens[b])
        t = np.arange(length)
        v = np.zeros((h, length, d), np.float16)
        sign = rng.choice(np.array([-MARK, MARK], np.float16), size=(h, length))
        for head in range(h):
            v[head, t, (t + head) % d] = sign[head]
        if equal_keys:
            k0 = rng.standard_normal((h, 1, d)).astype(np.float16)
            k = np.broadcast_to(k0, (h, length, d)).copy()
        else:
            k = rng.standard_normal((h, length, d)).astype(np.float16)
        return torch.from_numpy(k), torch.from_numpy(v)

    need = sum(-(-int(x) // block_size) for x in lens)
    wl = workloads.build_paged(f"row markers seed={seed}", seed, lens, h, d, block_size,
                               int(need * 1.5) + 1, 1.0 / np.sqrt(d), logical_fn=logical)
    if not equal_keys:
        wl.q.zero_()
    return wl


def _mutant_gap(wl):
    """Smallest output change the oracle sees from dropping the last row of
    one sequence, or from reading one row twice: the test's power."""
    kc, vc = oracle.reshape_and_cache(wl.new_key.numpy(), wl.new_value.numpy(),
                                      wl.k_cache.numpy(), wl.v_cache.numpy(),
                                      wl.slot_mapping, wl.block_size)
    q = wl.q.numpy()
    ref = oracle.paged_decode(q, kc, vc, wl.block_tables, wl.context_lens, wl.scale)
    short = wl.context_lens.copy()
    short[0] -= 1
    dropped = oracle.paged_decode(q, kc, vc, wl.block_tables, short, wl.scale)
    tables = wl.block_tables.copy()
    tables[0, 1] = tables[0, 0]                      # block 0 read twice, block 1 never
    doubled = oracle.paged_decode(q, kc, vc, tables, wl.context_lens, wl.scale)
    return min(np.abs(dropped - ref).max(), np.abs(doubled - ref).max())


CASES = [
    # (seed, heads, head_dim, block_size, lengths, equal_keys)
    (601, 8, 128, 16, [2000, 8192, 4097, 6001, 3333, 5120], False),
    (602, 8, 128, 16, [8192, 2049, 7777, 4000, 5555, 2500], True),
    (603, 72, 128, 8, [4096, 1024, 3001], False),
    (604, 72, 128, 32, [2222, 4095, 1500], True),
    (605, 72, 128, 128, [4096, 3000, 1100], False),
    (606, 16, 64, 16, [8192, 3000, 6500, 2001], False),
]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    binding.load()
    torch.cuda.init()


@pytest.mark.parametrize("seed,h,d,bs,lens,equal_keys", CASES)
def test_every_row_counts_once_in_pa_decode(seed, h, d, bs, lens, equal_keys):
    wl = marked_workload(seed, lens, h, d, bs, equal_keys)
    assert _mutant_gap(wl) > 3 * ATOL
    out, _, _ = gpu_write_and_decode(wl)
    ref, _, _ = oracle_write_and_decode(wl)
    err = max_abs_err(out, ref)
    assert err <= ATOL, f"max-abs {err:.3e}"
    assert binding.pa_get_last_device_error() == 0


@pytest.mark.parametrize("seed,h,d,bs,lens,equal_keys", CASES)
def test_every_row_counts_once_in_pa_decode_append(seed, h, d, bs, lens, equal_keys):
    wl = marked_workload(seed, lens, h, d, bs, equal_keys)
    t = to_dev(wl)
    out = torch.empty_like(t["q"])
    ws = binding.new_workspace(wl.num_seqs, wl.num_heads, wl.head_dim, wl.max_context_len)
    binding.pa_decode_append(out, t["q"], t["new_key"], t["new_value"], t["k_cache"],
                             t["v_cache"], t["slots"], t["tables"], t["lens"],
                             wl.max_context_len, wl.scale, ws)
    torch.cuda.synchronize()
    ref, okc, _ = oracle_write_and_decode(wl)
    err = max_abs_err(out, ref)
    assert err <= ATOL, f"max-abs {err:.3e}"
    assert np.array_equal(t["k_cache"].cpu().numpy().view(np.uint16), okc.view(np.uint16))
    assert binding.pa_get_last_device_error() == 0
