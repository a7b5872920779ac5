"""pa_decode_grouped (shared prefix once per group and head, scored for the
whole group on the tensor cores, tails scored alone, merged by their softmax
normalisers)
against the oracle's plain paged decode of every member over its full block
table -- the same mathematics (comfyai.app "6.4 PagedAttention", 6.4.2;
polomodov.tech slides 13-14)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_481_b200 import binding, build, workloads

from gpu_helpers import ATOL, max_abs_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    binding.load()
    torch.cuda.init()


def _groups(seed, sizes, prefix_blocks, max_tail, bs, h=4, d=128):
    """Groups of sequences sharing prefix blocks, each member with a private
    tail (0..max_tail tokens); random pool placement and values."""
    rng = np.random.default_rng(seed)
    tails = [[int(rng.integers(0, max_tail + 1)) for _ in range(n)] for n in sizes]
    need = sum(prefix_blocks) + sum(-(-t // bs) for ts in tails for t in ts) + 4
    nb = need * 2
    perm = rng.permutation(nb).astype(np.int32)
    off = 0
    lens, rows = [], []
    for pbk, ts in zip(prefix_blocks, tails):
        shared = perm[off:off + pbk]
        off += pbk
        for t in ts:
            own = perm[off:off + -(-t // bs)]
            off += len(own)
            rows.append(np.concatenate([shared, own]))
            lens.append(pbk * bs + t)
    mb = max(1, max(len(r) for r in rows))
    tables = np.full((len(rows), mb), -1, np.int32)
    for i, r in enumerate(rows):
        tables[i, :len(r)] = r
    g = torch.Generator().manual_seed(seed)
    kc = torch.randn((nb, h, bs, d), generator=g).half()
    vc = torch.randn((nb, h, bs, d), generator=g).half()
    q = torch.randn((len(rows), h, d), generator=g).half()
    gs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    pl = (np.asarray(prefix_blocks) * bs).astype(np.int32)
    return dict(kc=kc, vc=vc, q=q, tables=tables, lens=np.asarray(lens, np.int32), gs=gs, pl=pl,
                scale=d ** -0.5, max_group=max(sizes))


def _run(c, prefix_lens=None):
    dev = "cuda"
    b, h, d = c["q"].shape
    out = torch.full((b, h, d), float("nan"), dtype=torch.float16, device=dev)
    ws = binding.new_grouped_workspace(b, len(c["gs"]) - 1, h, d, int(c["lens"].max()),
                                       c["tables"].shape[1])
    pl = c["pl"] if prefix_lens is None else prefix_lens
    binding.pa_decode_grouped(out, c["q"].to(dev), c["kc"].to(dev), c["vc"].to(dev),
                              torch.from_numpy(c["tables"]).to(dev), torch.from_numpy(c["lens"]).to(dev),
                              int(c["lens"].max()), torch.from_numpy(c["gs"]).to(dev),
                              torch.from_numpy(np.ascontiguousarray(pl, np.int32)).to(dev),
                              c["max_group"], c["scale"], ws)
    torch.cuda.synchronize()
    ref = oracle.paged_decode(c["q"].numpy(), c["kc"].numpy(), c["vc"].numpy(), c["tables"],
                              c["lens"], c["scale"])
    return out, ref


@pytest.mark.parametrize("seed,sizes,prefix_blocks,max_tail,bs", [
    (501, [3, 1, 5, 2], [4, 0, 2, 7], 40, 16),        # a group with nothing shared
    (502, [8, 8], [64, 30], 256, 16),                 # long prefixes, several context tiles
    (503, [6, 4, 9], [9, 20, 3], 0, 16),              # no tails at all: prefix is everything
    (504, [4, 4], [33, 17], 100, 8),
    (505, [2, 3], [5, 3], 300, 64),
    (506, [130, 3], [4, 2], 20, 16),                  # a group larger than one query tile
    (508, [3, 5], [3, 2], 150, 128),                  # blocks as large as a context tile
    (509, [1, 1, 2], [6, 1, 3], 33, 32),              # single-member groups
])
def test_grouped_equals_plain_decode(seed, sizes, prefix_blocks, max_tail, bs):
    c = _groups(seed, sizes, prefix_blocks, max_tail, bs)
    out, ref = _run(c)
    assert not torch.isnan(out).any()
    assert max_abs_err(out, ref) <= ATOL
    assert binding.pa_get_last_device_error() == 0


def test_grouped_many_groups_and_both_work_lists_on_one_workspace():
    """More groups (40) than the prefix kernel builds a work list for by
    itself (32): the set-up kernel's list, the set-up launched first.  Then a
    3-group call (the prefix kernel first, on its own list) and the 40-group
    call again on the same workspace: each call leaves the work-list counters
    at zero for the next, whichever order it ran in."""
    rng = np.random.default_rng(512)
    sizes = [int(x) for x in rng.integers(1, 4, 40)]
    prefix_blocks = [int(x) for x in rng.integers(0, 6, 40)]
    many = _groups(512, sizes, prefix_blocks, 30, 16)
    few = _groups(513, [5, 2, 7], [6, 3, 9], 60, 16)
    dev = "cuda"
    cap = max(many["q"].shape[0], few["q"].shape[0])
    ws = binding.new_grouped_workspace(cap, 40, 4, 128, int(max(many["lens"].max(), few["lens"].max())),
                                       max(many["tables"].shape[1], few["tables"].shape[1]))
    for c in (many, few, many):
        b, h, d = c["q"].shape
        out = torch.full((b, h, d), float("nan"), dtype=torch.float16, device=dev)
        binding.pa_decode_grouped(out, c["q"].to(dev), c["kc"].to(dev), c["vc"].to(dev),
                                  torch.from_numpy(c["tables"]).to(dev),
                                  torch.from_numpy(c["lens"]).to(dev), int(c["lens"].max()),
                                  torch.from_numpy(c["gs"]).to(dev), torch.from_numpy(c["pl"]).to(dev),
                                  c["max_group"], c["scale"], ws)
        torch.cuda.synchronize()
        ref = oracle.paged_decode(c["q"].numpy(), c["kc"].numpy(), c["vc"].numpy(), c["tables"],
                                  c["lens"], c["scale"])
        assert not torch.isnan(out).any()
        assert max_abs_err(out, ref) <= ATOL
    assert binding.pa_get_last_device_error() == 0


def test_grouped_prefix_breaking_the_rules_falls_back():
    c = _groups(507, [3, 2], [4, 3], 30, 16)
    bad = c["pl"].copy()
    bad[0] += 5                                       # not a whole number of blocks
    out, ref = _run(c, bad)
    assert max_abs_err(out, ref) <= ATOL              # that group decodes without a shared prefix
    assert binding.pa_get_last_device_error() & binding.PA_DEVERR_CONTEXT_LEN


def test_grouped_on_the_shared_prefix_workload():
    """The shared-prefix workload (8 groups of 8, prefix 1024 tokens), smaller
    heads: through the aliased tables (all 64 prefix blocks shared) and the
    copy-on-write tables (the prefix's last block copied per member)."""
    wl = workloads.make_shared_prefix(device="cuda", num_heads=8)
    t = to_dev(wl)
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"], t["slots"])
    binding.pa_copy_blocks(t["k_cache"], t["v_cache"], torch.from_numpy(wl.copy_pairs).cuda())
    okc, ovc = oracle.reshape_and_cache(wl.new_key.cpu().numpy(), wl.new_value.cpu().numpy(),
                                        wl.k_cache.cpu().numpy(), wl.v_cache.cpu().numpy(),
                                        wl.slot_mapping, wl.block_size)
    okc, ovc = oracle.copy_blocks(okc, ovc, wl.copy_pairs)
    gs = torch.arange(0, 65, 8, dtype=torch.int32, device="cuda")
    for tables, prefix in ((wl.alias_block_tables, 1024), (wl.block_tables, 1008)):
        out = torch.empty_like(t["q"])
        ws = binding.new_grouped_workspace(wl.num_seqs, 8, wl.num_heads, wl.head_dim,
                                           wl.max_context_len, tables.shape[1])
        binding.pa_decode_grouped(out, t["q"], t["k_cache"], t["v_cache"],
                                  torch.from_numpy(np.ascontiguousarray(tables)).cuda(), t["lens"],
                                  wl.max_context_len, gs,
                                  torch.full((8,), prefix, dtype=torch.int32, device="cuda"), 8,
                                  wl.scale, ws)
        ref = oracle.paged_decode(wl.q.cpu().numpy(), okc, ovc, tables, wl.context_lens, wl.scale)
        assert max_abs_err(out, ref) <= ATOL
    assert binding.pa_get_last_device_error() == 0


def test_grouped_is_deterministic_and_the_workspace_reusable():
    """Repeated calls give the same bits (fixed merge order); a smaller
    problem on the same workspace afterwards is still right (the merge
    tickets reset themselves)."""
    c = _groups(510, [8, 8, 3], [40, 20, 9], 200, 16)
    b, h, d = c["q"].shape
    dev = "cuda"
    ws = binding.new_grouped_workspace(b, 3, h, d, int(c["lens"].max()), c["tables"].shape[1])
    args = [c["q"].to(dev), c["kc"].to(dev), c["vc"].to(dev), torch.from_numpy(c["tables"]).to(dev),
            torch.from_numpy(c["lens"]).to(dev), int(c["lens"].max()),
            torch.from_numpy(c["gs"]).to(dev), torch.from_numpy(c["pl"]).to(dev), c["max_group"],
            c["scale"], ws]
    outs = []
    for _ in range(4):
        out = torch.empty((b, h, d), dtype=torch.float16, device=dev)
        binding.pa_decode_grouped(out, *args)
        outs.append(out)
    for o in outs[1:]:
        assert torch.equal(outs[0].view(torch.int16), o.view(torch.int16))
    ref = oracle.paged_decode(c["q"].numpy(), c["kc"].numpy(), c["vc"].numpy(), c["tables"],
                              c["lens"], c["scale"])
    assert max_abs_err(outs[0], ref) <= ATOL
    small = _groups(511, [2, 5], [3, 6], 50, 16)
    sb, sh_, sd = small["q"].shape
    out = torch.empty((sb, sh_, sd), dtype=torch.float16, device=dev)
    binding.pa_decode_grouped(out, small["q"].to(dev), small["kc"].to(dev), small["vc"].to(dev),
                              torch.from_numpy(small["tables"]).to(dev),
                              torch.from_numpy(small["lens"]).to(dev), int(small["lens"].max()),
                              torch.from_numpy(small["gs"]).to(dev),
                              torch.from_numpy(small["pl"]).to(dev), small["max_group"],
                              small["scale"], ws)
    ref = oracle.paged_decode(small["q"].numpy(), small["kc"].numpy(), small["vc"].numpy(),
                              small["tables"], small["lens"], small["scale"])
    assert max_abs_err(out, ref) <= ATOL
    assert binding.pa_get_last_device_error() == 0


def _mark(c, seed):
    """Exactly uniform weights (q = 0) and V rows that are zero except +-64 in
    one dim, so a row read twice or not at all moves the output by 64 / L,
    far above the tolerance even at long contexts."""
    nb, h, bs, d = c["vc"].shape
    rng = np.random.default_rng(seed)
    v = np.zeros((nb, h, bs, d), np.float16)
    p, hh, j = np.meshgrid(np.arange(nb), np.arange(h), np.arange(bs), indexing="ij")
    v[p, hh, j, (p * bs + j + hh) % d] = rng.choice(np.array([-64.0, 64.0], np.float16),
                                                    size=(nb, h, bs))
    c = dict(c)
    c["vc"] = torch.from_numpy(v)
    c["q"] = torch.zeros_like(c["q"])
    return c


@pytest.mark.parametrize("seed,sizes,prefix_blocks,max_tail,bs", [
    (520, [8, 8], [256, 128], 600, 16),               # prefixes of 4096 and 2048 tokens
    (521, [16, 5, 1], [200, 64, 10], 900, 8),
    (522, [4, 20], [40, 33], 2000, 128),
])
def test_grouped_every_row_counts_once(seed, sizes, prefix_blocks, max_tail, bs):
    c = _mark(_groups(seed, sizes, prefix_blocks, max_tail, bs), seed)
    out, ref = _run(c)
    err = max_abs_err(out, ref)
    assert err <= ATOL, f"max-abs {err:.3e}"
    # the test's power: the oracle with one row dropped differs by > 3 ATOL
    short = c["lens"].copy()
    short[0] -= 1
    dropped = oracle.paged_decode(c["q"].numpy(), c["kc"].numpy(), c["vc"].numpy(), c["tables"],
                                  short, c["scale"])
    assert np.abs(dropped - ref).max() > 3 * ATOL
    assert binding.pa_get_last_device_error() == 0


@pytest.mark.slow
def test_grouped_on_the_full_shared_prefix_workload():
    """The shared-prefix workload at full size (40 heads) after its
    copy-on-write copies, through both tables, against the oracle."""
    wl = workloads.make_workload(4, device="cuda")
    t = to_dev(wl)
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"], t["slots"])
    binding.pa_copy_blocks(t["k_cache"], t["v_cache"], torch.from_numpy(wl.copy_pairs).cuda())
    okc, ovc = oracle.reshape_and_cache(wl.new_key.cpu().numpy(), wl.new_value.cpu().numpy(),
                                        wl.k_cache.cpu().numpy(), wl.v_cache.cpu().numpy(),
                                        wl.slot_mapping, wl.block_size)
    okc, ovc = oracle.copy_blocks(okc, ovc, wl.copy_pairs)
    gs = torch.arange(0, 65, 8, dtype=torch.int32, device="cuda")
    ws = binding.new_grouped_workspace(wl.num_seqs, 8, wl.num_heads, wl.head_dim,
                                       wl.max_context_len, wl.block_tables.shape[1])
    for tables, prefix in ((wl.alias_block_tables, 1024), (wl.block_tables, 1008)):
        out = torch.empty_like(t["q"])
        binding.pa_decode_grouped(out, t["q"], t["k_cache"], t["v_cache"],
                                  torch.from_numpy(np.ascontiguousarray(tables)).cuda(), t["lens"],
                                  wl.max_context_len, gs,
                                  torch.full((8,), prefix, dtype=torch.int32, device="cuda"), 8,
                                  wl.scale, ws)
        ref = oracle.paged_decode(wl.q.cpu().numpy(), okc, ovc, tables, wl.context_lens, wl.scale)
        err = max_abs_err(out, ref)
        assert err <= ATOL, f"max-abs {err:.3e}"
    assert binding.pa_get_last_device_error() == 0
