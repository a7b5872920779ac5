"""Seeded synthetic inputs for the paged decode path.

This module only builds inputs: sequence lengths, physical block placement,
block tables, slot numbers and fp16 values.  It performs none of the
attention arithmetic and is the only code shared by the CUDA path's tests and
the CPU oracle.

Input recipe (all values fp16 ~ N(0, 1), integer structure from
``numpy.random.default_rng(seed)``, values from a ``torch.Generator`` seeded
with the same seed on the device the tensors are built on):

* each sequence b has a logical K/V of shape [H, L_b, D]; it is placed into
  ceil(L_b / bs) physical blocks drawn from a random permutation of the pool
  (polomodov.tech "vLLM and PagedAttention", slide 10: logically contiguous
  blocks live at scattered physical ids; slide 12: one shared pool);
* every pool position that holds no token (free blocks, and the tail of each
  sequence's last block) is filled with a NaN canary, so any read of it shows
  up in the output;
* the newest token of each sequence (position L_b - 1) is left as canary in
  the pool and handed out as ``new_key`` / ``new_value`` with its slot
  (slot = physical_block * bs + offset), so the cache write must run before
  the decode reads it (slide 11: a new token goes into the next free slot and a
  new block is taken only when the last one is full).

Workloads (sizes from the path's five standard configurations):
  1 tiny: B=4, H=4, D=64, bs=16, L={1,17,33,50}, pool 32 blocks, scale 1/8
  2 LLaMA-13B decode: B=32, H=40, D=128, bs=16, L~U[256,2048], pool 2x needed
  3 serving batch: B=256, H=40, D=128, bs=16, L=clip(round(lognormal(ln 512,
    0.8)), 1, 4096), pool 1.5x needed (free blocks interleaved)
  4 shared prefix: 8 groups x 8 sequences sharing a 1024-token prefix, private
    tails U[1,256]; logical block 63 is duplicated per member by a CoW copy
  5 OPT-66B heads: B=128, H=72, D=128, L~U[1024,4096], bs in {8,...,128},
    same lengths and values for every bs
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

# fp16 quiet NaN bit pattern used as canary for pool positions without a token.
CANARY_BITS = 0x7E00

WORKLOAD_NAMES = {
    1: "tiny: B=4 H=4 D=64 bs=16 L={1,17,33,50}",
    2: "LLaMA-13B single-layer decode: B=32 H=40 D=128 bs=16 L~U[256,2048]",
    3: "13B serving batch: B=256 H=40 D=128 bs=16 L~lognormal(512,0.8) clip [1,4096]",
    4: "shared prefix: 8x8 seqs H=40 D=128 bs=16 prefix 1024 + tail U[1,256]",
    5: "OPT-66B heads: B=128 H=72 D=128 L~U[1024,4096] bs sweep",
}


@dataclass
class PagedWorkload:
    """One batch of decode inputs.  Tensors live on ``device``; integer
    structure is kept as numpy arrays and mirrored as tensors on demand."""
    name: str
    seed: int
    num_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    context_lens: np.ndarray          # [B] int32, decode context (includes newest token)
    block_tables: np.ndarray          # [B, MB] int32, -1 past ceil(L/bs)
    q: torch.Tensor                   # [B, H, D] fp16
    k_cache: torch.Tensor             # [NB, H, bs, D] fp16 (newest token still canary)
    v_cache: torch.Tensor
    new_key: torch.Tensor             # [N, H, D] fp16
    new_value: torch.Tensor
    slot_mapping: np.ndarray          # [N] int64
    copy_pairs: np.ndarray = field(default_factory=lambda: np.zeros((0, 2), np.int64))
    alias_block_tables: np.ndarray | None = None   # config 4: tables before the CoW copy
    group_start: np.ndarray | None = None   # config 4: [G + 1] first sequence of each group
    prefix_lens: np.ndarray | None = None   # config 4: [G] tokens the copy-on-write tables share
    logical_k: list | None = None     # per sequence [H, L, D] fp16 (small configs only)
    logical_v: list | None = None
    device_k: list | None = None      # per sequence [H, L, D] fp16 on the device (on request)
    device_v: list | None = None

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def device(self) -> torch.device:
        return self.q.device


def _canary_tensor(shape, device) -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.int16, device=device)
    t.fill_(CANARY_BITS)
    return t.view(torch.float16)


def _randn_half(shape, gen, device) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).half()


def _place_sequences(lens, bs, num_blocks, rng, placement="shuffled"):
    """Give each sequence ceil(L/bs) distinct physical ids, in order, from a
    random permutation of the pool ("shuffled") or from the pool in address
    order ("sequential": each sequence's blocks are physically consecutive,
    the contiguous-cache baseline).  Returns the [B, MB] table (-1 unused)."""
    nblk = [(int(x) + bs - 1) // bs for x in lens]
    need = sum(nblk)
    if need > num_blocks:
        raise ValueError(f"pool of {num_blocks} blocks cannot hold {need}")
    if placement == "sequential":
        perm = np.arange(num_blocks, dtype=np.int32)
    elif placement == "shuffled":
        perm = rng.permutation(num_blocks).astype(np.int32)
    else:
        raise ValueError(placement)
    mb = max(max(nblk) if nblk else 1, 1)
    tables = np.full((len(lens), mb), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(nblk):
        tables[b, :n] = perm[off:off + n]
        off += n
    return tables


def _fill_pool(cache, table_row, logical, bs):
    """Write logical [H, L, D] values into the blocks listed in table_row;
    positions past L keep their canary."""
    h, length, d = logical.shape
    nblk = (length + bs - 1) // bs
    if nblk == 0:
        return
    padded = _canary_tensor((h, nblk * bs, d), cache.device)
    padded[:, :length] = logical
    ids = torch.as_tensor(np.asarray(table_row[:nblk], dtype=np.int64), device=cache.device)
    cache.index_copy_(0, ids, padded.view(h, nblk, bs, d).permute(1, 0, 2, 3).contiguous())


def _newest_token_slots(lens, tables, bs):
    """slot of position L-1 for each sequence (slot = block * bs + offset)."""
    slots = np.empty(len(lens), dtype=np.int64)
    for b, length in enumerate(lens):
        pos = int(length) - 1
        slots[b] = int(tables[b, pos // bs]) * bs + pos % bs
    return slots


def build_paged(name, seed, lens, num_heads, head_dim, block_size, num_blocks,
                scale, device="cpu", rng=None, keep_logical=False,
                logical_fn=None, placement="shuffled", keep_tokens=False) -> PagedWorkload:
    """Generic builder: lengths -> placement -> values -> canary-marked pool.

    Every sequence must have L >= 1 (its newest token is written by the cache
    write step).  ``logical_fn(b, gen)`` may supply the [H, L_b, D] values;
    by default they are drawn in sequence order from one generator so they do
    not depend on the block size."""
    device = torch.device(device)
    lens = np.asarray(lens, dtype=np.int32)
    if (lens < 1).any():
        raise ValueError("every sequence needs at least its newest token")
    rng = rng if rng is not None else np.random.default_rng(seed)
    tables = _place_sequences(lens, block_size, num_blocks, rng, placement)
    gen = torch.Generator(device=device).manual_seed(seed)
    h, d, bs = num_heads, head_dim, block_size
    q = _randn_half((len(lens), h, d), gen, device)
    k_cache = _canary_tensor((num_blocks, h, bs, d), device)
    v_cache = _canary_tensor((num_blocks, h, bs, d), device)
    new_key = torch.empty((len(lens), h, d), dtype=torch.float16, device=device)
    new_value = torch.empty_like(new_key)
    lk, lv = ([], []) if keep_logical else (None, None)
    dk, dv = ([], []) if keep_tokens else (None, None)
    for b, length in enumerate(lens):
        if logical_fn is not None:
            kb, vb = logical_fn(b, gen)
        else:
            kb = _randn_half((h, int(length), d), gen, device)
            vb = _randn_half((h, int(length), d), gen, device)
        new_key[b] = kb[:, -1]
        new_value[b] = vb[:, -1]
        # the newest token is not in the pool yet: the cache write puts it there
        _fill_pool(k_cache, tables[b], kb[:, :-1], bs)
        _fill_pool(v_cache, tables[b], vb[:, :-1], bs)
        if keep_logical:
            lk.append(kb.cpu())
            lv.append(vb.cpu())
        if keep_tokens:
            dk.append(kb)
            dv.append(vb)
    slots = _newest_token_slots(lens, tables, bs)
    return PagedWorkload(name=name, seed=seed, num_heads=h, head_dim=d, block_size=bs,
                         num_blocks=num_blocks, scale=scale, context_lens=lens,
                         block_tables=tables, q=q, k_cache=k_cache, v_cache=v_cache,
                         new_key=new_key, new_value=new_value, slot_mapping=slots,
                         logical_k=lk, logical_v=lv, device_k=dk, device_v=dv)


def config_lengths(cfg: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    if cfg == 1:
        return np.array([1, 17, 33, 50], dtype=np.int32)
    if cfg == 2:
        return rng.integers(256, 2048, size=32, endpoint=True).astype(np.int32)
    if cfg == 3:
        x = np.round(rng.lognormal(mean=math.log(512.0), sigma=0.8, size=256))
        return np.clip(x, 1, 4096).astype(np.int32)
    if cfg == 5:
        return rng.integers(1024, 4096, size=128, endpoint=True).astype(np.int32)
    raise ValueError(f"no plain length recipe for config {cfg}")


def make_workload(cfg: int, device="cpu", seed: int | None = None,
                  block_size: int | None = None, keep_logical: bool = False,
                  num_seqs: int | None = None, placement: str = "shuffled",
                  keep_tokens: bool = False) -> PagedWorkload:
    """Build standard configuration ``cfg`` (1..5).  ``seed`` defaults to the
    config index (use cfg + 10 for the second draw).  ``num_seqs`` truncates
    the batch (smaller parity cases with the same length distribution);
    ``placement="sequential"`` lays every sequence out in consecutive
    physical blocks (same lengths and values)."""
    seed = cfg if seed is None else seed
    if cfg == 4:
        return make_shared_prefix(device=device, seed=seed, keep_logical=keep_logical,
                                  num_groups=8 if num_seqs is None else max(1, num_seqs // 8))
    lens = config_lengths(cfg, seed)
    if num_seqs is not None:
        lens = lens[:num_seqs]
    rng = np.random.default_rng(seed + 1000)
    if cfg == 1:
        h, d, bs, factor, nb_fixed = 4, 64, 16, None, 32
    elif cfg == 2:
        h, d, bs, factor, nb_fixed = 40, 128, 16, 2.0, None
    elif cfg == 3:
        h, d, bs, factor, nb_fixed = 40, 128, 16, 1.5, None
    elif cfg == 5:
        h, d, bs, factor, nb_fixed = 72, 128, 16, 1.25, None
    else:
        raise ValueError(cfg)
    if block_size is not None:
        bs = block_size
    need = sum((int(x) + bs - 1) // bs for x in lens)
    nb = nb_fixed if nb_fixed is not None else int(math.ceil(factor * need))
    return build_paged(WORKLOAD_NAMES[cfg], seed, lens, h, d, bs, nb, 1.0 / math.sqrt(d),
                       device=device, rng=rng, keep_logical=keep_logical, placement=placement,
                       keep_tokens=keep_tokens)


def make_shared_prefix(device="cpu", seed: int = 4, num_groups: int = 8,
                       group_size: int = 8, prefix_len: int = 1024, num_heads: int = 40,
                       head_dim: int = 128, block_size: int = 16,
                       keep_logical: bool = False) -> PagedWorkload:
    """Parallel sampling / shared prefix (comfyai.app 6.4.2-6.4.3; polomodov.tech
    slides 13-14).  Each group's members alias the same physical blocks for
    the prefix; each member has a private tail of U[1, 256] tokens.  Logical
    block prefix_len/bs - 1 (the prefix's last block) is duplicated for every
    member by a copy-on-write pair (src = shared block, dst = private copy):
    ``alias_block_tables`` point at the shared block, ``block_tables`` at the
    copies (valid only after the copy runs).  The copy targets start as canary."""
    device = torch.device(device)
    rng = np.random.default_rng(seed)
    h, d, bs = num_heads, head_dim, block_size
    if prefix_len % bs:
        raise ValueError("prefix must fill whole blocks")
    n_prefix_blocks = prefix_len // bs
    nseq = num_groups * group_size
    tails = rng.integers(1, 256, size=nseq, endpoint=True).astype(np.int32)
    lens = (prefix_len + tails).astype(np.int32)
    tail_blocks = [(int(t) + bs - 1) // bs for t in tails]
    need = num_groups * n_prefix_blocks + sum(tail_blocks) + nseq
    nb = int(math.ceil(1.25 * need))
    perm = rng.permutation(nb).astype(np.int32)
    off = 0

    def take(n):
        nonlocal off
        ids = perm[off:off + n]
        off += n
        return ids

    mb = n_prefix_blocks + max(tail_blocks)
    alias_tables = np.full((nseq, mb), -1, dtype=np.int32)
    cow_tables = np.full((nseq, mb), -1, dtype=np.int32)
    pairs = np.zeros((nseq, 2), dtype=np.int64)
    gen = torch.Generator(device=device).manual_seed(seed)
    q = _randn_half((nseq, h, d), gen, device)
    k_cache = _canary_tensor((nb, h, bs, d), device)
    v_cache = _canary_tensor((nb, h, bs, d), device)
    new_key = torch.empty((nseq, h, d), dtype=torch.float16, device=device)
    new_value = torch.empty_like(new_key)
    lk, lv = ([], []) if keep_logical else (None, None)
    for g in range(num_groups):
        shared = take(n_prefix_blocks)
        pk = _randn_half((h, prefix_len, d), gen, device)
        pv = _randn_half((h, prefix_len, d), gen, device)
        _fill_pool(k_cache, shared, pk, bs)
        _fill_pool(v_cache, shared, pv, bs)
        for m in range(group_size):
            s = g * group_size + m
            private_last = take(1)[0]
            tail_ids = take(tail_blocks[s])
            alias_tables[s, :n_prefix_blocks] = shared
            alias_tables[s, n_prefix_blocks:n_prefix_blocks + tail_blocks[s]] = tail_ids
            cow_tables[s] = alias_tables[s]
            cow_tables[s, n_prefix_blocks - 1] = private_last
            pairs[s] = (shared[-1], private_last)
            tk = _randn_half((h, int(tails[s]), d), gen, device)
            tv = _randn_half((h, int(tails[s]), d), gen, device)
            new_key[s] = tk[:, -1]
            new_value[s] = tv[:, -1]
            _fill_pool(k_cache, tail_ids, tk[:, :-1], bs)
            _fill_pool(v_cache, tail_ids, tv[:, :-1], bs)
            if keep_logical:
                lk.append(torch.cat([pk, tk], dim=1).cpu())
                lv.append(torch.cat([pv, tv], dim=1).cpu())
    slots = _newest_token_slots(lens, cow_tables, bs)
    # after the copy-on-write, a group's members share all prefix blocks but the last
    group_start = (np.arange(num_groups + 1) * group_size).astype(np.int32)
    prefix_lens = np.full(num_groups, prefix_len - bs, dtype=np.int32)
    return PagedWorkload(name=WORKLOAD_NAMES[4], seed=seed, num_heads=h, head_dim=d,
                         block_size=bs, num_blocks=nb, scale=1.0 / math.sqrt(d),
                         context_lens=lens, block_tables=cow_tables, q=q, k_cache=k_cache,
                         v_cache=v_cache, new_key=new_key, new_value=new_value,
                         slot_mapping=slots, copy_pairs=pairs,
                         alias_block_tables=alias_tables, group_start=group_start,
                         prefix_lens=prefix_lens, logical_k=lk, logical_v=lv)


def make_random(seed: int, lens, num_heads: int, head_dim: int, block_size: int,
                pool_factor: float = 1.5, device="cpu", keep_logical=True,
                scale: float | None = None, keep_tokens: bool = False) -> PagedWorkload:
    """Small ad-hoc workload for parity and edge-case tests."""
    lens = np.asarray(lens, dtype=np.int32)
    need = sum((int(x) + block_size - 1) // block_size for x in lens)
    nb = max(int(math.ceil(pool_factor * need)), 1)
    scale = 1.0 / math.sqrt(head_dim) if scale is None else scale
    return build_paged(f"random seed={seed}", seed, lens, num_heads, head_dim, block_size,
                       nb, scale, device=device, keep_logical=keep_logical,
                       keep_tokens=keep_tokens)


def all_token_writes(wl: PagedWorkload, seqs=None):
    """Every context token of the chosen sequences as one cache-write batch:
    (keys [N, H, D], values [N, H, D], slots [N] int64), built from the kept
    device tokens (``keep_tokens=True``) and the block tables."""
    if wl.device_k is None:
        raise ValueError("workload was built without keep_tokens")
    seqs = range(wl.num_seqs) if seqs is None else seqs
    bs = wl.block_size
    keys, values, slots = [], [], []
    for b in seqs:
        length = int(wl.context_lens[b])
        pos = np.arange(length)
        slots.append(wl.block_tables[b, pos // bs].astype(np.int64) * bs + pos % bs)
        keys.append(wl.device_k[b].permute(1, 0, 2))
        values.append(wl.device_v[b].permute(1, 0, 2))
    return (torch.cat(keys).contiguous(), torch.cat(values).contiguous(),
            np.concatenate(slots))
