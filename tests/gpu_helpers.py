"""Shared plumbing for the GPU parity tests: run the CUDA path through the
C-ABI binding and the oracle on host copies of the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_481_b200 import binding

# max-abs tolerance on fp16 attention outputs (fp32 accumulation on the GPU
# versus fp64 in the oracle; the fp16 output rounding alone is <= 2^-11 relative)
ATOL = 2e-3


def to_dev(wl, device="cuda"):
    """Device copies of a workload's tensors and integer structure."""
    d = torch.device(device)
    return dict(
        q=wl.q.to(d), k_cache=wl.k_cache.to(d).clone(), v_cache=wl.v_cache.to(d).clone(),
        new_key=wl.new_key.to(d), new_value=wl.new_value.to(d),
        slots=torch.from_numpy(wl.slot_mapping).to(d),
        tables=torch.from_numpy(np.ascontiguousarray(wl.block_tables)).to(d),
        lens=torch.from_numpy(wl.context_lens).to(d),
    )


def gpu_write_and_decode(wl, t=None, max_context_len=None, tables=None, stream=None):
    """pa_reshape_and_cache of the newest tokens, then pa_decode.  Returns
    (out, k_cache, v_cache) on the device."""
    t = t or to_dev(wl)
    binding.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slots"], stream=stream)
    out = gpu_decode(wl, t, max_context_len=max_context_len, tables=tables, stream=stream)
    return out, t["k_cache"], t["v_cache"]


def gpu_decode(wl, t, max_context_len=None, tables=None, stream=None, workspace=None):
    mcl = wl.max_context_len if max_context_len is None else max_context_len
    tables = t["tables"] if tables is None else tables
    out = torch.empty_like(t["q"])
    ws = workspace if workspace is not None else binding.new_workspace(
        wl.num_seqs, wl.num_heads, wl.head_dim, mcl)
    binding.pa_decode(out, t["q"], t["k_cache"], t["v_cache"], tables, t["lens"], mcl,
                      wl.scale, ws, stream=stream)
    return out


def oracle_write_and_decode(wl, seqs=None):
    """The oracle on host copies: cache write, then decode (all sequences, or
    the listed ones)."""
    kc, vc = oracle.reshape_and_cache(wl.new_key.cpu().numpy(), wl.new_value.cpu().numpy(),
                                      wl.k_cache.cpu().numpy(), wl.v_cache.cpu().numpy(),
                                      wl.slot_mapping, wl.block_size)
    tables, lens, q = wl.block_tables, wl.context_lens, wl.q.cpu().numpy()
    if seqs is not None:
        tables, lens, q = tables[seqs], lens[seqs], q[seqs]
    out = oracle.paged_decode(q, kc, vc, tables, lens, wl.scale)
    return out, kc, vc


def max_abs_err(gpu_out, ref):
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    return float(np.max(np.abs(g - ref))) if ref.size else 0.0
