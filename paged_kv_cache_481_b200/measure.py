"""Measurements of the path's secondary entry points on one GPU.

    python -m paged_kv_cache_481_b200.measure prefill [--iters N]
    python -m paged_kv_cache_481_b200.measure swap [--iters N]
    python -m paged_kv_cache_481_b200.measure grouped [--iters N]
    python -m paged_kv_cache_481_b200.measure cache [--iters N]

Each prints one JSON line per case.  Times are CUDA events on the launching
stream around N back-to-back calls after warm-up; inputs are synthetic
(seeded) with LLaMA-13B attention shapes (H=40, D=128) in randomly
placed (shuffled) pool blocks.

prefill: causal multi-query attention of each sequence's new tokens over its
paged cache.  Algorithmic FLOPs count only the unmasked scores: a new token
at position p does 2*D*(p+1) multiply-adds for q.K and the same for P.V per
head, i.e. 4*D*(p+1) FLOPs.  The roofline peak is the measured dense bf16
tensor rate (fp16 runs at the same rate on this architecture).

grouped: decode of the shared-prefix batch (8 groups of 8 sequences, a
1024-token prefix, private tails of 1-256 tokens, H=40, D=128, bs=16) with
pa_decode and with pa_decode_grouped (the prefix read once per group and
head); bytes = what DRAM must deliver, each physical row once.

cache: pa_reshape_and_cache of one decode step's new tokens (32 and 256
sequences, H=40, D=128, bs=16) and pa_copy_blocks of 64 copy-on-write pairs,
GB/s = (bytes read + bytes written) / t; these kernels are a few
microseconds, so they are timed as 20 launches replayed from a CUDA graph
(host launch overhead excluded).

swap: pa_swap_blocks between the device pool and a page-locked host pool, in
both directions, against a plain copy of the same number of contiguous bytes
over the same link (cudaMemcpyAsync via torch) as the link's reference.
"""
from __future__ import annotations

import argparse
import json
import os

import numpy as np
import torch

from . import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


def _time_ms(fn, iters, warmup=3):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def _time_graph_ms(fn, launches: int = 20, iters: int = 5):
    """Per-launch device time of a short kernel: `launches` calls captured in
    a CUDA graph and replayed, so host launch overhead does not show."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(launches):
            fn()
    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / (iters * launches)


PREFILL_CASES = [
    # (name, num_seqs, context length L, new tokens n per sequence)
    ("prompts 8 x 2048", 8, 2048, 2048),
    ("prompts 4 x 4096", 4, 4096, 4096),
    ("prompts 16 x 1024", 16, 1024, 1024),
    ("chunks 8 x 512 new of 4096", 8, 4096, 512),
    ("prompts 32 x 512", 32, 512, 512),
]


def measure_prefill(iters: int, block_size: int = 16, seed: int = 0, case: str | None = None):
    h, d, bs = 40, 128, block_size
    peak, peak_sus, kind = _peaks()
    g = torch.Generator(device="cuda").manual_seed(seed)
    out_lines = []
    for name, b, length, n in PREFILL_CASES:
        if case is not None and case != name:
            continue
        per_seq = -(-length // bs)
        nb = b * per_seq
        kc = torch.randn((nb, h, bs, d), generator=g, device="cuda").half()
        vc = torch.randn((nb, h, bs, d), generator=g, device="cuda").half()
        tables = torch.randperm(nb, generator=g, device="cuda").int().view(b, per_seq)
        lens = torch.full((b,), length, dtype=torch.int32, device="cuda")
        qsl = torch.arange(b + 1, dtype=torch.int32, device="cuda") * n
        q = torch.randn((b * n, h, d), generator=g, device="cuda").half()
        out = torch.empty_like(q)
        ms = _time_ms(lambda: binding.pa_prefill(out, q, kc, vc, tables, lens, length, qsl, n,
                                                 d ** -0.5), iters)
        pos = np.arange(length - n, length, dtype=np.float64)
        flops = b * h * 4 * d * float((pos + 1).sum())
        tflops = flops / (ms * 1e-3) / 1e12
        line = {"what": "pa_prefill", "case": name, "num_seqs": b, "context_len": length,
                "new_tokens": n, "num_heads": h, "head_dim": d, "block_size": bs,
                "ms": ms, "tflops": tflops, "peak_tflops": peak, "peak_kind": kind,
                "frac": tflops / peak, "algorithmic_flops": flops,
                "device_error": binding.pa_get_last_device_error()}
        print(json.dumps(line), flush=True)
        out_lines.append(line)
        del kc, vc, q, out
    return out_lines


def measure_swap(iters: int, num_blocks: int = 1024, seed: int = 0):
    h, d, bs = 40, 128, 16
    g = torch.Generator(device="cuda").manual_seed(seed)
    dev = torch.randn((num_blocks, h, bs, d), generator=g, device="cuda").half()
    host = torch.empty((num_blocks, h, bs, d), dtype=torch.float16).pin_memory()
    perm = torch.randperm(num_blocks, generator=g, device="cuda")
    pairs = torch.stack([torch.arange(num_blocks, device="cuda"), perm], 1).contiguous()
    nbytes = dev.numel() * dev.element_size()
    lines = []
    for direction, src, dst in (("device->host", dev, host), ("host->device", host, dev)):
        ms = _time_ms(lambda: binding.pa_swap_blocks(src, dst, pairs), iters)
        ms_ref = _time_ms(lambda: dst.copy_(src, non_blocking=True), iters)
        line = {"what": "pa_swap_blocks", "direction": direction, "blocks": num_blocks,
                "block_bytes": nbytes // num_blocks, "bytes": nbytes, "ms": ms,
                "gbs": nbytes / (ms * 1e-3) / 1e9,
                "link_copy_gbs": nbytes / (ms_ref * 1e-3) / 1e9,
                "frac_of_link_copy": ms_ref / ms,
                "device_error": binding.pa_get_last_device_error()}
        print(json.dumps(line), flush=True)
        lines.append(line)
    return lines


def measure_grouped(iters: int):
    from . import accounting, workloads
    wl = workloads.make_shared_prefix(device="cuda")
    h, d, bs = wl.num_heads, wl.head_dim, wl.block_size
    dev = torch.device("cuda")
    kc, vc = wl.k_cache, wl.v_cache
    binding.pa_reshape_and_cache(wl.new_key, wl.new_value, kc, vc,
                                 torch.from_numpy(wl.slot_mapping).to(dev))
    binding.pa_copy_blocks(kc, vc, torch.from_numpy(wl.copy_pairs).to(dev))
    q = wl.q
    lens = torch.from_numpy(wl.context_lens).to(dev)
    out = torch.empty_like(q)
    lines = []
    for name, tables, prefix in (("aliased prefix (64 shared blocks)", wl.alias_block_tables, 1024),
                                 ("copy-on-write prefix (63 shared blocks)", wl.block_tables, 1008)):
        t = torch.from_numpy(np.ascontiguousarray(tables)).to(dev)
        nbytes = accounting.decode_unique_bytes(tables, wl.context_lens, h, d, bs)
        ws = binding.new_workspace(wl.num_seqs, h, d, wl.max_context_len)
        ms_plain = _time_ms(lambda: binding.pa_decode(out, q, kc, vc, t, lens, wl.max_context_len,
                                                      wl.scale, ws), iters)
        gws = binding.new_grouped_workspace(wl.num_seqs, wl.num_seqs // 8, h, d,
                                            wl.max_context_len, tables.shape[1])
        gs = torch.arange(0, wl.num_seqs + 1, 8, dtype=torch.int32, device=dev)
        pl = torch.full((wl.num_seqs // 8,), prefix, dtype=torch.int32, device=dev)
        ms_grp = _time_ms(lambda: binding.pa_decode_grouped(out, q, kc, vc, t, lens,
                                                            wl.max_context_len, gs, pl, 8,
                                                            wl.scale, gws), iters)
        line = {"what": "pa_decode_grouped", "case": name, "num_seqs": wl.num_seqs,
                "groups": wl.num_seqs // 8, "prefix_len": prefix, "num_heads": h,
                "unique_bytes": nbytes, "plain_us": ms_plain * 1e3, "grouped_us": ms_grp * 1e3,
                "plain_gbs": nbytes / (ms_plain * 1e-3) / 1e9,
                "grouped_gbs": nbytes / (ms_grp * 1e-3) / 1e9, "speedup": ms_plain / ms_grp,
                "device_error": binding.pa_get_last_device_error()}
        print(json.dumps(line), flush=True)
        lines.append(line)
    return lines


def measure_cache(iters: int, seed: int = 0):
    from . import accounting
    h, d, bs = 40, 128, 16
    g = torch.Generator(device="cuda").manual_seed(seed)
    nb = 8192
    kc = torch.randn((nb, h, bs, d), generator=g, device="cuda").half()
    vc = torch.randn_like(kc)
    lines = []
    for n in (32, 256):
        key = torch.randn((n, h, d), generator=g, device="cuda").half()
        value = torch.randn_like(key)
        slots = (torch.randperm(nb, generator=g, device="cuda")[:n] * bs
                 + torch.randint(0, bs, (n,), generator=g, device="cuda")).long()
        ms = _time_graph_ms(lambda: binding.pa_reshape_and_cache(key, value, kc, vc, slots))
        nbytes = accounting.cache_write_bytes(n, h, d)
        line = {"what": "pa_reshape_and_cache", "tokens": n, "num_heads": h, "head_dim": d,
                "bytes": nbytes, "us": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9}
        print(json.dumps(line), flush=True)
        lines.append(line)
    perm = torch.randperm(nb, generator=g, device="cuda")[:128]
    pairs = torch.stack([perm[:64], perm[64:]], 1).contiguous().long()
    ms = _time_graph_ms(lambda: binding.pa_copy_blocks(kc, vc, pairs))
    nbytes = accounting.copy_blocks_bytes(64, h, d, bs)
    line = {"what": "pa_copy_blocks", "pairs": 64, "num_heads": h, "block_size": bs,
            "bytes": nbytes, "us": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9,
            "device_error": binding.pa_get_last_device_error()}
    print(json.dumps(line), flush=True)
    lines.append(line)
    return lines


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("what", choices=["prefill", "swap", "grouped", "cache"])
    ap.add_argument("--iters", type=int, default=10)
    ap.add_argument("--block-size", type=int, default=16)
    ap.add_argument("--case", default=None, help="only the prefill case of this name")
    args = ap.parse_args(argv)
    build.build()
    binding.load()
    if args.what == "prefill":
        measure_prefill(args.iters, args.block_size, case=args.case)
    elif args.what == "grouped":
        measure_grouped(args.iters)
    elif args.what == "cache":
        measure_cache(args.iters)
    else:
        measure_swap(args.iters)


if __name__ == "__main__":
    main()
