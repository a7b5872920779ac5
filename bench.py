"""Benchmark of the paged decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload C] [--block-size BS]
    python bench.py --kv-dtype int8 ...      # the same step over the int8 cache
    python bench.py --path prefill ...       # prompt cache write + pa_prefill, TFLOP/s
    python bench.py --workload 4 ...         # shared prefixes through pa_decode_grouped
    python bench.py --decode-only ...        # the decode alone (pa_decode / pa_decode_grouped)
    python bench.py --layout contiguous ...  # the same decode, contiguous K / V, no block table
    python bench.py --path prefill --new-tokens 512 --prompt-len 4096 ...  # chunked prefill
    python bench.py --path cache-write|copy-blocks|swap ...  # those entry points alone, GB/s
    python bench.py --impl reference ...     # the fp64 CPU oracle, same metric

One step = one decode iteration of the whole hot path over one batch: the
cache write of each sequence's newest token and the decode over all
(sequence, head) pairs -- fused into one pa_decode_append launch
(pa_decode_append_int8 for the int8 cache; --unfused: the cache write, then
the decode) -- and, for the shared-prefix workload, the
copy-on-write pa_copy_blocks before them and the decode done by pa_decode_grouped
(each shared prefix read once per group and head).  The default workload is the LLaMA-13B-shaped
single-layer decode batch (B=32, H=40, D=128, bs=16, context U[256, 2048]).

Under torchrun each rank runs its own batch (a different seed) on its own GPU:
sequences are independent, so there is no collective on the data path
("weak" scaling); rank 0 prints one JSON line with the whole-job throughput.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention: KV-cache GB/s (% of HBM peak), seq-heads/s"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2**20


def _peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = {
    "grouped": ("paged_kv_cache_481_b200/csrc/grouped_kernel.cuh",
                "paged_kv_cache_481_b200/csrc/grouped.cu",
                "paged_kv_cache_481_b200/csrc/tcgen05.cuh",
                "paged_kv_cache_481_b200/csrc/tma_host.cuh",
                "paged_kv_cache_481_b200/csrc/decode_kernel.cuh",
                "paged_kv_cache_481_b200/csrc/decode.cu",
                "paged_kv_cache_481_b200/csrc/ptx.cuh",
                "paged_kv_cache_481_b200/csrc/host_common.cuh"),
    "decode": ("paged_kv_cache_481_b200/csrc/decode_kernel.cuh",
               "paged_kv_cache_481_b200/csrc/quant.cuh",
               "paged_kv_cache_481_b200/csrc/ptx.cuh",
               "paged_kv_cache_481_b200/csrc/host_common.cuh",
               "paged_kv_cache_481_b200/csrc/decode.cu"),
    "prefill": ("paged_kv_cache_481_b200/csrc/prefill_kernel.cuh",
                "paged_kv_cache_481_b200/csrc/tcgen05.cuh",
                "paged_kv_cache_481_b200/csrc/ptx.cuh",
                "paged_kv_cache_481_b200/csrc/host_common.cuh",
                "paged_kv_cache_481_b200/csrc/prefill.cu"),
}


def _decode_kernel_hash(kind: str = "decode"):
    """Hash of a kernel's code (its sources with comments and whitespace
    removed), so that a recorded ncu capture stays attached to the code it
    measured."""
    import re
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update("".join(src.split()).encode())
    return h.hexdigest()


def _recorded_traffic(workload: str, launch: str = "pa_decode", kind: str = "decode"):
    """DRAM bytes per launch from the committed ncu summary of that kernel,
    only if it was taken on the current kernel source and this workload."""
    path = os.path.join(ROOT, "profiles", f"{kind}_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if (rec.get("kernel_sha256") != _decode_kernel_hash(kind) or rec.get("workload") != workload
            or rec.get("launch", "pa_decode") != launch):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """Polls the GPU's SM clock and clock-event reasons through NVML (read
    only) from a background thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            handle = None
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                try:
                    handle = pynvml.nvmlDeviceGetHandleByUUID(f"GPU-{uuid}")
                except Exception:
                    handle = None
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nvml, self._h = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) \
                or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception as e:  # no NVML: report that instead of guessing
            self.error = f"{type(e).__name__}: {e}"
            self._h = None
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self._nvml.nvmlDeviceGetClockInfo(self._h, self._nvml.NVML_CLOCK_SM)
                reasons = int(self._reasons_fn(self._h))
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception as e:
                self.error = f"{type(e).__name__}: {e}"
                return
            time.sleep(self._period)

    def start(self):
        if self._h is not None:
            self._thread.start()
        return self

    def stop(self):
        self._stop.set()
        if self._thread.is_alive():
            self._thread.join()

    def summary(self, t0: float, t1: float):
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:   # very short timed region: fall back to the whole window
            inside = self.samples
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "error": self.error}
        bits = 0
        for s in inside:
            bits |= s[2]
        names = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(inside)}


def rank_seed(cfg: int, rank: int) -> int:
    """Each rank decodes its own batch: same recipe, a rank-specific seed."""
    return cfg + 100 * rank


def reduce_over_ranks(max_vals, sum_vals, device):
    """Max of the device-timed regions and sum of the work over all ranks
    (identity on one process).  Runs outside any timed region."""
    import torch
    import torch.distributed as dist
    mx = torch.tensor([float(v) for v in max_vals], dtype=torch.float64, device=device)
    sm = torch.tensor([float(v) for v in sum_vals], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(mx, op=dist.ReduceOp.MAX)
        dist.all_reduce(sm, op=dist.ReduceOp.SUM)
    return mx.tolist(), sm.tolist()


def _workload_desc(wl, cfg):
    from paged_kv_cache_481_b200 import workloads
    return {
        "workload": workloads.WORKLOAD_NAMES[cfg] if cfg != 5 else
        f"{workloads.WORKLOAD_NAMES[5]} (bs={wl.block_size})",
        "num_seqs": wl.num_seqs, "num_heads": wl.num_heads, "head_dim": wl.head_dim,
        "block_size": wl.block_size, "num_blocks": wl.num_blocks,
        "mean_context_len": float(np.mean(wl.context_lens)),
        "max_context_len": wl.max_context_len, "seed": wl.seed,
    }


def _cpu_sample(wl, max_units: int, seqs=None):
    """Host inputs for the oracle on a bounded sample, cut from the pool as
    generated (before any GPU work): the first sequences' blocks, renumbered,
    completed by the oracle's own cache write of their newest tokens."""
    import oracle
    import torch
    if seqs is None:
        seqs = np.arange(min(wl.num_seqs, max(1, math.ceil(max_units / wl.num_heads))))
    tables = wl.block_tables[seqs]
    ids = np.unique(tables[tables >= 0])
    remap = np.full(wl.num_blocks, -1, np.int64)
    remap[ids] = np.arange(len(ids))
    sub_tables = np.where(tables >= 0, remap[np.maximum(tables, 0)], -1).astype(np.int32)
    idx = torch.from_numpy(ids).to(wl.k_cache.device)
    kc = wl.k_cache.index_select(0, idx).cpu().numpy()
    vc = wl.v_cache.index_select(0, idx).cpu().numpy()
    bs = wl.block_size
    slots = wl.slot_mapping[seqs]
    kc, vc = oracle.reshape_and_cache(wl.new_key[seqs].cpu().numpy(),
                                      wl.new_value[seqs].cpu().numpy(), kc, vc,
                                      remap[slots // bs] * bs + slots % bs, bs)
    return dict(q=wl.q[seqs].cpu().numpy(), kc=kc, vc=vc, tables=sub_tables,
                lens=wl.context_lens[seqs].copy(), scale=wl.scale)


def _quantize_sample(sample):
    """The int8 cache of a sample: every row of its fp16 pool quantized by the
    oracle (the same decisions as the CUDA cache write, bit for bit)."""
    import oracle
    out = dict(sample)
    for name in ("kc", "vc"):
        x = sample[name]
        codes, params = oracle.quantize_rows(x.reshape(-1, x.shape[-1]))
        out[name] = codes.reshape(x.shape)
        out[name[0] + "p"] = params.reshape(x.shape[:-1] + (2,))
    out["int8"] = True
    return out


def _oracle_decode(sample):
    import oracle
    if sample.get("int8"):
        return oracle.paged_decode_int8(sample["q"], sample["kc"], sample["vc"], sample["kp"],
                                        sample["vp"], sample["tables"], sample["lens"],
                                        sample["scale"])
    return oracle.paged_decode(sample["q"], sample["kc"], sample["vc"], sample["tables"],
                               sample["lens"], sample["scale"])


def _time_oracle(sample, reps: int = 1):
    t = []
    for _ in range(reps):
        t0 = time.perf_counter()
        _oracle_decode(sample)
        t.append(time.perf_counter() - t0)
    return statistics.median(t)


def cpu_baseline_sample(wl, target_s: float = 10.0, int8: bool = False):
    """Size and cut the CPU-baseline sample (call before any GPU work touches
    the pool): about target_s seconds of oracle decode -- the first sequences
    of the batch, or, when the whole batch takes less, the whole batch
    decoded repeatedly.  int8: over the oracle-quantized cache."""
    cut = (lambda units: _quantize_sample(_cpu_sample(wl, units))) if int8 else \
        (lambda units: _cpu_sample(wl, units))
    probe = cut(wl.num_heads)                                   # one sequence
    per_seq = max(_time_oracle(probe), 1e-4)
    nseq = int(min(wl.num_seqs, max(1, target_s / per_seq)))
    sample = cut(nseq * wl.num_heads)
    reps = 1
    if nseq == wl.num_seqs:
        per_batch = max(_time_oracle(sample), 1e-4)
        reps = int(max(1, min(10000, target_s / per_batch)))
    sample["reps"] = reps
    return sample


def cpu_baseline(wl, sample):
    """The oracle as it stands, on the host cores, on a bounded sample of the
    same workload; GB/s over the sample's algorithmic bytes."""
    import oracle
    from paged_kv_cache_481_b200 import accounting
    reps = int(sample.get("reps", 1))
    t0 = time.perf_counter()
    for _ in range(reps):
        _oracle_decode(sample)
    t = time.perf_counter() - t0
    int8 = bool(sample.get("int8"))
    nbytes = (accounting.decode_bytes_int8 if int8 else accounting.decode_bytes)(
        sample["lens"], wl.num_heads, wl.head_dim) * reps
    what = (f"first {len(sample['lens'])} of {wl.num_seqs} sequences" if reps == 1 else
            f"all {wl.num_seqs} sequences, {reps} times")
    return {"value": nbytes / t / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{what} x {wl.num_heads} heads (decode only, fp64"
                      f"{' over the int8 cache' if int8 else ''}), {t:.1f} s wall"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from paged_kv_cache_481_b200 import accounting, workloads
    import torch
    cfg = args.workload
    wl = workloads.make_workload(cfg, device="cpu" if not torch.cuda.is_available() else "cuda",
                                 seed=cfg, block_size=args.block_size)
    # size each step's sample so that warm-up + timed steps stay within ~2 min
    probe = _cpu_sample(wl, wl.num_heads)
    t1 = max(_time_oracle(probe), 1e-4)
    budget = 120.0 / max(1, args.steps + args.warmup)
    nseq = int(max(1, min(wl.num_seqs, budget / t1)))
    if nseq == 1 and t1 > budget:
        units = max(1, int(wl.num_heads * budget / t1))
        sample = _cpu_sample(wl, units, seqs=np.arange(1))
        sample["q"] = sample["q"][:, :units].copy()
        sample["kc"] = np.ascontiguousarray(sample["kc"][:, :units])
        sample["vc"] = np.ascontiguousarray(sample["vc"][:, :units])
        heads = units
    else:
        sample = _cpu_sample(wl, nseq * wl.num_heads)
        heads = wl.num_heads
    for _ in range(args.warmup):
        _time_oracle(sample)
    times = [_time_oracle(sample) for _ in range(args.steps)]
    total = sum(times)
    nbytes = accounting.decode_bytes(sample["lens"], heads, wl.head_dim)
    value = nbytes * args.steps / total / 1e9
    desc = (f"per step: {len(sample['lens'])} of {wl.num_seqs} sequences x {heads} heads "
            f"(decode only, fp64 oracle)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _workload_desc(wl, cfg),
        "seq_heads_per_s": len(sample["lens"]) * heads * args.steps / total,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _init_ranks(args):
    """This process's rank on its GPU (one process per GPU; NCCL process group
    with a short timeout when there are several), and the library loaded."""
    import torch
    import torch.distributed as dist
    from paged_kv_cache_481_b200 import binding, build
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    build.build()
    binding.load()
    return world, rank, local


def pipelined_e2e(parts, out_like, step, stream, warmup, steps, world):
    """End-to-end timing through the public API with host buffers: each
    step's inputs (`parts`, packed in one pinned host buffer) are copied to
    the device and its output back to pinned host memory.  As a serving loop
    would, the copies are pipelined with the compute: two device staging
    buffers and two outputs, the inputs of step i + 1 going up on one copy
    stream and the result of step i - 1 coming back on another while step i
    runs on `stream`.  The timed region (CUDA events on `stream`) ends when
    the last result is in host memory, so every step's copies are inside it.
    `step(views, out)` launches one step on `stream` from the staged inputs.
    Returns (ms for `steps` steps, h2d bytes per step, d2h bytes per step)."""
    import torch
    import torch.distributed as dist
    dev = out_like.device
    offs, total = [], 0
    for t in parts:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_stage = torch.empty(total, dtype=torch.uint8, pin_memory=True)
    d_stages = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]
    stage_views = []
    for d_stage in d_stages:
        views = []
        for t, o in zip(parts, offs):
            n = t.numel() * t.element_size()
            views.append(d_stage[o:o + n].view(t.dtype).view(t.shape))
        stage_views.append(views)
    for t, o in zip(parts, offs):
        n = t.numel() * t.element_size()
        h_stage[o:o + n].copy_(t.reshape(-1).view(torch.uint8).cpu())
    outs = [torch.empty_like(out_like) for _ in range(2)]
    h_outs = [torch.empty(out_like.shape, dtype=out_like.dtype, pin_memory=True)
              for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in parts)
    d2h = h_outs[0].numel() * h_outs[0].element_size()
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def run(n, start_event):
        up_done = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        down_done = [torch.cuda.Event() for _ in range(2)]
        up.wait_event(start_event)
        with torch.cuda.stream(up):
            d_stages[0].copy_(h_stage, non_blocking=True)
            up_done[0].record(up)
        for i in range(n):
            cur, nxt = i % 2, (i + 1) % 2
            if i + 1 < n:  # inputs of the next step, once step i - 1 has used that buffer
                with torch.cuda.stream(up):
                    if i >= 1:
                        up.wait_event(done[nxt])
                    d_stages[nxt].copy_(h_stage, non_blocking=True)
                    up_done[nxt].record(up)
            stream.wait_event(up_done[cur])
            if i >= 2:  # step i - 2's result has left outs[cur]
                stream.wait_event(down_done[cur])
            with torch.cuda.stream(stream):
                step(stage_views[cur], outs[cur])
                done[cur].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(done[cur])
                h_outs[cur].copy_(outs[cur], non_blocking=True)
                down_done[cur].record(down)
        stream.wait_event(down_done[(n - 1) % 2])

    warm = torch.cuda.Event()
    warm.record(stream)
    run(max(3, warmup), warm)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(steps, e0)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return e0.elapsed_time(e1), h2d, d2h


def run_gpu(args):
    import torch
    import torch.distributed as dist
    from paged_kv_cache_481_b200 import accounting, binding, workloads

    world, rank, local = _init_ranks(args)

    cfg = args.workload
    int8 = args.kv_dtype == "int8"
    wl = workloads.make_workload(cfg, device="cuda", seed=rank_seed(cfg, rank),
                                 block_size=args.block_size, placement=args.placement,
                                 keep_tokens=int8)
    dev = torch.device("cuda", local)
    cpu_sample = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_sample = cpu_baseline_sample(wl, target_s=args.cpu_seconds, int8=int8)
    stream = torch.cuda.Stream(device=dev)
    b, h, d = wl.num_seqs, wl.num_heads, wl.head_dim
    q = wl.q
    kc, vc = wl.k_cache, wl.v_cache
    key, value = wl.new_key, wl.new_value
    slots = torch.from_numpy(wl.slot_mapping).to(dev)
    tables = torch.from_numpy(np.ascontiguousarray(wl.block_tables)).to(dev)
    lens = torch.from_numpy(wl.context_lens).to(dev)
    pairs = torch.from_numpy(wl.copy_pairs).to(dev) if len(wl.copy_pairs) else None
    out = torch.empty_like(q)
    mcl = wl.max_context_len
    ws = binding.new_workspace(b, h, d, mcl, device=dev)
    if int8:
        # the int8 pool is filled by the int8 cache write of every context
        # token; the fp16 pool is then released
        nbk, bsz = wl.num_blocks, wl.block_size
        kc = torch.zeros((nbk, h, bsz, d), dtype=torch.uint8, device=dev)
        vc = torch.zeros_like(kc)
        kp = torch.zeros((nbk, h, bsz, 2), dtype=torch.float32, device=dev)
        vp = torch.zeros_like(kp)
        all_k, all_v, all_s = workloads.all_token_writes(wl)
        binding.pa_reshape_and_cache_int8(all_k, all_v, kc, vc, kp, vp,
                                          torch.from_numpy(all_s).to(dev))
        del all_k, all_v
        wl.device_k = wl.device_v = None
        torch.cuda.synchronize()
    torch.cuda.synchronize()

    def write_step(d_key, d_value, d_slots):
        if int8:
            binding.pa_reshape_and_cache_int8(d_key, d_value, kc, vc, kp, vp, d_slots,
                                              stream=stream)
        else:
            binding.pa_reshape_and_cache(d_key, d_value, kc, vc, d_slots, stream=stream)

    def decode_step(d_out, d_q, d_tables, d_lens):
        if int8:
            binding.pa_decode_int8(d_out, d_q, kc, vc, kp, vp, d_tables, d_lens, mcl, wl.scale,
                                   ws, stream=stream)
        else:
            binding.pa_decode(d_out, d_q, kc, vc, d_tables, d_lens, mcl, wl.scale, ws,
                              stream=stream)

    def copy_step():
        if int8:
            for cache in (kc, vc, kp, vp):
                binding.pa_copy_blocks_raw(cache, pairs, stream=stream)
        else:
            binding.pa_copy_blocks(kc, vc, pairs, stream=stream)

    fused = not args.unfused
    # the shared-prefix workload decodes its groups with pa_decode_grouped
    # (each shared prefix read once per group and head); --no-grouped: pa_decode
    grouped = wl.group_start is not None and not args.no_grouped and not int8
    if grouped:
        d_gs = torch.from_numpy(wl.group_start).to(dev)
        d_pl = torch.from_numpy(wl.prefix_lens).to(dev)
        max_group = int(np.diff(wl.group_start).max())
        gws = binding.new_grouped_workspace(b, len(wl.prefix_lens), h, d, mcl, tables.shape[1],
                                            device=dev)
        fused = False

    # decode alone (the newest tokens written, and the shared-prefix workload's
    # blocks copied, once before timing): over the paged pool (--decode-only;
    # pa_decode_grouped for the shared-prefix workload), or over a contiguous
    # copy of the same values with no block table (--layout contiguous)
    contig = args.layout == "contiguous"
    decode_only = args.decode_only or contig
    if decode_only:
        if int8 or (contig and pairs is not None):
            raise SystemExit("--decode-only: fp16 only; --layout contiguous: workloads 1, 2, 3 "
                             "and 5")
        if pairs is not None:
            copy_step()
        write_step(key, value, slots)
        fused = False
    if contig:
        # gather each sequence's blocks into [B, H, Lmax, D] (the same values)
        kcont = torch.zeros((b, h, mcl, d), dtype=torch.float16, device=dev)
        vcont = torch.zeros_like(kcont)
        bsz = wl.block_size
        for i, length in enumerate(wl.context_lens):
            length = int(length)
            nblk = (length + bsz - 1) // bsz
            ids = tables[i, :nblk].long()
            for src, dst in ((kc, kcont), (vc, vcont)):
                dst[i, :, :length] = src.index_select(0, ids).permute(1, 0, 2, 3).reshape(
                    h, nblk * bsz, d)[:, :length]
        torch.cuda.synchronize()

    def contig_step(o, q_, lens_):
        binding.pa_decode_contiguous(o, q_, kcont, vcont, lens_, mcl, wl.scale, ws, stream=stream)

    def grouped_step(o, q_, tables_, lens_, gs_, pl_):
        binding.pa_decode_grouped(o, q_, kc, vc, tables_, lens_, mcl, gs_, pl_, max_group,
                                  wl.scale, gws, stream=stream)

    def append_step(o, q_, key_, value_, slots_, tables_, lens_):
        if int8:
            binding.pa_decode_append_int8(o, q_, key_, value_, kc, vc, kp, vp, slots_, tables_,
                                          lens_, mcl, wl.scale, ws, stream=stream)
        else:
            binding.pa_decode_append(o, q_, key_, value_, kc, vc, slots_, tables_, lens_, mcl,
                                     wl.scale, ws, stream=stream)

    def step(ev_pair=None):
        if pairs is not None and not decode_only:
            copy_step()
        if not fused and not decode_only:
            write_step(key, value, slots)
        if ev_pair is not None:
            ev_pair[0].record(stream)
        if contig:
            contig_step(out, q, lens)
        elif grouped:
            grouped_step(out, q, tables, lens, d_gs, d_pl)
        elif fused:
            append_step(out, q, key, value, slots, tables, lens)
        else:
            decode_step(out, q, tables, lens)
        if ev_pair is not None:
            ev_pair[1].record(stream)

    launches_per_step = ((4 if grouped else 1) if decode_only else
                         (1 if fused else 2) + ((4 if int8 else 1) if pairs is not None else 0)
                         + (3 if grouped else 0))
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    assert binding.pa_get_last_device_error() == 0

    sampler = ClockSampler(local).start()
    # a step of one call (one launch, or the decode alone) is timed as K
    # back-to-back calls between two events (the region's mean is that call's
    # mean duration, gaps included); a step of several calls brackets each
    # decode with its own events
    single_launch = launches_per_step == 1 or decode_only
    evs = [None if single_launch else
           (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    start.record(stream)
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    w1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    sampler.stop()
    ms = start.elapsed_time(end)
    decode_ms = ([ms / args.steps] * args.steps if single_launch
                 else [a.elapsed_time(z) for a, z in evs])
    assert binding.pa_get_last_device_error() == 0

    # end to end: each step's inputs (q, the new tokens' K/V, slots, block
    # tables, context lengths) leave pinned host memory and out comes back to
    # it, pipelined with the decode; the KV pool stays resident.
    def decode_from(views, o):
        d_q, d_key, d_value, d_slots, d_tables, d_lens = views[:6]
        if pairs is not None and not decode_only:
            copy_step()
        if contig:
            contig_step(o, d_q, d_lens)
        elif decode_only and grouped:
            grouped_step(o, d_q, d_tables, d_lens, views[6], views[7])
        elif decode_only:
            decode_step(o, d_q, d_tables, d_lens)
        elif grouped:
            write_step(d_key, d_value, d_slots)
            grouped_step(o, d_q, d_tables, d_lens, views[6], views[7])
        elif fused:
            append_step(o, d_q, d_key, d_value, d_slots, d_tables, d_lens)
        else:
            write_step(d_key, d_value, d_slots)
            decode_step(o, d_q, d_tables, d_lens)

    e2e_parts = [q, key, value, slots, tables, lens] + ([d_gs, d_pl] if grouped else [])
    if decode_only:  # the step's inputs: q, (tables,) context lengths (, groups)
        e2e_parts = ([q, key[:1], value[:1], slots[:1], tables if not contig else tables[:1], lens]
                     + ([d_gs, d_pl] if grouped else []))
    e2e_ms, h2d, d2h = pipelined_e2e(e2e_parts, out, decode_from, stream, args.warmup, args.steps,
                                     world)
    assert binding.pa_get_last_device_error() == 0

    dec_bytes = (accounting.decode_bytes_int8(wl.context_lens, h, d) if int8
                 else accounting.decode_bytes(wl.context_lens, h, d))
    # aliased blocks are read once from DRAM and then hit L2: the roofline uses
    # the bytes DRAM must deliver (each physical row once)
    roof_bytes = dec_bytes
    if wl.alias_block_tables is not None and not int8:
        roof_bytes = accounting.decode_unique_bytes(wl.block_tables, wl.context_lens, h, d,
                                                    wl.block_size)
    if fused:  # the fused launch also writes each new K and V row to the cache
        roof_bytes += 2 * b * h * (d + 8) if int8 else 2 * b * h * d * 2
    step_bytes = dec_bytes + (0 if decode_only else
                              b * h * (2 * d * 2 + 2 * (d + 8)) if int8
                              else accounting.cache_write_bytes(b, h, d))
    if pairs is not None and not decode_only:
        step_bytes += accounting.copy_blocks_bytes(len(wl.copy_pairs), h, d, wl.block_size)

    # max over ranks of the device-timed regions; totals over ranks
    (ms, e2e_ms), (total_bytes, total_units) = reduce_over_ranks(
        [ms, e2e_ms], [step_bytes, b * h], dev)

    result = None
    if rank == 0:
        peak, peak_kind = _peak_hbm()
        mean_dec_ms = statistics.fmean(decode_ms)
        achieved = roof_bytes / (mean_dec_ms * 1e-3) / 1e9
        clocks = sampler.summary(w0, w1)
        desc = _workload_desc(wl, cfg)
        kv_bytes = dec_bytes
        desc.update({
            "step": "pa_decode_contiguous (K / V [B, H, Lmax, D], no block table)" if contig else
                    (f"pa_decode_grouped ({len(wl.prefix_lens)} groups, prefixes of "
                     f"{int(wl.prefix_lens[0])} tokens; blocks copied and newest tokens written "
                     f"before timing)" if grouped else
                     "pa_decode (the newest tokens written before timing)") if decode_only else
                    ("pa_copy_blocks + " if pairs is not None else "")
                    + (f"pa_reshape_and_cache({b} tokens) + pa_decode_grouped "
                       f"({len(wl.prefix_lens)} groups, prefixes of {int(wl.prefix_lens[0])} tokens)"
                       if grouped else
                       f"pa_decode_append{'_int8' if int8 else ''} (cache write of {b} tokens "
                       f"fused into the decode)"
                       if fused else f"pa_reshape_and_cache({b} tokens) + pa_decode"),
            "l2": f"inputs larger than L2: {kv_bytes / 1e9:.2f} GB of K/V read per step "
                  f"vs {L2_BYTES / 2**20:.0f} MiB L2 (no flush)",
            "parallelism": f"dp{world} (independent batches per GPU)",
            "placement": args.placement,
            "layout": args.layout,
            "kv_cache": ("int8 codes + fp32 (s, z) per row" if int8 else "fp16"),
        })
        result = {
            "metric": METRIC,
            "value": total_bytes * args.steps / (ms * 1e-3) / 1e9,
            "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "storage_dtype": "u8" if int8 else "f16", "data": "synthetic",
            "config": desc,
            "seq_heads_per_s": total_units * args.steps / (ms * 1e-3),
            "hbm_frac": achieved / peak,
            "decode_us_mean": mean_dec_ms * 1e3,
            "launch_timing": ("events around the K back-to-back calls of the timed region"
                              if single_launch else "events around each decode launch"),
            **({} if single_launch else {
                "decode_us_median": statistics.median(decode_ms) * 1e3,
                "decode_us_max": max(decode_ms) * 1e3,
                "decode_us_argmax": int(np.argmax(decode_ms))}),
            "roofline": {
                "kernel": ("pa_decode_grouped (set-up, grouped_decode_kernel, paged_decode_kernel "
                           "over the tails, merge)" if grouped else
                           "paged_decode_kernel<contiguous>" if contig else
                           "paged_decode_kernel" + ("<int8>" if int8 else "")), "bound": "hbm",
                "achieved": achieved,
                "peak": peak, "peak_kind": f"{peak_kind} (hbm_gbs)", "unit": "GB/s",
                "frac": achieved / peak,
                "traffic": None if int8 or contig else _recorded_traffic(
                    desc["workload"], "pa_decode_grouped" if grouped else
                    "pa_decode_append" if fused else "pa_decode",
                    "grouped" if grouped else "decode"),
                "algorithmic_bytes_per_launch": roof_bytes,
                "logical_bytes_per_launch": dec_bytes,
            },
            "e2e": {"value": total_bytes * args.steps / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "copies": "pinned host <-> device every step, pipelined with the decode "
                              "(two staging buffers and outputs, separate copy streams)",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / args.steps},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        if cpu_sample is not None:
            result["cpu_baseline"] = cpu_baseline(wl, cpu_sample)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if result is not None:
        print(json.dumps(result), flush=True)
    return 0


PREFILL_METRIC = "paged prefill attention: algorithmic TFLOP/s (causal; % of tensor peak)"


def _prefill_flops(lens, n_new, num_heads, head_dim):
    """Algorithmic FLOPs of causal multi-query attention: a new token at
    position p attends to p + 1 cached tokens, 2 D multiply-adds each for
    q . K and for P V."""
    total = 0.0
    for length, n in zip(lens, n_new):
        pos = np.arange(length - n, length, dtype=np.float64)
        total += float((pos + 1).sum())
    return total * num_heads * 4 * head_dim


def prefill_cpu_baseline(q, key, value, n, length, num_heads, head_dim, block_size, scale,
                         target_s: float = 10.0):
    """The oracle's paged prefill as it stands, on the host cores, on a bounded
    sample of the same workload: the first prompt, its first heads (about
    target_s seconds); TFLOP/s over the sample's algorithmic FLOPs."""
    import oracle
    nblk = length // block_size

    def sample(heads):
        k = key[:length, :heads].reshape(nblk, block_size, heads, head_dim).transpose(0, 2, 1, 3)
        v = value[:length, :heads].reshape(nblk, block_size, heads, head_dim).transpose(0, 2, 1, 3)
        return (np.ascontiguousarray(q[:n, :heads]), np.ascontiguousarray(k),
                np.ascontiguousarray(v), np.arange(nblk, dtype=np.int32)[None],
                np.array([length], np.int32), np.array([0, n], np.int32))

    def run(heads):
        a = sample(heads)
        t0 = time.perf_counter()
        oracle.paged_prefill(*a, scale)
        return time.perf_counter() - t0

    per_head = max(run(1), 1e-4)
    heads = int(max(1, min(num_heads, target_s / per_head)))
    t = run(heads)
    flops = _prefill_flops([length], [n], heads, head_dim)
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"prompt 0 of the batch ({n} new tokens), {heads} of {num_heads} heads "
                      f"(attention only, fp64), {t:.1f} s wall"}


def run_prefill(args):
    """One step = the prefill of a batch of prompts through the paged cache:
    pa_reshape_and_cache of every prompt token's K/V into its slot, then
    pa_prefill (causal multi-query attention on the tensor cores)."""
    import torch
    import torch.distributed as dist
    from paged_kv_cache_481_b200 import binding

    world, rank, local = _init_ranks(args)
    dev = torch.device("cuda", local)

    b, length, h, d = args.prompts, args.prompt_len, 40, 128
    bs = args.block_size or 16
    n = args.new_tokens or length
    if length % bs:
        raise SystemExit("--prompt-len must be a multiple of the block size")
    if not 0 < n <= length:
        raise SystemExit("--new-tokens must be in [1, --prompt-len]")
    seed = 7 + 100 * rank
    rng = np.random.default_rng(seed)
    gen = torch.Generator().manual_seed(seed)
    tokens = b * n
    # inputs drawn on the host (seeded), as the oracle sample needs them there too;
    # K / V of every context token, of which the last n per sequence are new
    q_h = torch.randn((tokens, h, d), generator=gen).half()
    key_h = torch.randn((b * length, h, d), generator=gen).half()
    value_h = torch.randn((b * length, h, d), generator=gen).half()
    per_seq = length // bs
    nb = b * per_seq
    tables_h = rng.permutation(nb).astype(np.int32).reshape(b, per_seq)
    pos = np.arange(length)
    slots_all = np.stack([tables_h[i, pos // bs].astype(np.int64) * bs + pos % bs
                          for i in range(b)])
    slots_h = np.ascontiguousarray(slots_all[:, length - n:]).reshape(-1)
    scale = d ** -0.5
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = prefill_cpu_baseline(q_h.numpy(), key_h.numpy(), value_h.numpy(), n, length, h, d,
                                   bs, scale, target_s=args.cpu_seconds)

    q = q_h.to(dev)
    key = key_h.view(b, length, h, d)[:, length - n:].reshape(tokens, h, d).to(dev)
    value = value_h.view(b, length, h, d)[:, length - n:].reshape(tokens, h, d).to(dev)
    slots = torch.from_numpy(slots_h).to(dev)
    tables = torch.from_numpy(tables_h).to(dev)
    lens = torch.full((b,), length, dtype=torch.int32, device=dev)
    qsl = torch.arange(b + 1, dtype=torch.int32, device=dev) * n
    kc = torch.zeros((nb, h, bs, d), dtype=torch.float16, device=dev)
    vc = torch.zeros_like(kc)
    if n < length:  # the earlier chunks' K / V are in the cache before the step
        binding.pa_reshape_and_cache(key_h.to(dev), value_h.to(dev), kc, vc,
                                     torch.from_numpy(slots_all.reshape(-1)).to(dev))
        torch.cuda.synchronize()
    out = torch.empty_like(q)
    stream = torch.cuda.Stream(device=dev)
    flops = _prefill_flops([length] * b, [n] * b, h, d)

    def step(views, o, ev=None):
        d_q, d_key, d_value, d_slots, d_tables, d_lens, d_qsl = views
        binding.pa_reshape_and_cache(d_key, d_value, kc, vc, d_slots, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        binding.pa_prefill(o, d_q, kc, vc, d_tables, d_lens, length, d_qsl, n, scale,
                           stream=stream)
        if ev is not None:
            ev[1].record(stream)

    views = [q, key, value, slots, tables, lens, qsl]
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step(views, out)
    torch.cuda.synchronize()
    assert binding.pa_get_last_device_error() == 0
    sampler = ClockSampler(local).start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    start.record(stream)
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            step(views, out, evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    w1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    sampler.stop()
    ms = start.elapsed_time(end)
    launch_ms = [a.elapsed_time(z) for a, z in evs]
    assert binding.pa_get_last_device_error() == 0

    e2e_ms, h2d, d2h = pipelined_e2e(views, out, step, stream, args.warmup, args.steps, world)
    assert binding.pa_get_last_device_error() == 0

    (ms, e2e_ms), (total_flops,) = reduce_over_ranks([ms, e2e_ms], [flops], dev)
    result = None
    if rank == 0:
        try:
            with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
                pk = json.load(f)
            peak, peak_sus, kind = float(pk["bf16_tflops"]), float(pk["bf16_tflops_sustained"]), "measured"
        except Exception:
            peak, peak_sus, kind = 1590.0, 1400.0, "fallback"
        mean_ms = statistics.fmean(launch_ms)
        achieved = flops / (mean_ms * 1e-3) / 1e12
        if n == length:
            workload = (f"13B prefill: {b} prompts x {length} tokens, H={h} D={d} bs={bs}, "
                        f"shuffled blocks, causal")
        else:
            workload = (f"13B chunked prefill: {b} sequences, {n} new of {length} tokens, "
                        f"H={h} D={d} bs={bs}, shuffled blocks, causal")
        result = {
            "metric": PREFILL_METRIC, "value": total_flops * args.steps / (ms * 1e-3) / 1e12,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": workload,
                       "num_seqs": b, "prompt_len": length, "new_tokens": n,
                       "num_heads": h, "head_dim": d,
                       "block_size": bs, "seed": seed,
                       "step": f"pa_reshape_and_cache({tokens} tokens) + pa_prefill",
                       "l2": f"K/V {2 * nb * h * bs * d * 2 / 1e9:.2f} GB and q/out "
                             f"{2 * tokens * h * d * 2 / 1e9:.2f} GB per step vs "
                             f"{L2_BYTES / 2**20:.0f} MiB L2 (no flush)",
                       "parallelism": f"dp{world} (independent prompts per GPU)"},
            "prefill_us_mean": mean_ms * 1e3,
            "roofline": {"kernel": "paged_prefill_kernel", "bound": "tensor",
                         "achieved": achieved, "peak": peak,
                         "peak_kind": f"{kind} (bf16_tflops, burst; fp16 runs at the bf16 rate)",
                         "peak_sustained": peak_sus, "unit": "TFLOP/s", "frac": achieved / peak,
                         "traffic": _recorded_traffic(workload, "pa_prefill", "prefill"),
                         "algorithmic_flops_per_launch": flops},
            "e2e": {"value": total_flops * args.steps / (e2e_ms * 1e-3) / 1e12,
                    "unit": "TFLOP/s",
                    "copies": "pinned host <-> device every step (q, prompt K/V, slots, tables), "
                              "pipelined with the step (two staging buffers and outputs)",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / args.steps},
            "gpu_launches": 2 * args.steps,
            "clocks": sampler.summary(w0, w1),
        }
        if cpu is not None:
            result["cpu_baseline"] = cpu
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if result is not None:
        print(json.dumps(result), flush=True)
    return 0


BLOCK_OP_METRIC = {
    "cache-write": "pa_reshape_and_cache: GB/s (new K/V read + cache rows written; % of HBM peak)",
    "copy-blocks": "pa_copy_blocks: GB/s (blocks read + written; % of HBM peak)",
    "swap": "pa_swap_blocks: GB/s over the host link (% of a plain copy of the same bytes)",
}


def _graph_ms(launch, stream, warmup, steps):
    """Device time of `steps` calls launch(0), ..., launch(steps - 1) captured
    in one CUDA graph and replayed once.  These kernels run for a few
    microseconds, less than a host launch takes, so issuing them one by one
    would time the host; the replay times the device.  Warm-up: one replay
    of a graph of `warmup` calls."""
    import torch

    def capture(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                launch(i, stream)
        return g

    with torch.cuda.stream(stream):
        for i in range(3):  # outside any capture: the library's first launches
            launch(i, stream)
    torch.cuda.synchronize()
    warm, timed = capture(warmup), capture(steps)
    with torch.cuda.stream(stream):  # a graph replays on the current stream
        warm.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        timed.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def _host_fed_ms(parts, launch, stream, warmup, steps):
    """The same calls issued one by one through the public API, each step's
    inputs (`parts`) copied from pinned host memory just before it on the
    launching stream; returns (ms for `steps` steps, h2d bytes per step)."""
    import torch
    hosts = [p.cpu().pin_memory() for p in parts]
    devs = [torch.empty_like(p) for p in parts]

    def one(i):
        with torch.cuda.stream(stream):
            for h_, d_ in zip(hosts, devs):
                d_.copy_(h_, non_blocking=True)
            launch(devs, stream)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        one(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1), sum(p.numel() * p.element_size() for p in parts)


def run_block_ops(args):
    """The cache-management entry points, one JSON line each.

    cache-write: one decode step's pa_reshape_and_cache of --tokens new
    tokens (13B shapes, H=40, D=128, bs=16) into random slots of an 8192-block
    pool.  copy-blocks: pa_copy_blocks of --pairs copy-on-write pairs.  A
    step's inputs (new K/V and slots; the pairs) rotate through enough
    distinct sets that they and the rows they touch do not stay in L2 from
    one step to the next.  Timed as a CUDA graph of the K calls.

    swap: pa_swap_blocks of --swap-blocks blocks (160 KB each at 13B shapes)
    between the device pool and a page-locked host pool, in the direction
    --direction, to a permuted set of blocks, against a plain copy of the
    same number of contiguous bytes over the same link; events per call."""
    import torch
    import torch.distributed as dist
    from paged_kv_cache_481_b200 import accounting, binding

    world, rank, local = _init_ranks(args)
    dev = torch.device("cuda", local)
    h, d, bs = 40, 128, args.block_size or 16
    seed = 11 + 100 * rank
    g = torch.Generator(device=dev).manual_seed(seed)
    stream = torch.cuda.Stream(device=dev)
    peak_hbm, peak_kind = _peak_hbm()
    sampler = ClockSampler(local).start()
    extra = {}
    if args.path == "swap":
        nblk = args.swap_blocks
        pool = torch.randn((nblk, h, bs, d), generator=g, device=dev).half()
        host = torch.empty((nblk, h, bs, d), dtype=torch.float16).pin_memory()
        perm = torch.randperm(nblk, generator=g, device=dev)
        pairs = torch.stack([torch.arange(nblk, device=dev), perm], 1).contiguous()
        src, dst = (pool, host) if args.direction == "d2h" else (host, pool)
        nbytes = pool.numel() * pool.element_size()

        def timed(fn):
            with torch.cuda.stream(stream):
                for _ in range(args.warmup):
                    fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            with torch.cuda.stream(stream):
                for _ in range(args.steps):
                    fn()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1)

        if world > 1:
            dist.barrier()
        w0 = time.perf_counter()
        ms = timed(lambda: binding.pa_swap_blocks(src, dst, pairs, stream=stream))
        w1 = time.perf_counter()
        ms_link = timed(lambda: dst.copy_(src, non_blocking=True))
        unit_bytes = nbytes
        launches = args.steps
        workload = (f"13B swap {'device -> host' if args.direction == 'd2h' else 'host -> device'}"
                    f": {nblk} blocks of {nbytes // nblk // 1024} KB (H={h} D={d} bs={bs}), "
                    f"permuted destination blocks")
        link_gbs = nbytes * args.steps / (ms_link * 1e-3) / 1e9
        roof = {"kernel": "copy_blocks_kernel (host pool)", "bound": "link",
                "achieved": nbytes * args.steps / (ms * 1e-3) / 1e9, "peak": link_gbs,
                "peak_kind": "measured in this run: a plain cudaMemcpyAsync of the same bytes "
                             "over the same link (torch copy_)",
                "unit": "GB/s", "traffic": None}
        roof["frac"] = roof["achieved"] / roof["peak"]
        config = {"workload": workload, "blocks": nblk, "block_bytes": nbytes // nblk,
                  "direction": args.direction, "seed": seed,
                  "l2": "host link bound; the pool (one copy per step) is "
                        f"{nbytes / 2**20:.0f} MiB vs {L2_BYTES / 2**20:.0f} MiB L2"}
        e2e = {"value": roof["achieved"], "unit": "GB/s",
               "note": "the call is itself the host <-> device transfer",
               "h2d_bytes_per_step": nbytes if args.direction == "h2d" else 0,
               "d2h_bytes_per_step": nbytes if args.direction == "d2h" else 0}
    else:
        nb = 8192
        kc = torch.randn((nb, h, bs, d), generator=g, device=dev).half()
        vc = torch.randn_like(kc)
        if args.path == "cache-write":
            n = args.tokens
            unit_bytes = accounting.cache_write_bytes(n, h, d)
            # distinct sets of inputs and target rows: 2x L2 of inputs, at most 1024
            sets = int(min(1024, max(8, math.ceil(2 * L2_BYTES / (4 * n * h * d)))))
            key = torch.randn((sets, n, h, d), generator=g, device=dev).half()
            value = torch.randn_like(key)
            slots = (torch.randint(0, nb, (sets, n), generator=g, device=dev) * bs
                     + torch.randint(0, bs, (sets, n), generator=g, device=dev)).long()

            def launch(i, st):
                j = i % sets
                binding.pa_reshape_and_cache(key[j], value[j], kc, vc, slots[j], stream=st)

            parts = [key[0], value[0], slots[0]]

            def fed(views, st):
                binding.pa_reshape_and_cache(views[0], views[1], kc, vc, views[2], stream=st)

            kernel = "reshape_and_cache_kernel"
            workload = (f"13B decode-step cache write: {n} new tokens (H={h} D={d} bs={bs}) "
                        f"into random slots of an {nb}-block pool")
            config_extra = {"tokens": n, "input_sets": sets}
        else:
            p = args.pairs
            unit_bytes = accounting.copy_blocks_bytes(p, h, d, bs)
            sets = int(min(1024, max(4, math.ceil(2 * L2_BYTES / (unit_bytes / 2)))))
            sets = min(sets, nb // (2 * p))
            pairs = torch.stack([torch.randperm(nb, generator=g, device=dev)[:2 * p].view(p, 2)
                                 for _ in range(sets)]).long().contiguous()

            def launch(i, st):
                binding.pa_copy_blocks(kc, vc, pairs[i % sets], stream=st)

            parts = [pairs[0]]

            def fed(views, st):
                binding.pa_copy_blocks(kc, vc, views[0], stream=st)

            kernel = "copy_blocks_kernel"
            workload = (f"13B copy-on-write: {p} block pairs (H={h} D={d} bs={bs}, K and V) "
                        f"in an {nb}-block pool")
            config_extra = {"pairs": p, "pair_sets": sets}
        if world > 1:
            dist.barrier()
        w0 = time.perf_counter()
        ms = _graph_ms(launch, stream, args.warmup, args.steps)
        w1 = time.perf_counter()
        e2e_ms, h2d = _host_fed_ms(parts, fed, stream, args.warmup, args.steps)
        launches = args.steps
        achieved = unit_bytes * args.steps / (ms * 1e-3) / 1e9
        roof = {"kernel": kernel, "bound": "hbm", "achieved": achieved, "peak": peak_hbm,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak_hbm,
                "traffic": None, "algorithmic_bytes_per_launch": unit_bytes}
        config = {"workload": workload, "num_heads": h, "head_dim": d, "block_size": bs,
                  "seed": seed, **config_extra,
                  "timing": f"one CUDA graph of the {args.steps} calls, replayed once",
                  "l2": f"inputs rotate through {sets} distinct sets (no flush)"}
        e2e = {"value": unit_bytes * args.steps / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "copies": "the step's inputs from pinned host memory each step, calls issued "
                         "one by one from the host",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 0,
               "ms_per_step": e2e_ms / args.steps}
        extra["us_per_call"] = ms * 1e3 / args.steps
    sampler.stop()
    assert binding.pa_get_last_device_error() == 0
    (ms,), (total,) = reduce_over_ranks([ms], [unit_bytes * args.steps], dev)
    result = None
    if rank == 0:
        result = {
            "metric": BLOCK_OP_METRIC[args.path], "value": total / (ms * 1e-3) / 1e9,
            "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic", "config": config,
            **extra, "roofline": roof, "e2e": e2e, "gpu_launches": launches,
            "clocks": sampler.summary(w0, w1),
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if result is not None:
        print(json.dumps(result), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--block-size", type=int, default=None)
    ap.add_argument("--placement", choices=["shuffled", "sequential"], default="shuffled",
                    help="physical block placement (sequential = contiguous-cache baseline)")
    ap.add_argument("--kv-dtype", choices=["fp16", "int8"], default="fp16",
                    help="KV cache storage (int8 = 8-bit affine codes per row)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="time the cache write and the decode as two launches")
    ap.add_argument("--layout", choices=["paged", "contiguous"], default="paged",
                    help="contiguous: the same decode over K / V [B, H, Lmax, D] with no block "
                         "table (the baseline for the indirection's cost); times the decode alone")
    ap.add_argument("--decode-only", action="store_true",
                    help="time the decode alone, K back-to-back calls (pa_decode; pa_decode_grouped "
                         "for the shared-prefix workload; the newest tokens written and the blocks "
                         "copied before timing)")
    ap.add_argument("--no-grouped", action="store_true",
                    help="shared-prefix workload: plain pa_decode instead of pa_decode_grouped")
    ap.add_argument("--path", choices=["decode", "prefill", "cache-write", "copy-blocks", "swap"],
                    default="decode",
                    help="prefill: the prompt cache write + pa_prefill step instead of decode; "
                         "cache-write / copy-blocks / swap: those entry points alone")
    ap.add_argument("--prompts", type=int, default=8, help="prefill: prompts per step")
    ap.add_argument("--prompt-len", type=int, default=2048, help="prefill: tokens per prompt")
    ap.add_argument("--new-tokens", type=int, default=None,
                    help="prefill: new tokens per sequence (the last ones of its --prompt-len "
                         "context; the earlier ones already cached): chunked prefill")
    ap.add_argument("--tokens", type=int, default=256, help="cache-write: new tokens per step")
    ap.add_argument("--pairs", type=int, default=64, help="copy-blocks: block pairs per step")
    ap.add_argument("--swap-blocks", type=int, default=1024, help="swap: blocks per step")
    ap.add_argument("--direction", choices=["d2h", "h2d"], default="d2h", help="swap direction")
    ap.add_argument("--cpu-threads", type=int, default=None,
                    help="host threads for the oracle (CPU baseline / reference arm); default all")
    args = ap.parse_args(argv)
    if args.cpu_threads:
        # read by the oracle's OpenMP runtime when the oracle library first loads
        os.environ["OMP_NUM_THREADS"] = str(args.cpu_threads)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.kv_dtype == "int8" and args.workload == 4:
        raise SystemExit("--kv-dtype int8 is not built for the shared-prefix workload (4): "
                         "its int8 pool would need every aliased block's tokens once")
    if args.impl == "reference":
        if args.path != "decode":
            raise SystemExit("--impl reference times the decode path")
        return run_reference(args)
    if args.path == "prefill":
        return run_prefill(args)
    if args.path in BLOCK_OP_METRIC:
        return run_block_ops(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
