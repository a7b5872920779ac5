"""The benchmark's multi-rank host logic on CPU with gloo, world size 2:
per-rank batches (weak scaling, no data-path collective) and the
max-over-ranks timing / sum-over-ranks work reduction."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "took" 10 + r ms and did 100 * (r + 1) bytes of work
        mx, sm = bench.reduce_over_ranks([10.0 + rank, 1.0], [100.0 * (rank + 1), 7.0], "cpu")
        from paged_kv_cache_481_b200 import workloads
        wl = workloads.make_workload(1, seed=bench.rank_seed(1, rank))
        q.put((rank, mx, sm, wl.q.numpy().copy(), wl.num_seqs))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_shard():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res.sort(key=lambda x: x[0])
    for _, mx, sm, _, _ in res:
        assert mx == [11.0, 1.0]               # max over ranks
        assert sm == [300.0, 14.0]             # sum over ranks
    # weak scaling: same per-rank batch size, different data per rank
    assert res[0][4] == res[1][4]
    assert not np.array_equal(res[0][3], res[1][3])


def test_single_process_reduction_is_identity():
    mx, sm = bench.reduce_over_ranks([3.0, 4.0], [5.0], "cpu")
    assert mx == [3.0, 4.0] and sm == [5.0]


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_one_json_line():
    r = _run_bench(["--impl", "reference", "--workload", "1", "--steps", "3", "--warmup", "3"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--workload", "1", "--steps", "3", "--warmup", "3"],
                   {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    r = _run_bench(["--impl", "reference", "--workload", "1", "--steps", "3", "--warmup", "2"])
    assert r.returncode != 0


def test_cpu_baselines_of_the_other_paths():
    """The oracle legs of `bench.py --kv-dtype int8` and `--path prefill` on
    tiny inputs: a positive rate over the sample they describe."""
    from paged_kv_cache_481_b200 import workloads
    wl = workloads.make_workload(1, keep_tokens=True)
    sample = bench.cpu_baseline_sample(wl, target_s=0.05, int8=True)
    assert sample["int8"] and sample["kc"].dtype == np.uint8 and sample["kp"].shape[-1] == 2
    line = bench.cpu_baseline(wl, sample)
    assert line["kind"] == "oracle" and line["value"] > 0 and "int8" in line["sample"]
    rng = np.random.default_rng(0)
    n, h, d, bs = 64, 2, 128, 16
    q, k, v = (rng.standard_normal((n, h, d)).astype(np.float16) for _ in range(3))
    line = bench.prefill_cpu_baseline(q, k, v, n, n, h, d, bs, d ** -0.5, target_s=0.05)
    assert line["unit"] == "TFLOP/s" and line["value"] > 0 and line["cores"] >= 1
    assert bench._prefill_flops([n], [n], h, d) == 4 * d * h * n * (n + 1) / 2
    # chunked prefill (--new-tokens): the last 16 of 64 context tokens are new;
    # token p of them attends to p + 1 cached tokens
    m = 16
    line = bench.prefill_cpu_baseline(q[:m], k, v, m, n, h, d, bs, d ** -0.5, target_s=0.05)
    assert line["value"] > 0 and f"({m} new tokens)" in line["sample"]
    assert bench._prefill_flops([n], [m], h, d) == 4 * d * h * sum(p + 1 for p in range(n - m, n))


def test_secondary_bench_paths_parse_and_refuse_bad_combinations():
    """The cache-write / copy-blocks / swap and chunked-prefill options parse,
    and combinations the bench does not measure are refused before any GPU
    work."""
    ap_help = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"],
                             capture_output=True, text=True, timeout=120)
    assert ap_help.returncode == 0
    for opt in ("cache-write", "copy-blocks", "swap", "--new-tokens", "--direction", "--decode-only"):
        assert opt in ap_help.stdout
    r = _run_bench(["--impl", "reference", "--path", "swap", "--steps", "3", "--warmup", "3"])
    assert r.returncode != 0 and "times the decode path" in (r.stdout + r.stderr)
    r = _run_bench(["--kv-dtype", "int8", "--workload", "4", "--steps", "3", "--warmup", "3"])
    assert r.returncode != 0 and "int8" in (r.stdout + r.stderr)
