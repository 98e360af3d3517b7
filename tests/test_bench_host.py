"""Host-side logic of bench.py that runs on CPU: the max-over-ranks reduction with two gloo
ranks, the reference arm's rank handling, and the JSON contract of the reference line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r times (1 + r) ms and an end-to-end leg only on rank 0
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank, None], dist, "cpu")
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        assert out[r] == [2.0, 5.0, None]


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks([3.0, None], None, "cpu") == [3.0, None]


def _run_bench(extra_env, *args):
    env = dict(os.environ, **extra_env)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=env, timeout=600)


def test_reference_arm_non_zero_rank_exits_quietly():
    p = _run_bench({"WORLD_SIZE": "2", "RANK": "1"}, "--impl", "reference", "--steps", "1", "--warmup", "3",
                   "--ref-n", "4096")
    assert p.returncode == 0 and p.stdout.strip() == ""


def test_reference_arm_json_line():
    p = _run_bench({"WORLD_SIZE": "1", "RANK": "0"}, "--impl", "reference", "--steps", "2", "--warmup", "3",
                   "--ref-n", "8192")
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line
    assert line["metric"] == bench.METRIC and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cores"] == 1 and line["warmup"] >= 3


def test_workload_oracle_small_workloads():
    # the oracle leg of `bench.py --workload`: one step of the two small workloads end to end
    import numpy as np
    import oracle
    import synth
    n = 1 << 20
    g = [synth.flat_mixture(n, seed=0)]
    b = oracle.golomb_b_star(0.01)
    dense, outs = bench.workload_oracle("flat2e20", g, n, None, (1, 100), b)
    assert outs is None and np.count_nonzero(dense) == oracle.k_for(n, 1, 100)
    seg = synth.offsets(synth.mlp_layout())
    n = int(seg[-1])
    g = [synth.mlp_gradient(w, 0) for w in range(4)]
    dense, _ = bench.workload_oracle("mlp", g, n, seg, (1, 100), None)
    kept = sum(oracle.k_for(int(seg[t + 1] - seg[t]), 1, 100) for t in range(len(seg) - 1))
    assert kept <= np.count_nonzero(dense) <= 4 * kept


def test_reference_arm_with_momentum():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1", "--ref-n", "4096", "--momentum", "0.9"],
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0


def test_profile_hash_ignores_comments_only():
    """The pass-1 profile stays valid across comment edits and is invalidated by a code edit."""
    src = "// header\n__global__ void k(int* p) {  /* note */\n  p[0] = 1;  // store\n}\n"
    same = "// another header\n\n__global__ void k(int* p) {\n  p[0] = 1;\n}\n"
    other = "__global__ void k(int* p) {\n  p[0] = 2;\n}\n"
    assert bench.code_text(src) == bench.code_text(same)
    assert bench.code_text(src) != bench.code_text(other)
    assert len(bench.source_sha()) == 16
