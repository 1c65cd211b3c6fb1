"""Host-side logic of the benchmark: the slowest-rank timing over a 2-rank gloo group on
CPU, the whole-job throughput, the FLOP accounting, and the reference arm's contract."""
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
import synth  # noqa: E402


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(10.0 + 5.0 * rank, dist)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1000, 4, 5, 2000.0) == pytest.approx(1000 * 4 * 5 / 2.0)
    assert bench.max_over_ranks(3.5, None) == 3.5


def test_flop_counts_closed_form():
    # one sequence of 4 blocks of 128, D 64, 2 heads, top_k 3: closed forms by hand
    w = synth.Workload("f", [512], 2, 1, 64, 128, 3, seed=1)
    fl = bench.flop_counts(w, routed_rows=100)
    assert fl["past"] == 4 * 64 * 128 * 100
    own_keys = 4 * (128 * 129 // 2)  # every block: 1 + 2 + ... + 128 keys
    assert fl["own"] == 4 * 64 * 2 * own_keys
    gate_dots = 128 * (0 + 1 + 2 + 3)
    assert fl["gate"] == 2 * 64 * 2 * gate_dots


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "1", "--warmup", "0"],
                         env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_reference_arm_prints_its_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "1", "--warmup", "0", "--ref-seconds", "0.3"],
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_dense_causal_flops_closed_form():
    # two sequences of 3 and 5 tokens, D 8, 2 heads: 4 * D * H * (1+2+3 + 1+2+3+4+5)
    w = synth.Workload("d", [3, 5], 2, 1, 8, 128, 3, seed=1)
    assert bench.dense_causal_flops(w) == 4 * 8 * 2 * (6 + 15)


def test_reference_arm_reports_its_measured_step_and_the_same_config():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "2", "--warmup", "1", "--ref-seconds", "0.3"],
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    # the same workload description as the GPU arm prints
    assert line["config"] == bench.config_dict(synth.CONFIGS["tiny"], 1)
    # a step is one bounded sample: its measured length, not the extrapolated full pass
    assert 300.0 <= line["ms_per_step"] < 60_000.0
    assert line["ms_per_full_pass_extrapolated"] == pytest.approx(
        1e3 * synth.CONFIGS["tiny"].total_tokens / line["value"])
    assert line["cpu_baseline"]["value"] == line["value"] == line["e2e"]["value"]
