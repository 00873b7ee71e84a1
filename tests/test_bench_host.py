"""Host-side logic of bench.py's multi-GPU run (weak scaling, no data-path collective),
exercised on two gloo ranks on the CPU."""
import json
import os
import socket
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_max_and_weak_scaling(tmp_path):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(HERE, "bench_host_worker.py"), str(tmp_path)]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=240)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    outs = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(2)]
    for o in outs:
        assert o["world"] == 2
        assert o["slowest"] == 15.0  # the max over ranks, seen by every rank
        # 2 ranks x 4096 tokens in the slowest rank's 0.15 ms per step
        assert o["value"] == pytest.approx(2 * 4096 / 0.15e-3)


def test_single_process_aggregate_is_identity():
    import torch
    assert bench.aggregate_max(3.5, torch.device("cpu")) == 3.5
    assert bench.job_tokens_per_s(1, 4096, 1.0) == pytest.approx(4096e3)


def test_reference_arm_other_ranks_do_no_work(capsys):
    class Args:
        steps, warmup, gpus = 2, 3, 2
    from bit_activation_linear_b200 import synth
    t = bench.run_reference(Args(), synth.WORKLOADS["wo_2048"], rank=1, world=2)
    assert t is None
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_line_on_rank0(capsys):
    class Args:
        steps, warmup, gpus = 1, 3, 1
    from bit_activation_linear_b200 import synth
    bench.run_reference(Args(), synth.WORKLOADS["tiny"], rank=0, world=1)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["value"] > 0 and line["config"]["workload"] == "tiny"
