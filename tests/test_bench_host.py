"""Host-side checks of bench.py: the multi-rank (replica) reduction under a
2-rank gloo process group on CPU, and the reference arm's rank behaviour."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports times (r + 1, 10 r, 5): the slowest rank sets each one
        vals = bench.max_over_ranks([rank + 1.0, 10.0 * rank, 5.0], world, "cpu")
        out[rank] = vals
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        assert out[0] == out[1] == [2.0, 10.0, 5.0]


def test_job_throughput_counts_every_rank():
    # 4096 tokens per rank and step, 3 steps, 2 ranks, slowest rank 1.5 ms total
    assert bench.job_throughput(4096, 2, 3, 1.5) == pytest.approx(4096 * 2 * 3 / 1.5e-3)
    assert bench.max_over_ranks([1.0, 2.0], 1) == [1.0, 2.0]


def test_reference_arm_other_ranks_exit_silently():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--ref-heads", "1"], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["higher_is_better"] is True and line["unit"] == "tokens/s"


def test_prefill_shape_option():
    import argparse
    from gated_delta_rule_124_b200 import workloads as wl
    args = argparse.Namespace(prefill_shape="2,128,3", prefill_config=1)
    pc = bench.prefill_case(wl, args)
    assert (pc.B, pc.T, pc.H, pc.dk, pc.dv, pc.chunk, pc.dtype) == (2, 128, 3, 128, 128, 64,
                                                                     "bf16")
    assert pc.cu_seqlens is None and pc.name == "prefill: B=2 H=3 T=128 d=128 C=64 bf16"
    args = argparse.Namespace(prefill_shape=None, prefill_config=1)
    assert bench.prefill_case(wl, args).name == wl.prefill_config(1).name


def test_measured_traffic_is_hash_guarded(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    import hashlib
    sha = hashlib.sha1(b"kernel v1").hexdigest()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {("kern", "wl"): ("k.cu", sha, 123)})
    assert bench.measured_traffic("kern", "wl") == 123
    assert bench.measured_traffic("kern", "other workload") is None
    src.write_text("kernel v2")  # the kernel changed since the capture
    assert bench.measured_traffic("kern", "wl") is None
