"""Host-side checks of bench.py: the CPU reference arm prints one JSON line with
the contract's keys, alone and under a 2-rank gloo launch (rank 0 prints,
rank 1 exits cleanly), and the cross-rank reductions take the maximum/sum."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
        "cpu_baseline", "e2e"}


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _json_lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def test_reference_arm_single_process():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_two_ranks_gloo():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                        "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
                        "--gpus", "2", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=900, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["impl"] == "reference"


def _reduce_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    out[rank] = (bench.max_over_ranks(1.0 + rank, world), bench.sum_over_ranks(10.0, world))
    bench.barrier(world)
    torch.distributed.destroy_process_group()


def test_cross_rank_reductions_gloo():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_reduce_worker, args=(2, _free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    assert out[0] == (2.0, 20.0) and out[1] == (2.0, 20.0)


def test_traffic_figure_is_keyed_to_workload_and_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed counters only for the workload they were
    taken on and while the kernel source still hashes to the recorded value."""
    sys.path.insert(0, ROOT)
    import hashlib
    import bench
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel source\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    fig = tmp_path / "traffic.json"
    fig.write_text(json.dumps({"workload": "wl_a", "source_sha256": sha,
                               "dram_bytes_per_launch_full_size": 123}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(fig))
    monkeypatch.setattr(bench, "TC_SOURCE", str(src))
    assert bench.traffic_from_profile("wl_a") == 123.0
    assert bench.traffic_from_profile("wl_b") is None          # another workload
    src.write_text("// kernel source, changed\n")
    assert bench.traffic_from_profile("wl_a") is None          # the kernel changed since
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.traffic_from_profile("wl_a") is None


def test_committed_traffic_figure_matches_the_current_kernel():
    """The figure under profiles/ belongs to the kernel source in the tree."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.traffic_from_profile(bench.HEADLINE_6P7B) is not None
