"""The benchmark's multi-process plumbing (replicas, one process per device) on CPU ranks over
gloo: the max-over-ranks timing, the barrier, and the reference arm running on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        # each rank reports its own time; every rank must see the slowest one
        t = bench.max_over_ranks(dist, 10.0 + rank, dev)
        dist.barrier()
        out[rank] = t
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_world2():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert dict(out) == {0: 11.0, 1: 11.0}


def test_reference_arm_other_ranks_do_no_work():
    """Under torchrun the reference arm prints on rank 0 only; other ranks exit 0 silently."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_reference_arm_line_on_rank0():
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--layers", "1"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_committed_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    """The roofline's DRAM traffic is reported only while the warp-level kernel's sources hash to
    the value recorded with the capture: the committed tree matches, and any edit of one of those
    sources (a copy of the tree here) makes the number disappear."""
    import shutil
    sys.path.insert(0, ROOT)
    import bench
    assert bench.committed_traffic("qmm_warp_kernel_decode_chain") is not None
    assert bench.committed_traffic("no_such_kernel") is None
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(ROOT, "profiles"), root / "profiles")
    shutil.copytree(os.path.join(ROOT, "group_wise_affine_qmv_b200", "csrc"), root / "group_wise_affine_qmv_b200" / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.committed_traffic("qmm_warp_kernel_decode_chain") is not None
    src = root / "group_wise_affine_qmv_b200" / "csrc" / "warp_mma_kernel.cuh"
    src.write_text(src.read_text() + "\n// edited\n")
    assert bench.committed_traffic("qmm_warp_kernel_decode_chain") is None
