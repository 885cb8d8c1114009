"""Host logic of the multi-GPU benchmark path on CPU (gloo, world size 2): the
per-rank timings reduce to the slowest rank on every rank, the whole-job value
counts every rank's work, and the reference arm prints one line from rank 0
only. No GPU is touched."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench

        got = bench.max_over_ranks([10.0 + rank, 5.0 - rank], world, "cpu")
        total = bench.sum_over_ranks(1e12 * (rank + 1), world, "cpu")
        out.put((rank, got, bench.job_value(1e12, got[0], world), total))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value, total in res:
        assert got == [11.0, 5.0]  # slowest rank per entry
        assert value == pytest.approx(2 * 1e12 / 11e-3 / 1e12)
        assert total == pytest.approx(3e12)  # every rank's own work, summed on every rank


@pytest.mark.parametrize("B,H,world", [(1, 40, 8), (1, 40, 3), (2, 3, 4), (1, 24, 24), (3, 5, 2)])
def test_head_slices_cover_every_pair_once_and_balance(B, H, world):
    """The head-sharded layout: the ranks' contiguous shares of the (b, h)
    pairs are disjoint, cover all B*H pairs in order, and differ in size by at
    most one."""
    import bench

    slices = [bench.head_slice(B, H, r, world) for r in range(world)]
    flat = [p for sl in slices for p in sl]
    assert flat == [(b, h) for b in range(B) for h in range(H)]
    sizes = [len(sl) for sl in slices]
    assert max(sizes) - min(sizes) <= 1


def test_reference_arm_prints_once_from_rank_zero_under_torchrun():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny", "--beta", "0.5"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [ln for ln in proc.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
