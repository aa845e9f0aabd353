"""Multi-process plumbing of the benchmark on CPU (gloo, world size 2): the
max-over-ranks timing and the reference arm's one-line output under torchrun."""
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
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench

        out[rank] = bench.max_over_ranks(1.5 + rank, world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_reference_arm_under_torchrun_prints_one_line():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def _bench_rank(rank, world, port, out):
    """One rank of bench.run_ours on CPU with the library calls recorded; rank r
    reports r + 2 ms for every timed region, so the line must carry rank 1's."""
    import argparse
    import contextlib
    import io

    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import bench_fakes
        import block_sparse_attention_pooled_b200 as pkg
        from block_sparse_attention_pooled_b200 import synth

        calls = []
        bench_fakes.install(None, bench, pkg, calls, elapsed_ms=2.0 + rank)
        w = synth.Workload("plumbing", 1, 2, 256, 64, (1, 16, 16), 64, 64, 0.1, 0.9, 1.5, False)
        args = argparse.Namespace(gpus=world, steps=4, warmup=3, workload=w.name, impl="ours", variant="bf16",
                                  router=0, no_cpu_baseline=False, no_e2e=False)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_ours(args, w, rank, world, 0)
        out[rank] = (buf.getvalue(), sum(c[0] == "attn_fwd" for c in calls))
    finally:
        dist.destroy_process_group()


def test_bench_ranks_report_the_slowest_rank_once():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_bench_rank, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    text0, n0 = res[0]
    text1, n1 = res[1]
    assert text1 == "" and n0 == n1  # rank 1 prints nothing and ran the same steps
    lines = [ln for ln in text0.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["n_gpus"] == 2 and rec["scaling"] == "weak"
    assert rec["ms_per_step"] == 3.0  # the slower rank's 3 ms per step (each step has its own events)
    assert rec["e2e"]["ms_per_step"] == 3.0 / max(3, 4 // 4)
    assert rec["cpu_baseline"] is None  # the oracle is timed at N = 1 only
    # value = the work of both ranks over the slowest rank's time
    one_rank_flops = rec["kept_fraction"] * 4.0 * 2 * 256 * 256 * 64
    assert abs(rec["value"] - 2 * one_rank_flops / (3.0 * 1e-3) / 1e12) < 1e-9 * rec["value"]
