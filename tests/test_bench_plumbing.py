"""The benchmark's own Python, run on CPU with the library calls replaced by
recorders: argument flow through one step, the device-timed loop, both
end-to-end schedules and the JSON line. Nothing here computes attention; it
checks that the harness calls the library the way the timing claims and that
every key of the line is present."""
import argparse
import json

import bench_fakes
import pytest

import bench
import block_sparse_attention_pooled_b200 as pkg
from block_sparse_attention_pooled_b200 import synth


@pytest.mark.parametrize("variant,sla2,cpu", [("bf16", False, False), ("bf16", True, True), ("bwd", False, False),
                                              ("bwd", True, True), ("q8", False, False)])
def test_bench_line_with_recorded_library_calls(monkeypatch, capsys, variant, sla2, cpu):
    calls = []
    bench_fakes.install(monkeypatch, bench, pkg, calls)
    w = synth.Workload("plumbing", 1, 2, 256, 64, (1, 16, 16), 64, 64, 0.1, 0.9, 1.5, sla2)
    steps, warmup = 8, 3
    args = argparse.Namespace(gpus=1, steps=steps, warmup=warmup, workload=w.name, impl="ours", variant=variant,
                              router=0, no_cpu_baseline=not cpu, no_e2e=False)
    bench.run_ours(args, w, 0, 1, 0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    attn = {"bf16": "sla2_attn_fwd" if sla2 else "attn_fwd", "q8": "attn_fwd_q8",
            "bwd": "sla2_attn_bwd" if sla2 else "attn_bwd"}[variant]
    ksteps = max(3, steps // 4)
    per_step = [c for c in calls if c[0] == attn]
    # warm-up, timed steps, serial e2e (2 + k) and overlapped e2e (2 + k)
    assert len(per_step) == warmup + steps + 2 * (2 + ksteps)
    assert sum(c[0] == "mask" for c in calls) == len(per_step)
    # The overlapped schedule alternates between two input buffer sets.
    tail = [c[1] for c in per_step[-ksteps:]]
    assert len(set(tail)) == 2 and all(tail[i] != tail[i + 1] for i in range(len(tail) - 1))
    e2e = line["e2e"]
    assert e2e["copies"].startswith("overlapped") and "overlap_error" not in e2e
    n_in = 4 if variant == "bwd" else 3
    assert e2e["h2d_bytes_per_step"] == n_in * 2 * 256 * 64 * 2
    n_out = (3 * 2 * 256 * 64 * 2 + (2 * 4 if sla2 else 0)) if variant == "bwd" else 2 * 256 * 64 * 2
    assert e2e["d2h_bytes_per_step"] == n_out
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["steps"] == steps and line["warmup"] == warmup and line["n_gpus"] == 1
    assert line["roofline"]["bound"] == "tensor" and line["roofline"]["frac"] > 0
    assert line["config"]["workload"] == "plumbing"
    if cpu:
        cb = line["cpu_baseline"]
        assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0 and "plumbing" in cb["sample"]
    else:
        assert line["cpu_baseline"] is None
