"""The benchmark's own Python, run on CPU with the library calls replaced by
recorders: argument flow through one step, the device-timed loop, both
end-to-end schedules and the JSON line. Nothing here computes attention; it
checks that the harness calls the library the way the timing claims and that
every key of the line is present."""
import argparse
import contextlib
import json
import types

import pytest
import torch

import bench
import block_sparse_attention_pooled_b200 as pkg
from block_sparse_attention_pooled_b200 import synth


class _Stream:
    def wait_event(self, ev):
        pass


class _Event:
    def __init__(self, enable_timing=False):
        pass

    def record(self, stream=None):
        pass

    def elapsed_time(self, other):
        return 2.0


def _fake_cuda():
    ns = types.SimpleNamespace()
    main = _Stream()
    ns.set_device = lambda dev: None
    ns.current_stream = lambda *a: main
    ns.Stream = lambda device=None: _Stream()
    ns.Event = _Event
    ns.synchronize = lambda *a: None
    ns.stream = lambda s: contextlib.nullcontext()

    def no_props(dev):
        raise RuntimeError("no device")

    ns.get_device_properties = no_props
    return ns


class _Torch(types.ModuleType):
    """The torch module with a CPU device and a fake CUDA namespace."""

    def __getattr__(self, name):
        return getattr(torch, name)


def _fake_sparge(calls):
    from block_sparse_attention_pooled_b200 import sparge as real

    ns = types.SimpleNamespace(**{k: getattr(real, k) for k in dir(real) if k.isupper()})
    ns.make_shape, ns.workspace_bytes, ns.order_launches = real.make_shape, real.workspace_bytes, real.order_launches

    def mask(Q, K, bq, bk, topk, topp, kv_idx=None, kv_cnt=None, workspace=None, **kw):
        calls.append(("mask", Q.data_ptr()))
        nkb = kv_idx.shape[-1]
        kv_idx.copy_(torch.arange(nkb, dtype=torch.int32).expand_as(kv_idx))
        kv_cnt.fill_(min(2, nkb))

    def record(name):
        def f(*a, **kw):
            calls.append((name, a[0].data_ptr()))
        return f

    ns.sparge_mask = mask
    ns.sparge_mask_router = record("mask_router")
    ns.sparge_attn_fwd = record("attn_fwd")
    ns.sparge_attn_fwd_q8 = record("attn_fwd_q8")
    ns.sla2_attn_fwd = record("sla2_attn_fwd")
    ns.sparge_attn_bwd = record("attn_bwd")
    ns.sla2_attn_bwd = record("sla2_attn_bwd")
    ns.device_status = lambda *a: 0
    return ns


@pytest.mark.parametrize("variant,sla2,cpu", [("bf16", False, False), ("bf16", True, True), ("bwd", False, False),
                                              ("bwd", True, True), ("q8", False, False)])
def test_bench_line_with_recorded_library_calls(monkeypatch, capsys, variant, sla2, cpu):
    calls = []
    fake_torch = _Torch("torch")
    fake_torch.device = lambda *a, **k: torch.device("cpu", 0)
    fake_torch.cuda = _fake_cuda()
    monkeypatch.setattr(bench, "torch", fake_torch)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self, *a, **k: self)
    monkeypatch.setattr(pkg, "sparge", _fake_sparge(calls), raising=False)
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
