"""Stand-ins for the CUDA runtime and the library binding, so that the
benchmark's Python can run on CPU: streams and events that do nothing (events
report a fixed elapsed time), a torch module whose devices are the CPU, and a
binding whose calls are recorded instead of launched."""
import contextlib
import types

import torch


class _Stream:
    def wait_event(self, ev):
        pass


def fake_cuda(elapsed_ms=2.0):
    class _Event:
        def __init__(self, enable_timing=False):
            pass

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return elapsed_ms

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


class FakeTorch(types.ModuleType):
    """The torch module with a CPU device and a fake CUDA namespace."""

    def __getattr__(self, name):
        return getattr(torch, name)


def fake_sparge(calls):
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


def install(monkeypatch, bench, pkg, calls, elapsed_ms=2.0):
    """Points the benchmark at the CPU stand-ins: for the rest of a test when
    given pytest's monkeypatch, for good (a throw-away process) when given
    None."""
    def put(obj, name, value):
        if monkeypatch is None:
            setattr(obj, name, value)
        else:
            monkeypatch.setattr(obj, name, value, raising=False)

    fake_torch = FakeTorch("torch")
    fake_torch.device = lambda *a, **k: torch.device("cpu", 0)
    fake_torch.cuda = fake_cuda(elapsed_ms)
    put(bench, "torch", fake_torch)
    put(torch.Tensor, "pin_memory", lambda self, *a, **k: self)
    put(pkg, "sparge", fake_sparge(calls))
