"""The C ABI loads, exports every declared symbol and rejects bad arguments
on the host (no GPU needed: nothing here reaches a CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparge.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sparge_\w+|sla2_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_pooled_b200 import build

    build.build()
    from block_sparse_attention_pooled_b200 import sparge

    return sparge


def test_header_declares_the_three_operations():
    names = _declared_functions()
    for n in ("sparge_mask", "sparge_attn_fwd", "sla2_attn_fwd", "sparge_workspace_bytes",
              "sparge_device_status", "sparge_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    raw = lib.raw()
    for name in _declared_functions():
        assert hasattr(raw, name), name
    assert set(_declared_functions()) == set(lib.EXPORTS)


def test_status_strings(lib):
    raw = lib.raw()
    for code in range(6):
        assert raw.sparge_status_string(code)
    assert raw.sparge_status_string(0) == b"ok"


def test_workspace_bytes_host_arithmetic(lib):
    s = lib.Shape(1, 40, 75600, 128, 128, 64)
    nqb, nkb = 591, 1182
    need = lib.workspace_bytes(lib.OP_MASK, s)
    # pooled Q and K and the score rows, all in double
    assert need >= 40 * (nqb + nkb) * 128 * 8 + 40 * nqb * nkb * 8
    assert lib.workspace_bytes(lib.OP_ATTN, s) >= 40 * nqb * 4  # the tiles' launch order
    bad = lib.Shape(1, 1, 100, 96, 64, 64)  # unsupported head dim
    assert lib.workspace_bytes(lib.OP_MASK, bad) == 0
    # Low-bit branch: three code tensors of one byte per element plus the scales.
    need_q8 = lib.workspace_bytes(lib.OP_ATTN_Q8, s)
    assert need_q8 >= 3 * 40 * 75600 * 128 + 4 * 40 * (nqb + nkb + 128)
    assert lib.workspace_bytes(lib.OP_ATTN_Q8, lib.Shape(1, 1, 4096, 64, 64, 64)) == 0  # d = 128 only
    # Learnt router: the mask's scratch plus the projected blocks at the widest router width.
    need_r = lib.workspace_bytes(lib.OP_MASK_ROUTER, s)
    assert need_r >= need + 40 * (nqb + nkb) * 128 * 8
    assert lib.workspace_bytes(lib.OP_MASK_ROUTER, bad) == 0


def test_selftest_wait_rejects_limits_before_any_launch(lib):
    raw = lib.raw()
    for bad in (0, -5, 1000001):
        assert raw.sparge_selftest_wait(bad, None, None) == lib.ERR_INVALID_ARG
    assert raw.sparge_selftest_wait(100, ctypes.c_void_p(2), None) == lib.ERR_INVALID_ARG  # misaligned flag


def test_invalid_arguments_rejected_before_any_launch(lib):
    raw = lib.raw()
    s = lib.Shape(1, 2, 4096, 64, 64, 64)
    P = ctypes.c_void_p(16 * 1024)  # never dereferenced: checks fail first
    # null shape, null inputs
    assert raw.sparge_mask(P, P, None, 0.1, 0.9, P, P, None, None, P, 1 << 30, None) == lib.ERR_INVALID_ARG
    assert raw.sparge_mask(None, P, ctypes.byref(s), 0.1, 0.9, P, P, None, None, P, 1 << 30, None) == lib.ERR_INVALID_ARG
    # fractions out of range
    assert raw.sparge_mask(P, P, ctypes.byref(s), 1.5, 0.9, P, P, None, None, P, 1 << 30, None) == lib.ERR_INVALID_ARG
    assert raw.sparge_mask(P, P, ctypes.byref(s), 0.1, -0.1, P, P, None, None, P, 1 << 30, None) == lib.ERR_INVALID_ARG
    assert raw.sparge_mask(P, P, ctypes.byref(s), float("nan"), 0.9, P, P, None, None, P, 1 << 30, None) == lib.ERR_INVALID_ARG
    # workspace missing / too small
    assert raw.sparge_mask(P, P, ctypes.byref(s), 0.1, 0.9, P, P, None, None, None, 0, None) == lib.ERR_WORKSPACE
    assert raw.sparge_mask(P, P, ctypes.byref(s), 0.1, 0.9, P, P, None, None, P, 16, None) == lib.ERR_WORKSPACE
    # misaligned input
    assert raw.sparge_mask(ctypes.c_void_p(16 * 1024 + 2), P, ctypes.byref(s), 0.1, 0.9, P, P, None, None, P,
                           1 << 30, None) == lib.ERR_INVALID_ARG
    # unsupported shapes
    for bad in (lib.Shape(1, 1, 100, 96, 64, 64), lib.Shape(1, 1, 100, 64, 32, 64), lib.Shape(1, 1, 100, 64, 64, 256),
                lib.Shape(1, 1, 64 * 5000, 64, 64, 64)):
        assert raw.sparge_attn_fwd(P, P, P, ctypes.byref(bad), P, P, P, None, None, 0, None) == lib.ERR_UNSUPPORTED
    # the block-count limit: 4096 key blocks per row, exactly
    assert lib.workspace_bytes(lib.OP_MASK, lib.Shape(1, 1, 64 * 4096, 64, 64, 64)) > 0
    assert lib.workspace_bytes(lib.OP_MASK, lib.Shape(1, 1, 64 * 4096 + 1, 64, 64, 64)) == 0
    assert lib.workspace_bytes(lib.OP_MASK, lib.Shape(1, 1, 128 * 4096, 64, 128, 128)) > 0
    for bad in (lib.Shape(0, 1, 100, 64, 64, 64), lib.Shape(1, 1, -5, 64, 64, 64)):
        assert raw.sparge_attn_fwd(P, P, P, ctypes.byref(bad), P, P, P, None, None, 0, None) == lib.ERR_INVALID_ARG
    assert raw.sparge_attn_fwd(P, P, None, ctypes.byref(s), P, P, P, None, None, 0, None) == lib.ERR_INVALID_ARG
    assert raw.sla2_attn_fwd(P, P, P, None, P, P, P, P, None, 0, None) == lib.ERR_INVALID_ARG
    # Low-bit branch: d = 128 only, workspace required.
    assert raw.sparge_attn_fwd_q8(P, P, P, ctypes.byref(s), P, P, P, P, 1 << 30, None) == lib.ERR_UNSUPPORTED
    s128 = lib.Shape(1, 2, 4096, 128, 128, 64)
    assert raw.sparge_attn_fwd_q8(P, P, P, ctypes.byref(s128), P, P, P, None, 0, None) == lib.ERR_WORKSPACE
    assert raw.sparge_attn_fwd_q8(P, P, P, ctypes.byref(s128), P, P, P, P, 64, None) == lib.ERR_WORKSPACE
    assert raw.sparge_attn_fwd_q8(P, None, P, ctypes.byref(s128), P, P, P, P, 1 << 30, None) == lib.ERR_INVALID_ARG
    # Backward entry points: d = 128 only, every buffer required, workspace sized for them.
    s128b = lib.Shape(1, 2, 4096, 128, 128, 64)
    nb = lib.workspace_bytes(lib.OP_ATTN_BWD, s128b)
    assert nb > 0 and lib.workspace_bytes(lib.OP_ATTN_BWD, s) == 0
    assert raw.sparge_attn_bwd(P, P, P, ctypes.byref(s), P, P, P, P, P, P, P, P, P, 1 << 30, None) == lib.ERR_UNSUPPORTED
    assert raw.sparge_attn_bwd(P, P, P, ctypes.byref(s128b), P, P, P, None, P, P, P, P, P, 1 << 30,
                               None) == lib.ERR_INVALID_ARG  # lse required
    assert raw.sparge_attn_bwd(P, P, P, ctypes.byref(s128b), P, P, P, P, P, P, P, P, P, nb - 1,
                               None) == lib.ERR_WORKSPACE
    ns = lib.workspace_bytes(lib.OP_SLA2_BWD, s128b)
    assert ns > nb
    assert raw.sla2_attn_bwd(P, P, P, ctypes.byref(s128b), P, P, None, P, P, P, P, P, P, 1 << 34,
                             None) == lib.ERR_INVALID_ARG  # alpha required
    assert raw.sla2_attn_bwd(P, P, P, ctypes.byref(s128b), P, P, P, P, P, P, P, None, P, 1 << 34,
                             None) == lib.ERR_INVALID_ARG  # dalpha required
    assert raw.sla2_attn_bwd(P, P, P, ctypes.byref(s128b), P, P, P, P, P, P, P, P, P, ns - 1,
                             None) == lib.ERR_WORKSPACE
    assert raw.sla2_attn_bwd(P, P, P, ctypes.byref(s), P, P, P, P, P, P, P, P, P, 1 << 34, None) == lib.ERR_UNSUPPORTED
    # Learnt router: both projections required, 4-byte aligned; dr 64 or 128; workspace sized for it.
    W, big = ctypes.c_void_p(32 * 1024), 1 << 30
    assert raw.sparge_mask_router(P, P, ctypes.byref(s), None, W, 64, 0.1, 0.9, P, P, None, None, P, big,
                                  None) == lib.ERR_INVALID_ARG
    assert raw.sparge_mask_router(P, P, ctypes.byref(s), W, None, 64, 0.1, 0.9, P, P, None, None, P, big,
                                  None) == lib.ERR_INVALID_ARG
    assert raw.sparge_mask_router(P, P, ctypes.byref(s), ctypes.c_void_p(32 * 1024 + 2), W, 64, 0.1, 0.9, P, P,
                                  None, None, P, big, None) == lib.ERR_INVALID_ARG
    assert raw.sparge_mask_router(P, P, ctypes.byref(s), W, W, 64, 1.5, 0.9, P, P, None, None, P, big,
                                  None) == lib.ERR_INVALID_ARG
    for dr in (0, 32, 96, 256):
        assert raw.sparge_mask_router(P, P, ctypes.byref(s), W, W, dr, 0.1, 0.9, P, P, None, None, P, big,
                                      None) == lib.ERR_UNSUPPORTED
    mask_only = lib.workspace_bytes(lib.OP_MASK, s)
    assert raw.sparge_mask_router(P, P, ctypes.byref(s), W, W, 64, 0.1, 0.9, P, P, None, None, P, mask_only,
                                  None) == lib.ERR_WORKSPACE
    assert raw.sparge_mask_router(P, P, ctypes.byref(s), W, W, 64, 0.1, 0.9, P, P, None, None,
                                  ctypes.c_void_p(16 * 1024 + 16), big, None) == lib.ERR_WORKSPACE


def test_binding_refuses_cpu_tensors(lib):
    import torch

    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lib.sparge_mask(q, q, 64, 64, 0.1, 0.9)
    w = torch.zeros(1, 64, 64, dtype=torch.float32)
    with pytest.raises(ValueError):
        lib.sparge_mask_router(q, q, w, w, 64, 64, 0.1, 0.9)
