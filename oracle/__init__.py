"""ctypes front end of the CPU oracle (test infrastructure only).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package. The CUDA library never uses it, and it shares no code
with the CUDA library.

Functions take CPU torch tensors or numpy arrays and return numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sparge_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

# IEEE semantics are part of the oracle's contract: no fast-math and no
# contraction of separate multiplies and adds into fused ones.
_CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (g++, single-threaded code)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *_CXXFLAGS, _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        p = ctypes.c_void_p
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.oracle_pool_f64.argtypes = [p, i64, i64, i32, i32, p]
        lib.oracle_block_probs_f64.argtypes = [p, p, i64, i64, i64, i32, p]
        lib.oracle_select_row.argtypes = [p, i64, dbl, dbl, p, p, p, p, p, p]
        lib.oracle_mask.argtypes = [p, p, i64, i64, i32, i32, i32, dbl, dbl, p, p, p]
        lib.oracle_attention_rows.argtypes = [p, p, p, i64, i64, i32, i32, i32, p, p, p, i64, i32,
                                              p, i64, p, p]
        lib.oracle_mask_router.argtypes = [p, p, i64, i64, i32, i32, i32, p, p, i64, i32, dbl, dbl, p, p, p]
        lib.oracle_quant_q8.argtypes = [p, p, p, i64, i64, i32, i32, i32, p, p, p, p, p, p]
        lib.oracle_e4m3.argtypes = [p, i64, p]
        lib.oracle_attention_bwd.argtypes = [p, p, p, p, i64, i64, i32, i32, i32, p, p, p, i64, i32, p, i64, p, i64,
                                             p, p, p, p]
        lib.oracle_attention_q8_rows.argtypes = [p, p, p, i64, i64, i32, i32, i32, p, p, p, i64, p]
        for f in (lib.oracle_pool_f64, lib.oracle_block_probs_f64, lib.oracle_select_row, lib.oracle_mask,
                  lib.oracle_attention_rows, lib.oracle_quant_q8, lib.oracle_e4m3,
                  lib.oracle_attention_q8_rows, lib.oracle_mask_router):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _bits(x) -> np.ndarray:
    """bf16 tensor/array -> contiguous uint16 numpy array of its bit patterns."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16, x.dtype
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16
    return a


def _check(rc: int, name: str):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments (code {rc})")


def pool(X, blk: int) -> np.ndarray:
    """Mean-pool [B,H,N,d] bf16 over blocks of blk rows -> float64 [B,H,ceil(N/blk),d]."""
    x = _bits(X)
    B, H, N, d = x.shape
    nb = -(-N // blk)
    out = np.empty((B, H, nb, d), np.float64)
    _check(_load().oracle_pool_f64(_ptr(x), B * H, N, d, blk, _ptr(out)), "pool")
    return out


def block_probs(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Row softmax of pooled scores, in float64."""
    B, H, nqb, d = qbar.shape
    nkb = kbar.shape[2]
    qb = np.ascontiguousarray(qbar, np.float64)
    kb = np.ascontiguousarray(kbar, np.float64)
    out = np.empty((B, H, nqb, nkb), np.float64)
    _check(_load().oracle_block_probs_f64(_ptr(qb), _ptr(kb), B * H, nqb, nkb, d, _ptr(out)), "probs")
    return out


def select_row(P, topk: float, topp: float):
    """Hybrid selection on one probability row.

    Returns dict(kept=ascending int32 array, m, kc, pc, order, cum)."""
    p = np.ascontiguousarray(P, np.float64)
    n = p.shape[0]
    kept = np.zeros(n, np.int32)
    order = np.zeros(n, np.int32)
    cum = np.zeros(n + 1, np.float64)
    m, kc, pc = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _check(_load().oracle_select_row(_ptr(p), n, float(topk), float(topp), _ptr(kept),
                                     ctypes.byref(m), ctypes.byref(kc), ctypes.byref(pc),
                                     _ptr(order), _ptr(cum)), "select_row")
    return dict(kept=kept[: m.value].copy(), m=m.value, kc=kc.value, pc=pc.value, order=order, cum=cum)


def mask(Q, K, bq: int, bk: int, topk: float, topp: float):
    """Block mask for every query-block row (the double-precision definition).

    Returns (kv_idx int32 [B,H,Nqb,Nkb], kv_cnt int32 [B,H,Nqb], P float64 [B,H,Nqb,Nkb])."""
    q, k = _bits(Q), _bits(K)
    B, H, N, d = q.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx = np.zeros((B, H, nqb, nkb), np.int32)
    kv_cnt = np.zeros((B, H, nqb), np.int32)
    P = np.zeros((B, H, nqb, nkb), np.float64)
    _check(_load().oracle_mask(_ptr(q), _ptr(k), B * H, N, d, bq, bk, float(topk), float(topp),
                               _ptr(kv_idx), _ptr(kv_cnt), _ptr(P)), "mask")
    return kv_idx, kv_cnt, P


def mask_router(Q, K, bq: int, bk: int, Wq, Wk, topk: float, topp: float):
    """Block mask with a learnt router: pooled blocks projected by Wq / Wk
    (float32 [H, d, dr], one pair per head) before scoring.

    Returns (kv_idx, kv_cnt, P) like mask()."""
    q, k = _bits(Q), _bits(K)
    B, H, N, d = q.shape
    wq = np.ascontiguousarray(np.asarray(Wq), np.float32)
    wk = np.ascontiguousarray(np.asarray(Wk), np.float32)
    assert wq.shape == wk.shape and wq.shape[:2] == (H, d), (wq.shape, wk.shape)
    dr = wq.shape[2]
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx = np.zeros((B, H, nqb, nkb), np.int32)
    kv_cnt = np.zeros((B, H, nqb), np.int32)
    P = np.zeros((B, H, nqb, nkb), np.float64)
    _check(_load().oracle_mask_router(_ptr(q), _ptr(k), B * H, N, d, bq, bk, _ptr(wq), _ptr(wk), H, dr,
                                      float(topk), float(topp), _ptr(kv_idx), _ptr(kv_cnt), _ptr(P)),
           "mask_router")
    return kv_idx, kv_cnt, P


MODES = {"sparse": 0, "linear": 1, "sla2": 2, "dense": 3}


def attention_rows(Q, K, V, bq: int, bk: int, kv_idx=None, kv_cnt=None, alpha=None,
                   mode: str = "sparse", rows=None):
    """Double-precision outputs for selected rows.

    rows: flat ids b*H*N + h*N + i (default: every row). Returns (O [nrows,d]
    float64, lse [nrows] float64)."""
    q, k, v = _bits(Q), _bits(K), _bits(V)
    B, H, N, d = q.shape
    if rows is None:
        rows = np.arange(B * H * N, dtype=np.int64)
    rows = np.ascontiguousarray(rows, np.int64)
    idx = None if kv_idx is None else np.ascontiguousarray(np.asarray(kv_idx), np.int32)
    cnt = None if kv_cnt is None else np.ascontiguousarray(np.asarray(kv_cnt), np.int32)
    al = None if alpha is None else np.ascontiguousarray(np.asarray(alpha), np.float32)
    O = np.zeros((rows.shape[0], d), np.float64)
    lse = np.zeros(rows.shape[0], np.float64)
    _check(_load().oracle_attention_rows(_ptr(q), _ptr(k), _ptr(v), B * H, N, d, bq, bk, _ptr(idx),
                                         _ptr(cnt), _ptr(al), H, MODES[mode], _ptr(rows),
                                         rows.shape[0], _ptr(O), _ptr(lse)), "attention_rows")
    return O, lse


def attention_bwd(Q, K, V, dO, bq: int, bk: int, kv_idx=None, kv_cnt=None, alpha=None, mode: str = "sparse",
                  rows=None, kblocks=None, want_dalpha: bool = False):
    """Double-precision gradients of the forward of attention_rows for dL/dO = dO (bf16).

    rows: flat query rows b*H*N + h*N + i whose dQ is wanted (default: all).
    kblocks: flat key blocks (b*H + h)*Nkb + J whose dK, dV are wanted
    (default: all). Returns (dQ [nrows,d], dK [nblocks,bk,d], dV [nblocks,bk,d],
    dalpha [H] or None), float64; dK / dV rows past N are zero."""
    q, k, v, g = _bits(Q), _bits(K), _bits(V), _bits(dO)
    B, H, N, d = q.shape
    nkb = -(-N // bk)
    rows = np.arange(B * H * N, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    kb = np.arange(B * H * nkb, dtype=np.int64) if kblocks is None else np.ascontiguousarray(kblocks, np.int64)
    idx = None if kv_idx is None else np.ascontiguousarray(np.asarray(kv_idx), np.int32)
    cnt = None if kv_cnt is None else np.ascontiguousarray(np.asarray(kv_cnt), np.int32)
    al = None if alpha is None else np.ascontiguousarray(np.asarray(alpha), np.float32)
    dQ = np.zeros((rows.shape[0], d), np.float64)
    dK = np.zeros((kb.shape[0], bk, d), np.float64)
    dV = np.zeros((kb.shape[0], bk, d), np.float64)
    da = np.zeros(H, np.float64) if want_dalpha else None
    _check(_load().oracle_attention_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B * H, N, d, bq, bk, _ptr(idx),
                                        _ptr(cnt), _ptr(al), H, MODES[mode], _ptr(rows), rows.shape[0], _ptr(kb),
                                        kb.shape[0], _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(da)), "attention_bwd")
    return dQ, dK, dV, da


def e4m3(x) -> np.ndarray:
    """Nearest fp8 e4m3 value of each element (ties to even, saturating at 448), as float64."""
    a = np.ascontiguousarray(np.asarray(x, np.float64))
    out = np.empty_like(a)
    _check(_load().oracle_e4m3(_ptr(a), a.size, _ptr(out)), "e4m3")
    return out


def quant_q8(Q, K, V, bq: int, bk: int):
    """Quantised operands of the low-bit sparse branch.

    Returns (q8 int8 [B,H,N,d], sq float32 [B,H,Nqb], k8 int8 [B,H,N,d],
    sk float32 [B,H,Nkb], v8 float64 [B,H,N,d] (e4m3 values), sv float32 [B,H,d])."""
    q, k, v = _bits(Q), _bits(K), _bits(V)
    B, H, N, d = q.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    q8 = np.empty((B, H, N, d), np.int8)
    k8 = np.empty((B, H, N, d), np.int8)
    v8 = np.empty((B, H, N, d), np.float64)
    sq = np.empty((B, H, nqb), np.float32)
    sk = np.empty((B, H, nkb), np.float32)
    sv = np.empty((B, H, d), np.float32)
    _check(_load().oracle_quant_q8(_ptr(q), _ptr(k), _ptr(v), B * H, N, d, bq, bk, _ptr(q8), _ptr(sq),
                                   _ptr(k8), _ptr(sk), _ptr(v8), _ptr(sv)), "quant_q8")
    return q8, sq, k8, sk, v8, sv


def attention_q8_rows(Q, K, V, bq: int, bk: int, kv_idx, kv_cnt, rows=None) -> np.ndarray:
    """Low-bit sparse branch outputs (float64 [nrows, d]) for selected rows
    (flat ids b*H*N + h*N + i; default every row)."""
    q, k, v = _bits(Q), _bits(K), _bits(V)
    B, H, N, d = q.shape
    if rows is None:
        rows = np.arange(B * H * N, dtype=np.int64)
    rows = np.ascontiguousarray(rows, np.int64)
    idx = np.ascontiguousarray(np.asarray(kv_idx), np.int32)
    cnt = np.ascontiguousarray(np.asarray(kv_cnt), np.int32)
    O = np.zeros((rows.shape[0], d), np.float64)
    _check(_load().oracle_attention_q8_rows(_ptr(q), _ptr(k), _ptr(v), B * H, N, d, bq, bk, _ptr(idx),
                                            _ptr(cnt), _ptr(rows), rows.shape[0], _ptr(O)),
           "attention_q8_rows")
    return O
