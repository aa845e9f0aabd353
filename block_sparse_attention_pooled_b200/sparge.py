"""Python binding of the C ABI in include/sparge.h (argument marshalling only).

Importing this module loads ``libsparge.so`` from the package directory and
raises ImportError when it is missing: there is no fallback implementation.
Tensors are torch CUDA tensors; every call is enqueued on the current torch
stream (or the stream given) and returns without synchronising.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsparge.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m block_sparse_attention_pooled_b200.build`")
_lib = ctypes.CDLL(_LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_TIMEOUT = range(6)
OP_MASK, OP_ATTN, OP_SLA2, OP_ATTN_Q8, OP_MASK_ROUTER, OP_ATTN_BWD, OP_SLA2_BWD = 0, 1, 2, 3, 4, 5, 6

# Kernel launches per call of each entry point (for launch accounting).
MASK_LAUNCHES, ATTN_LAUNCHES, SLA2_LAUNCHES, Q8_LAUNCHES, ROUTER_LAUNCHES, BWD_LAUNCHES = 3, 1, 4, 3, 5, 4
# sla2_attn_bwd: summaries + reduce, linear_out, sparse forward, row pass, dalpha, gradient summaries
# + reduce, transposed mask, dQ, dK/dV sparse part, dK/dV linear part (the memset is not a kernel).
# The attention, SLA2 and low-bit forward calls and both backward calls add order_launches(shape).
SLA2_BWD_LAUNCHES = 12

# Every symbol the header declares.
EXPORTS = ("sparge_workspace_bytes", "sparge_mask", "sparge_attn_fwd", "sla2_attn_fwd",
           "sparge_device_status", "sparge_status_string", "sparge_mask_noalloc", "sparge_attn_fwd_q8",
           "sparge_mask_router", "sparge_attn_bwd", "sla2_attn_bwd", "sparge_selftest_wait")


def order_launches(shape) -> int:
    """Launches of the tile-order kernel per attention call for this shape (launch accounting):
    1 when at least two heads' K and V (4 N d bytes each) fit in 64 MB, else 0."""
    return 1 if min(shape.B * shape.H, (64 << 20) // (4 * shape.N * shape.d)) >= 2 else 0


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "N", "d", "bq", "bk")]


_vp, _sz, _dbl = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_double
_lib.sparge_workspace_bytes.argtypes = [ctypes.c_int, ctypes.POINTER(Shape)]
_lib.sparge_workspace_bytes.restype = _sz
_lib.sparge_mask.argtypes = [_vp, _vp, ctypes.POINTER(Shape), _dbl, _dbl, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sparge_mask_router.argtypes = [_vp, _vp, ctypes.POINTER(Shape), _vp, _vp, ctypes.c_int, _dbl, _dbl, _vp, _vp,
                                     _vp, _vp, _vp, _sz, _vp]
_lib.sparge_mask_noalloc.argtypes = [_vp, _vp, ctypes.POINTER(Shape), _dbl, _dbl, _vp, _vp, _vp, _vp, _vp]
_lib.sparge_mask_noalloc.restype = ctypes.c_int
_lib.sparge_attn_fwd.argtypes = [_vp, _vp, _vp, ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sla2_attn_fwd.argtypes = [_vp, _vp, _vp, ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sparge_attn_fwd_q8.argtypes = [_vp, _vp, _vp, ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sparge_attn_bwd.argtypes = [_vp, _vp, _vp, ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _sz, _vp]
_lib.sla2_attn_bwd.argtypes = [_vp, _vp, _vp, ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                               _vp]
_lib.sparge_device_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_int32)]
_lib.sparge_selftest_wait.argtypes = [ctypes.c_int32, _vp, _vp]
_lib.sparge_status_string.argtypes = [ctypes.c_int]
_lib.sparge_status_string.restype = ctypes.c_char_p
for _f in ("sparge_mask", "sparge_mask_router", "sparge_attn_bwd", "sla2_attn_bwd", "sparge_attn_fwd", "sla2_attn_fwd", "sparge_device_status", "sparge_attn_fwd_q8",
           "sparge_selftest_wait"):
    getattr(_lib, _f).restype = ctypes.c_int


class SpargeError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {_lib.sparge_status_string(code).decode()} (status {code})")
        self.code = code


def lib_path() -> str:
    return _LIB_PATH


def raw() -> ctypes.CDLL:
    """The loaded library (for callers that marshal pointers themselves)."""
    return _lib


def _check(code: int, where: str):
    if code != OK:
        raise SpargeError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_shape(Q: torch.Tensor, bq: int, bk: int) -> Shape:
    B, H, N, d = Q.shape
    return Shape(B, H, N, d, bq, bk)


def workspace_bytes(op: int, shape: Shape) -> int:
    return int(_lib.sparge_workspace_bytes(op, ctypes.byref(shape)))


def _workspace(op: int, shape: Shape, device) -> Tuple[Optional[torch.Tensor], int]:
    n = workspace_bytes(op, shape)
    if n == 0:
        return None, 0
    return torch.empty(n, dtype=torch.uint8, device=device), n


def _check_qkv(*ts):
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("Q/K/V/O must be contiguous bf16 CUDA tensors of shape [B,H,N,d]")


def sparge_mask(Q, K, bq: int, bk: int, topk: float, topp: float, kv_idx=None, kv_cnt=None,
                row_thresh=None, probs=None, workspace=None, stream=None):
    """Hybrid Top-k / Top-p block mask. Returns (kv_idx, kv_cnt)."""
    _check_qkv(Q, K)
    shape = make_shape(Q, bq, bk)
    B, H, N, _ = Q.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    if kv_idx is None:
        kv_idx = torch.empty((B, H, nqb, nkb), dtype=torch.int32, device=Q.device)
    if kv_cnt is None:
        kv_cnt = torch.empty((B, H, nqb), dtype=torch.int32, device=Q.device)
    if workspace is None:
        workspace, nws = _workspace(OP_MASK, shape, Q.device)
    else:
        nws = workspace.numel() * workspace.element_size()
    _check(_lib.sparge_mask(_ptr(Q), _ptr(K), ctypes.byref(shape), float(topk), float(topp), _ptr(kv_idx),
                            _ptr(kv_cnt), _ptr(row_thresh), _ptr(probs), _ptr(workspace), nws, _stream(stream)),
           "sparge_mask")
    return kv_idx, kv_cnt


def sparge_mask_router(Q, K, Wq, Wk, bq: int, bk: int, topk: float, topp: float, kv_idx=None, kv_cnt=None,
                       row_thresh=None, probs=None, workspace=None, stream=None):
    """Block mask scored through the learnt router projections Wq, Wk (fp32 [H, d, dr]).
    Returns (kv_idx, kv_cnt)."""
    _check_qkv(Q, K)
    H, d = Q.shape[1], Q.shape[3]
    for W in (Wq, Wk):
        if W.dtype != torch.float32 or not W.is_cuda or not W.is_contiguous() or W.dim() != 3 \
                or W.shape[0] != H or W.shape[1] != d or W.shape != Wq.shape:
            raise ValueError("Wq/Wk must be contiguous fp32 CUDA tensors of shape [H, d, dr]")
    shape = make_shape(Q, bq, bk)
    B, _, N, _ = Q.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    if kv_idx is None:
        kv_idx = torch.empty((B, H, nqb, nkb), dtype=torch.int32, device=Q.device)
    if kv_cnt is None:
        kv_cnt = torch.empty((B, H, nqb), dtype=torch.int32, device=Q.device)
    if workspace is None:
        workspace, nws = _workspace(OP_MASK_ROUTER, shape, Q.device)
    else:
        nws = workspace.numel() * workspace.element_size()
    _check(_lib.sparge_mask_router(_ptr(Q), _ptr(K), ctypes.byref(shape), _ptr(Wq), _ptr(Wk), int(Wq.shape[2]),
                                   float(topk), float(topp), _ptr(kv_idx), _ptr(kv_cnt), _ptr(row_thresh),
                                   _ptr(probs), _ptr(workspace), nws, _stream(stream)), "sparge_mask_router")
    return kv_idx, kv_cnt


def sparge_attn_fwd(Q, K, V, kv_idx, kv_cnt, bq: int, bk: int, O=None, lse=None, workspace=None, stream=None):
    """Block-sparse attention over the kept blocks. Returns O (and fills lse if given)."""
    _check_qkv(Q, K, V)
    shape = make_shape(Q, bq, bk)
    if O is None:
        O = torch.empty_like(Q)
    if workspace is None:
        workspace, nws = _workspace(OP_ATTN, shape, Q.device)
    else:
        nws = workspace.numel() * workspace.element_size()
    _check(_lib.sparge_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shape), _ptr(kv_idx), _ptr(kv_cnt), _ptr(O),
                                _ptr(lse), _ptr(workspace), nws, _stream(stream)), "sparge_attn_fwd")
    return O


def sparge_attn_bwd(Q, K, V, kv_idx, kv_cnt, O, lse, dO, bq: int, bk: int, dQ=None, dK=None, dV=None,
                    workspace=None, stream=None):
    """Gradients of sparge_attn_fwd (O and lse from that call) for dL/dO = dO. Returns (dQ, dK, dV)."""
    _check_qkv(Q, K, V, O, dO)
    if lse is None or lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous():
        raise ValueError("lse must be the forward's contiguous float32 CUDA log-sum-exp [B,H,N]")
    shape = make_shape(Q, bq, bk)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    if workspace is None:
        workspace, nws = _workspace(OP_ATTN_BWD, shape, Q.device)
    else:
        nws = workspace.numel() * workspace.element_size()
    _check(_lib.sparge_attn_bwd(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shape), _ptr(kv_idx), _ptr(kv_cnt), _ptr(O),
                                _ptr(lse), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(workspace), nws,
                                _stream(stream)), "sparge_attn_bwd")
    return dQ, dK, dV


def sla2_attn_bwd(Q, K, V, kv_idx, kv_cnt, alpha, dO, bq: int, bk: int, dQ=None, dK=None, dV=None, dalpha=None,
                  workspace=None, stream=None):
    """Gradients of sla2_attn_fwd for dL/dO = dO. Returns (dQ, dK, dV, dalpha)."""
    _check_qkv(Q, K, V, dO)
    if alpha.dtype != torch.float32 or not alpha.is_cuda or alpha.numel() != Q.shape[1]:
        raise ValueError("alpha must be a float32 CUDA tensor with one value per head")
    shape = make_shape(Q, bq, bk)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    dalpha = torch.empty(Q.shape[1], dtype=torch.float32, device=Q.device) if dalpha is None else dalpha
    if workspace is None:
        workspace, nws = _workspace(OP_SLA2_BWD, shape, Q.device)
    else:
        nws = workspace.numel() * workspace.element_size()
    _check(_lib.sla2_attn_bwd(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shape), _ptr(kv_idx), _ptr(kv_cnt),
                              _ptr(alpha), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dalpha), _ptr(workspace), nws,
                              _stream(stream)), "sla2_attn_bwd")
    return dQ, dK, dV, dalpha


def sparge_attn_fwd_q8(Q, K, V, kv_idx, kv_cnt, bq: int, bk: int, O=None, workspace=None, stream=None):
    """Low-bit block-sparse attention (int8 Q/K codes, e4m3 P and V codes). Returns O."""
    _check_qkv(Q, K, V)
    shape = make_shape(Q, bq, bk)
    if O is None:
        O = torch.empty_like(Q)
    if workspace is None:
        workspace, nws = _workspace(OP_ATTN_Q8, shape, Q.device)
    else:
        nws = workspace.numel() * workspace.element_size()
    _check(_lib.sparge_attn_fwd_q8(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shape), _ptr(kv_idx), _ptr(kv_cnt),
                                   _ptr(O), _ptr(workspace), nws, _stream(stream)), "sparge_attn_fwd_q8")
    return O


def quant_q8_workspace_views(workspace, shape):
    """(q8, k8, v8, sq, sk, sv) views into a sparge_attn_fwd_q8 workspace, in the
    library's layout (codes [B,H,N,128] int8 / e4m3 bytes; scales fp32)."""
    B, H, N, d, bq, bk = shape.B, shape.H, shape.N, shape.d, shape.bq, shape.bk
    nqb, nkb = -(-N // bq), -(-N // bk)
    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    codes = a256(B * H * N * d)
    off_q8, off_k8, off_v8 = 0, codes, 2 * codes
    off_sq = 3 * codes
    off_sk = off_sq + a256(B * H * nqb * 4)
    off_sv = off_sk + a256(B * H * nkb * 4)
    w = workspace.view(torch.uint8)
    q8 = w[off_q8:off_q8 + B * H * N * d].view(torch.int8).view(B, H, N, d)
    k8 = w[off_k8:off_k8 + B * H * N * d].view(torch.int8).view(B, H, N, d)
    v8 = w[off_v8:off_v8 + B * H * N * d].view(B, H, N, d)
    sq = w[off_sq:off_sq + B * H * nqb * 4].view(torch.float32).view(B, H, nqb)
    sk = w[off_sk:off_sk + B * H * nkb * 4].view(torch.float32).view(B, H, nkb)
    sv = w[off_sv:off_sv + B * H * d * 4].view(torch.float32).view(B, H, d)
    return q8, k8, v8, sq, sk, sv


def sla2_attn_fwd(Q, K, V, kv_idx, kv_cnt, alpha, bq: int, bk: int, O=None, workspace=None, stream=None):
    """alpha * sparse + (1 - alpha) * linear (phi = elu + 1 over the blocks not kept). Returns O."""
    _check_qkv(Q, K, V)
    shape = make_shape(Q, bq, bk)
    if O is None:
        O = torch.empty_like(Q)
    if workspace is None:
        workspace, nws = _workspace(OP_SLA2, shape, Q.device)
    else:
        nws = workspace.numel() * workspace.element_size()
    _check(_lib.sla2_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shape), _ptr(kv_idx), _ptr(kv_cnt),
                              _ptr(alpha), _ptr(O), _ptr(workspace), nws, _stream(stream)), "sla2_attn_fwd")
    return O


SITE_SELFTEST = 0xF00


def selftest_wait(limit_us: int, gave_up=None, stream=None) -> None:
    """Launches the bounded-wait self-test kernel (it waits on a barrier that
    nothing arrives on and gives up after limit_us microseconds)."""
    _check(_lib.sparge_selftest_wait(int(limit_us), _ptr(gave_up), _stream(stream)), "sparge_selftest_wait")


def device_status(stream=None) -> int:
    """Synchronises the stream, returns and clears the device error word (0 = none)."""
    code = ctypes.c_int32(0)
    rc = _lib.sparge_device_status(_stream(stream), ctypes.byref(code))
    if rc not in (OK, ERR_DEVICE_TIMEOUT):
        raise SpargeError(rc, "sparge_device_status")
    return int(code.value)
