"""sparge_mask_noalloc: the block mask for callers that cannot allocate device
memory (code running inside a host framework that owns every device
allocation, or code that must not risk an allocation failure mid-run).

The entry point keeps its scratch in a fixed array inside the library, so the
caller passes only inputs and outputs. These tests call it through the C ABI
and check it against sparge_mask (which takes a caller-allocated workspace) on
two calls in a row, since every call reuses the same array.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_pooled_b200 import synth

pytestmark = pytest.mark.gpu


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, Q, K, shape, topk, topp, with_probs):
    B, H, N, _ = Q.shape
    nqb, nkb = -(-N // shape.bq), -(-N // shape.bk)
    idx = torch.full((B, H, nqb, nkb), -7, dtype=torch.int32, device=Q.device)
    cnt = torch.full((B, H, nqb), -7, dtype=torch.int32, device=Q.device)
    thr = torch.empty((B, H, nqb), dtype=torch.float32, device=Q.device)
    probs = torch.empty((B, H, nqb, nkb), dtype=torch.float32, device=Q.device) if with_probs else None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.raw().sparge_mask_noalloc(_ptr(Q), _ptr(K), ctypes.byref(shape), float(topk), float(topp), _ptr(idx),
                                       _ptr(cnt), _ptr(thr), _ptr(probs), stream)
    assert rc == lib.OK, lib.raw().sparge_status_string(rc)
    torch.cuda.synchronize()
    return idx, cnt, thr, probs


def _reference(lib, Q, K, shape, topk, topp):
    B, H, N, _ = Q.shape
    nqb, nkb = -(-N // shape.bq), -(-N // shape.bk)
    thr = torch.empty((B, H, nqb), dtype=torch.float32, device=Q.device)
    probs = torch.empty((B, H, nqb, nkb), dtype=torch.float32, device=Q.device)
    idx, cnt = lib.sparge_mask(Q, K, shape.bq, shape.bk, topk, topp, row_thresh=thr, probs=probs)
    torch.cuda.synchronize()
    return idx, cnt, thr, probs


def _same_mask(a_idx, a_cnt, b_idx, b_cnt):
    assert torch.equal(a_cnt, b_cnt)
    valid = torch.arange(a_idx.shape[-1], device=a_idx.device)[None, None, None, :] < a_cnt[..., None]
    assert torch.equal(a_idx[valid], b_idx[valid])


@pytest.mark.parametrize("N,d,bq,bk,topk,topp", [(4096, 64, 64, 64, 0.1, 0.9), (32760, 128, 128, 64, 0.05, 0.9),
                                                   (1000, 128, 64, 128, 0.2, 0.5)])
@pytest.mark.parametrize("with_probs", [False, True])
def test_noalloc_matches_workspace_entry_point_twice(N, d, bq, bk, topk, topp, with_probs):
    from block_sparse_attention_pooled_b200 import sparge

    Q, K, _ = synth.make_qkv(1, 4, N, d, grid=None, s=2.0, seed=N + d)
    Q, K = Q.cuda(), K.cuda()
    shape = sparge.Shape(1, 4, N, d, bq, bk)
    r_idx, r_cnt, r_thr, r_probs = _reference(sparge, Q, K, shape, topk, topp)
    for _ in range(2):  # the second call runs on whatever the first left in the array
        idx, cnt, thr, probs = _noalloc(sparge, Q, K, shape, topk, topp, with_probs)
        _same_mask(idx, cnt, r_idx, r_cnt)
        assert torch.equal(thr, r_thr)
        if with_probs:
            assert torch.equal(probs, r_probs)
    assert sparge.device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from block_sparse_attention_pooled_b200 import sparge

    P = ctypes.c_void_p(16 * 1024)  # never dereferenced: the size check comes first
    # 720p-sized mask: pooled Q/K 73 MB + score rows 224 MB > 16 MiB.
    big = sparge.Shape(1, 40, 75600, 128, 128, 64)
    rc = sparge.raw().sparge_mask_noalloc(P, P, ctypes.byref(big), 0.03, 0.9, P, P, None, None, None)
    assert rc == sparge.ERR_WORKSPACE
    # Still too large when the caller also asks for the probability rows.
    rc = sparge.raw().sparge_mask_noalloc(P, P, ctypes.byref(big), 0.03, 0.9, P, P, None, P, None)
    assert rc == sparge.ERR_WORKSPACE
