"""Learnt-router block mask on the GPU against the CPU oracle's
double-precision definition, under the same ambiguity rule as the plain
mask."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_pooled_b200 import synth
from parity import check_mask_outputs

pytestmark = pytest.mark.gpu


def _run(Q, K, Wq, Wk, bq, bk, topk, topp):
    from block_sparse_attention_pooled_b200 import sparge

    dev = torch.device("cuda")
    B, H, N, d = Q.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    probs = torch.empty((B, H, nqb, nkb), dtype=torch.float32, device=dev)
    thr = torch.empty((B, H, nqb), dtype=torch.float32, device=dev)
    idx, cnt = sparge.sparge_mask_router(Q.to(dev), K.to(dev), Wq.to(dev), Wk.to(dev), bq, bk, topk, topp,
                                         row_thresh=thr, probs=probs)
    torch.cuda.synchronize()
    assert sparge.device_status() == 0
    return idx.cpu().numpy(), cnt.cpu().numpy(), probs.cpu().numpy(), thr.cpu().numpy()


def _check(Q, K, Wq, Wk, bq, bk, topk, topp, what=""):
    g = _run(Q, K, Wq, Wk, bq, bk, topk, topp)
    o = oracle.mask_router(Q, K, bq, bk, Wq, Wk, topk, topp)
    n, bad, amb = check_mask_outputs(g, o, topk, topp)
    if what:
        print(f"{what}: rows {n}, rows differing from the fp64 definition {bad} (all within the ambiguity rule)")
    return n, bad, amb


@pytest.mark.parametrize("N,d,bq,bk", [(4096, 64, 64, 64), (1000, 128, 128, 64), (777, 128, 64, 128),
                                        (130, 64, 128, 128), (5000, 128, 64, 64)])
@pytest.mark.parametrize("dr", [64, 128])
@pytest.mark.parametrize("topk,topp", [(0.1, 0.9), (0.0, 0.9), (0.2, 0.0)])
def test_router_mask_small(N, d, bq, bk, dr, topk, topp):
    Q, K, _ = synth.make_qkv(1, 3, N, d, grid=None, s=1.5, seed=N + d)
    Wq, Wk = synth.make_router(3, d, dr, seed=dr)
    _check(Q, K, Wq, Wk, bq, bk, topk, topp)


def test_router_identity_is_the_plain_mask():
    from block_sparse_attention_pooled_b200 import sparge

    Q, K, _ = synth.make_qkv(1, 2, 4096, 64, grid=(4, 32, 32), s=1.5, seed=3)
    eye = torch.eye(64, dtype=torch.float32).expand(2, 64, 64).contiguous()
    a = _run(Q, K, eye, eye, 64, 64, 0.1, 0.9)
    Qd, Kd = Q.cuda(), K.cuda()
    probs = torch.empty((1, 2, 64, 64), dtype=torch.float32, device="cuda")
    idx, cnt = sparge.sparge_mask(Qd, Kd, 64, 64, 0.1, 0.9, probs=probs)
    np.testing.assert_array_equal(a[1], cnt.cpu().numpy())
    np.testing.assert_array_equal(a[2], probs.cpu().numpy())


def test_router_480p():
    w = synth.WORKLOADS["480p"]
    Q, K, _, _ = synth.make_workload(w)
    Wq, Wk = synth.make_router(w.H, w.d, 64, seed=1)
    _check(Q, K, Wq, Wk, w.bq, w.bk, w.topk, w.topp, what="480p router (dr 64)")


def test_router_multi_batch_heads():
    # B = 2: the head of a row is (row / Nb) % H, so batch 1 reuses batch 0's projections.
    Q, K, _ = synth.make_qkv(2, 3, 2048, 128, grid=(2, 32, 32), s=2.0, seed=8)
    Wq, Wk = synth.make_router(3, 128, 128, seed=4)
    _check(Q, K, Wq, Wk, 128, 64, 0.05, 0.9)


def test_router_is_deterministic():
    Q, K, _ = synth.make_qkv(1, 2, 8192, 128, grid=(8, 32, 32), s=2.0, seed=5)
    Wq, Wk = synth.make_router(2, 128, 64, seed=2)
    a = _run(Q, K, Wq, Wk, 128, 64, 0.05, 0.9)
    b = _run(Q, K, Wq, Wk, 128, 64, 0.05, 0.9)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("dr", [64, 128])
def test_router_long_rows_at_the_block_limit(dr):
    # 4096 key blocks per row, ragged last block: the CTA-per-row selection.
    N = 64 * 4096 - 17
    Q, K, _ = synth.make_qkv(1, 1, N, 64, grid=None, s=1.5, seed=4100)
    Wq, Wk = synth.make_router(1, 64, dr, seed=dr + 1)
    _check(Q, K, Wq, Wk, 128, 64, 0.03, 0.9)
