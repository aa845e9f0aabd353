"""Sparse-branch backward on the GPU against the CPU oracle's gradients
(fp64, from the chain rule of the forward's definition)."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_pooled_b200 import synth

pytestmark = pytest.mark.gpu


def _fwd_bwd(Q, K, V, dO, kv_idx, kv_cnt, bq, bk):
    from block_sparse_attention_pooled_b200 import sparge

    dev = torch.device("cuda")
    Qd, Kd, Vd, dOd = Q.to(dev), K.to(dev), V.to(dev), dO.to(dev)
    idx, cnt = torch.as_tensor(np.asarray(kv_idx)).to(dev), torch.as_tensor(np.asarray(kv_cnt)).to(dev)
    B, H, N, d = Q.shape
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    O = sparge.sparge_attn_fwd(Qd, Kd, Vd, idx, cnt, bq, bk, lse=lse)
    dQ, dK, dV = sparge.sparge_attn_bwd(Qd, Kd, Vd, idx, cnt, O, lse, dOd, bq, bk)
    torch.cuda.synchronize()
    assert sparge.device_status() == 0
    return dQ, dK, dV


def _kblocks_layout(x, bk):
    """[B,H,N,d] tensor as the oracle's [B*H*Nkb, bk, d] (rows past N zero)."""
    B, H, N, d = x.shape
    nkb = -(-N // bk)
    out = np.zeros((B * H, nkb * bk, d))
    out[:, :N] = x.float().cpu().numpy().reshape(B * H, N, d)
    return out.reshape(B * H * nkb, bk, d)


def _errs(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    return np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30), np.abs(got - ref).sum() / max(np.abs(ref).sum(), 1e-30)


def _assert_grad(name, got, ref):
    mx, rel = _errs(got, ref)
    print(f"{name}: max-abs / max|ref| {mx:.2e}, rel-L1 {rel:.2e}")
    assert mx <= 2e-2 and rel <= 1e-2, (name, mx, rel)


def _masks(Q, K, bq, bk, kind, seed):
    B, H, N, _ = Q.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    if kind == "oracle":
        kv_idx, kv_cnt, _ = oracle.mask(Q, K, bq, bk, 0.1, 0.9)
    elif kind == "all":
        kv_idx = np.tile(np.arange(nkb, dtype=np.int32), (B, H, nqb, 1))
        kv_cnt = np.full((B, H, nqb), nkb, np.int32)
    else:
        kv_idx, kv_cnt = (np.asarray(a) for a in synth.random_mask(B, H, nqb, nkb, 4, seed=seed))
    return kv_idx, kv_cnt


@pytest.mark.parametrize("N,bq,bk,kind", [(1000, 128, 64, "oracle"), (1000, 64, 64, "random"),
                                          (777, 64, 128, "random"), (4096, 128, 64, "oracle"),
                                          (130, 128, 128, "all"), (2048, 128, 64, "all")])
def test_bwd_matches_oracle(N, bq, bk, kind):
    Q, K, V = synth.make_qkv(1, 2, N, 128, grid=None, s=1.5, seed=N + bq)
    dO = synth.make_dout(1, 2, N, 128, seed=N)
    kv_idx, kv_cnt = _masks(Q, K, bq, bk, kind, seed=N)
    dQ, dK, dV = _fwd_bwd(Q, K, V, dO, kv_idx, kv_cnt, bq, bk)
    rQ, rK, rV, _ = oracle.attention_bwd(Q, K, V, dO, bq, bk, kv_idx, kv_cnt, mode="sparse")
    _assert_grad("dQ", dQ.float().cpu().numpy().reshape(-1, 128), rQ)
    _assert_grad("dK", _kblocks_layout(dK, bk), rK)
    _assert_grad("dV", _kblocks_layout(dV, bk), rV)


def test_bwd_zero_where_nothing_flows():
    # Rows whose block keeps nothing get dQ = 0; keys that no block keeps get dK = dV = 0.
    N, bq, bk = 1024, 128, 64
    Q, K, V = synth.make_qkv(1, 2, N, 128, grid=None, s=1.5, seed=5)
    dO = synth.make_dout(1, 2, N, 128, seed=5)
    nqb, nkb = N // bq, N // bk
    kv_idx = np.zeros((1, 2, nqb, nkb), np.int32)
    kv_cnt = np.zeros((1, 2, nqb), np.int32)
    kv_idx[0, :, ::2, :3] = [1, 4, 9]
    kv_cnt[0, :, ::2] = 3
    dQ, dK, dV = _fwd_bwd(Q, K, V, dO, kv_idx, kv_cnt, bq, bk)
    for I in range(1, nqb, 2):
        assert torch.count_nonzero(dQ[0, :, I * bq:(I + 1) * bq]) == 0
    kept = {1, 4, 9}
    for J in range(nkb):
        sl = slice(J * bk, (J + 1) * bk)
        if J not in kept:
            assert torch.count_nonzero(dK[0, :, sl]) == 0 and torch.count_nonzero(dV[0, :, sl]) == 0
        else:
            assert torch.count_nonzero(dV[0, :, sl]) > 0


def test_bwd_480p_sampled():
    w = synth.WORKLOADS["480p"]
    heads = [(0, 0), (0, 7)]
    Q, K, V, _ = synth.make_workload(w, heads=heads)
    dO = synth.make_dout(w.B, w.H, w.N, w.d, seed=1, heads=heads)
    kv_idx, kv_cnt, _ = oracle.mask(Q, K, w.bq, w.bk, w.topk, w.topp)
    dQ, dK, dV = _fwd_bwd(Q, K, V, dO, kv_idx, kv_cnt, w.bq, w.bk)
    rng = np.random.default_rng(3)
    rows = np.sort(rng.choice(2 * w.N, 64, replace=False))
    kb = np.sort(rng.choice(2 * w.nkb, 6, replace=False))
    rQ, rK, rV, _ = oracle.attention_bwd(Q, K, V, dO, w.bq, w.bk, kv_idx, kv_cnt, mode="sparse", rows=rows,
                                         kblocks=kb)
    _assert_grad("dQ", dQ.float().cpu().numpy().reshape(-1, w.d)[rows], rQ)
    _assert_grad("dK", _kblocks_layout(dK, w.bk)[kb], rK)
    _assert_grad("dV", _kblocks_layout(dV, w.bk)[kb], rV)


def test_bwd_long_rows_at_the_block_limit():
    # 4096 key blocks per row (the library's maximum), ragged last block: the
    # first query block keeps every key block, the rest a few each. dQ is
    # checked on rows of the full block and of the ragged last query block,
    # dK and dV on the ragged last key block (which the full row keeps).
    N, d, bq, bk = 64 * 4096 - 17, 128, 128, 64
    Q, K, V = synth.make_qkv(1, 1, N, d, grid=None, s=1.5, seed=4097)
    dO = synth.make_dout(1, 1, N, d, seed=4097)
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx, kv_cnt = (np.asarray(a) for a in synth.random_mask(1, 1, nqb, nkb, 4, seed=12))
    kv_idx[0, 0, 0] = np.arange(nkb, dtype=np.int32)
    kv_cnt[0, 0, 0] = nkb
    dQ, dK, dV = _fwd_bwd(Q, K, V, dO, kv_idx, kv_cnt, bq, bk)
    rows = np.concatenate([np.arange(0, 128, 11), np.arange((nqb - 1) * bq, N, 13)]).astype(np.int64)
    kb = np.array([nkb - 1], np.int64)
    rQ, rK, rV, _ = oracle.attention_bwd(Q, K, V, dO, bq, bk, kv_idx, kv_cnt, mode="sparse", rows=rows, kblocks=kb)
    _assert_grad("dQ", dQ.float().cpu().numpy().reshape(-1, d)[rows], rQ)
    _assert_grad("dK", _kblocks_layout(dK, bk)[kb], rK)
    _assert_grad("dV", _kblocks_layout(dV, bk)[kb], rV)


def test_bwd_is_deterministic():
    Q, K, V = synth.make_qkv(1, 2, 4096, 128, grid=None, s=1.5, seed=11)
    dO = synth.make_dout(1, 2, 4096, 128, seed=11)
    kv_idx, kv_cnt = _masks(Q, K, 128, 64, "oracle", 0)
    a = _fwd_bwd(Q, K, V, dO, kv_idx, kv_cnt, 128, 64)
    b = _fwd_bwd(Q, K, V, dO, kv_idx, kv_cnt, 128, 64)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
