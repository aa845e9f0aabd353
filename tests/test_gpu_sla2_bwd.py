"""SLA2 backward (sparse + linear branches and the alpha mix) on the GPU
against the CPU oracle's gradients (fp64, chain rule of the forward)."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_pooled_b200 import synth
from test_gpu_bwd import _assert_grad, _kblocks_layout, _masks

pytestmark = pytest.mark.gpu


def _run(Q, K, V, dO, kv_idx, kv_cnt, alpha, bq, bk):
    from block_sparse_attention_pooled_b200 import sparge

    dev = torch.device("cuda")
    idx, cnt = torch.as_tensor(np.asarray(kv_idx)).to(dev), torch.as_tensor(np.asarray(kv_cnt)).to(dev)
    out = sparge.sla2_attn_bwd(Q.to(dev), K.to(dev), V.to(dev), idx, cnt, alpha.to(dev), dO.to(dev), bq, bk)
    torch.cuda.synchronize()
    assert sparge.device_status() == 0
    return out


@pytest.mark.parametrize("N,bq,bk,kind", [(1000, 128, 64, "oracle"), (1000, 64, 64, "random"),
                                          (777, 64, 128, "random"), (4096, 128, 64, "oracle"),
                                          (2048, 128, 64, "all")])
def test_sla2_bwd_matches_oracle(N, bq, bk, kind):
    Q, K, V = synth.make_qkv(1, 2, N, 128, grid=None, s=1.5, seed=N + bk)
    dO = synth.make_dout(1, 2, N, 128, seed=N + 1)
    alpha = torch.tensor([0.7, 0.9], dtype=torch.float32)
    kv_idx, kv_cnt = _masks(Q, K, bq, bk, kind, seed=N)
    dQ, dK, dV, da = _run(Q, K, V, dO, kv_idx, kv_cnt, alpha, bq, bk)
    rQ, rK, rV, ra = oracle.attention_bwd(Q, K, V, dO, bq, bk, kv_idx, kv_cnt, alpha=alpha, mode="sla2",
                                          want_dalpha=True)
    _assert_grad("dQ", dQ.float().cpu().numpy().reshape(-1, 128), rQ)
    _assert_grad("dK", _kblocks_layout(dK, bk), rK)
    _assert_grad("dV", _kblocks_layout(dV, bk), rV)
    got = da.cpu().numpy().astype(np.float64)
    print("dalpha", got, ra)
    np.testing.assert_allclose(got, ra, rtol=1e-2, atol=1e-2 * np.abs(ra).max())


def test_sla2_bwd_many_short_heads():
    # Short heads: the summary kernel's runs (forward summaries and the
    # gradient summaries G_all, g_all) cross three or more heads per CTA.
    B, H, N, bq, bk = 1, 750, 100, 64, 64
    Q, K, V = synth.make_qkv(B, H, N, 128, grid=None, s=1.5, seed=31)
    dO = synth.make_dout(B, H, N, 128, seed=32)
    alpha = torch.linspace(0.6, 0.95, H, dtype=torch.float32)
    kv_idx, kv_cnt = synth.random_mask(B, H, -(-N // bq), -(-N // bk), 2, seed=33)
    kv_idx, kv_cnt = kv_idx.numpy(), kv_cnt.numpy()
    dQ, dK, dV, da = _run(Q, K, V, dO, kv_idx, kv_cnt, alpha, bq, bk)
    rQ, rK, rV, ra = oracle.attention_bwd(Q, K, V, dO, bq, bk, kv_idx, kv_cnt, alpha=alpha, mode="sla2",
                                          want_dalpha=True)
    _assert_grad("dQ", dQ.float().cpu().numpy().reshape(-1, 128), rQ)
    _assert_grad("dK", _kblocks_layout(dK, bk), rK)
    _assert_grad("dV", _kblocks_layout(dV, bk), rV)
    got = da.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got, ra, rtol=1e-2, atol=1e-2 * np.abs(ra).max())


def test_sla2_bwd_alpha_one_is_the_sparse_backward():
    # alpha = 1: the linear branch carries no weight, so every linear term is an
    # exact zero and the gradients equal the sparse backward's bit for bit.
    from block_sparse_attention_pooled_b200 import sparge

    N, bq, bk = 2048, 128, 64
    Q, K, V = synth.make_qkv(1, 2, N, 128, grid=None, s=1.5, seed=12)
    dO = synth.make_dout(1, 2, N, 128, seed=12)
    kv_idx, kv_cnt = _masks(Q, K, bq, bk, "oracle", 0)
    dQ, dK, dV, _ = _run(Q, K, V, dO, kv_idx, kv_cnt, torch.ones(2), bq, bk)
    dev = torch.device("cuda")
    Qd, Kd, Vd, dOd = Q.to(dev), K.to(dev), V.to(dev), dO.to(dev)
    idx, cnt = torch.as_tensor(kv_idx).to(dev), torch.as_tensor(kv_cnt).to(dev)
    lse = torch.empty((1, 2, N), dtype=torch.float32, device=dev)
    O = sparge.sparge_attn_fwd(Qd, Kd, Vd, idx, cnt, bq, bk, lse=lse)
    sQ, sK, sV = sparge.sparge_attn_bwd(Qd, Kd, Vd, idx, cnt, O, lse, dOd, bq, bk)
    torch.cuda.synchronize()
    assert torch.equal(dQ, sQ) and torch.equal(dK, sK) and torch.equal(dV, sV)


def test_sla2_bwd_sampled_workload():
    # Full-size check on sampled query rows (dQ). A key's linear-branch gradient
    # sums over every query row of its head, so the oracle's dK / dV of one key
    # block costs N^2 d here; those are checked at the sizes above.
    w = synth.WORKLOADS["sla2_480p"]
    heads = [(0, 3), (1, 8)]
    Q, K, V, alpha = synth.make_workload(w, heads=heads)
    al = torch.tensor([float(alpha[h]) for _, h in heads], dtype=torch.float32)
    dO = synth.make_dout(w.B, w.H, w.N, w.d, seed=2, heads=heads)
    kv_idx, kv_cnt, _ = oracle.mask(Q, K, w.bq, w.bk, w.topk, w.topp)
    dQ, dK, dV, _ = _run(Q, K, V, dO, kv_idx, kv_cnt, al, w.bq, w.bk)
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(2 * w.N, 24, replace=False))
    rQ, _, _, _ = oracle.attention_bwd(Q, K, V, dO, w.bq, w.bk, kv_idx, kv_cnt, alpha=al, mode="sla2",
                                       rows=rows, kblocks=np.zeros(0, np.int64))
    _assert_grad("dQ", dQ.float().cpu().numpy().reshape(-1, w.d)[rows], rQ)
    assert torch.isfinite(dK.float()).all() and torch.isfinite(dV.float()).all()


def test_sla2_bwd_is_deterministic():
    Q, K, V = synth.make_qkv(1, 2, 2048, 128, grid=None, s=1.5, seed=13)
    dO = synth.make_dout(1, 2, 2048, 128, seed=13)
    kv_idx, kv_cnt = _masks(Q, K, 128, 64, "oracle", 0)
    alpha = torch.tensor([0.6, 0.8], dtype=torch.float32)
    a = _run(Q, K, V, dO, kv_idx, kv_cnt, alpha, 128, 64)
    b = _run(Q, K, V, dO, kv_idx, kv_cnt, alpha, 128, 64)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
