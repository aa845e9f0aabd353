"""GPU block mask vs the CPU oracle's double-precision definition.

The kept sets must be identical except where the ambiguity rule allows a
difference (a block within 1e-6 relative of the row's threshold probability,
or a Top-p boundary whose running sum lies within 1e-6 of p); such rows are
counted and printed. The probabilities and the row thresholds the GPU
returns (rounded to float) must equal the oracle's to float rounding."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_pooled_b200 import synth
from parity import check_mask_outputs

pytestmark = pytest.mark.gpu


def _run(Q, K, bq, bk, topk, topp):
    from block_sparse_attention_pooled_b200 import sparge

    dev = torch.device("cuda")
    Qd, Kd = Q.to(dev), K.to(dev)
    B, H, N, d = Q.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    probs = torch.empty((B, H, nqb, nkb), dtype=torch.float32, device=dev)
    thr = torch.empty((B, H, nqb), dtype=torch.float32, device=dev)
    idx, cnt = sparge.sparge_mask(Qd, Kd, bq, bk, topk, topp, row_thresh=thr, probs=probs)
    torch.cuda.synchronize()
    assert sparge.device_status() == 0
    return idx.cpu().numpy(), cnt.cpu().numpy(), probs.cpu().numpy(), thr.cpu().numpy()


def _check(Q, K, bq, bk, topk, topp, what=""):
    g = _run(Q, K, bq, bk, topk, topp)
    o_idx, o_cnt, o_P = oracle.mask(Q, K, bq, bk, topk, topp)
    n, bad, amb = check_mask_outputs(g, (o_idx, o_cnt, o_P), topk, topp)
    if what:
        print(f"{what}: rows {n}, rows differing from the fp64 definition {bad} (all within the ambiguity rule)")
    return n, bad, amb


@pytest.mark.parametrize("N,d,bq,bk", [(4096, 64, 64, 64), (1000, 64, 64, 64), (1000, 128, 128, 64),
                                        (777, 128, 64, 128), (130, 64, 128, 128), (64, 128, 64, 64)])
@pytest.mark.parametrize("topk,topp", [(0.1, 0.9), (0.0, 0.9), (0.2, 0.0), (0.0, 0.0), (1.0, 0.5), (0.05, 1.0)])
def test_mask_small(N, d, bq, bk, topk, topp):
    Q, K, _ = synth.make_qkv(1, 2, N, d, grid=None, s=1.5, seed=N + d)
    _check(Q, K, bq, bk, topk, topp)


@pytest.mark.parametrize("nkb,topk,topp", [(2048, 0.03, 0.9), (2049, 0.03, 0.9), (2049, 0.0, 0.5),
                                           (4096, 0.01, 0.0), (4096, 0.03, 0.9)])
def test_mask_long_rows(nkb, topk, topp):
    # Rows of up to 2048 blocks take the warp-per-row selection (2048 is its
    # limit); longer rows take the CTA-per-row kernel, up to the 4096-block
    # maximum the library accepts. The last key block is ragged.
    N = nkb * 64 - 17
    Q, K, _ = synth.make_qkv(1, 1, N, 64, grid=None, s=1.5, seed=nkb)
    _check(Q, K, 128, 64, topk, topp)


@pytest.mark.parametrize("name", ["tiny", "480p", "sla2_480p", "sweep_flat", "sweep_peaked"])
def test_mask_workloads(name):
    w = synth.WORKLOADS[name]
    Q, K, _, _ = synth.make_workload(w)
    _check(Q, K, w.bq, w.bk, w.topk, w.topp, what=name)


def test_mask_720p_all_heads():
    w = synth.WORKLOADS["720p"]
    Q, K, _, _ = synth.make_workload(w)
    _check(Q, K, w.bq, w.bk, w.topk, w.topp, what="720p")


@pytest.mark.parametrize("topk,topp", [(t, p) for t in synth.SWEEP_TOPK for p in synth.SWEEP_TOPP]
                         + [(0.05, 0.0), (0.0, 0.9)])
def test_mask_sweep_regimes(topk, topp):
    for name in ("sweep_flat", "sweep_peaked"):
        w = synth.WORKLOADS[name]
        Q, K, _ = synth.make_qkv(1, 4, w.N, w.d, w.grid, w.s, w.seed)
        _check(Q, K, w.bq, w.bk, topk, topp, what=f"{name} k={topk} p={topp} (4 heads)")


def test_mask_is_deterministic():
    from block_sparse_attention_pooled_b200 import sparge

    w = synth.WORKLOADS["480p"]
    Q, K, _ = synth.make_qkv(1, 3, w.N, w.d, w.grid, w.s, w.seed)
    Qd, Kd = Q.cuda(), K.cuda()
    a = [t.clone() for t in sparge.sparge_mask(Qd, Kd, w.bq, w.bk, w.topk, w.topp)]
    b = sparge.sparge_mask(Qd, Kd, w.bq, w.bk, w.topk, w.topp)
    cnt = a[1]
    assert torch.equal(a[1], b[1])
    cols = torch.arange(a[0].shape[-1], device=cnt.device)
    valid = cols[None, None, None, :] < cnt[..., None]
    assert torch.equal(a[0][valid], b[0][valid])


@pytest.mark.parametrize("topk,topp", [(0.1, 0.0), (0.0, 0.3), (0.05, 0.5), (0.0, 1.0)])
def test_mask_exact_ties_take_lower_indices(topk, topp):
    # Every key block holds the same rows, so every pooled score of a row is
    # the same number on both sides: all probabilities tie exactly and the
    # kept blocks must be the lowest indices, in the counts the oracle gives.
    B, H, N, d, bq, bk = 1, 2, 4096, 64, 64, 64
    Q, K, _ = synth.make_qkv(B, H, N, d, grid=None, s=1.5, seed=77)
    K = K[:, :, :bk].repeat(1, 1, N // bk, 1).contiguous()
    g_idx, g_cnt, g_P, _ = _run(Q, K, bq, bk, topk, topp)
    o_idx, o_cnt, o_P = oracle.mask(Q, K, bq, bk, topk, topp)
    np.testing.assert_array_equal(g_P, o_P.astype(np.float32))
    np.testing.assert_array_equal(g_cnt, o_cnt)
    for r, c in enumerate(g_cnt.reshape(-1)):
        np.testing.assert_array_equal(g_idx.reshape(-1, g_idx.shape[-1])[r, :c], np.arange(c))
        np.testing.assert_array_equal(o_idx.reshape(-1, o_idx.shape[-1])[r, :c], np.arange(c))


@pytest.mark.parametrize("s", [20.0, 60.0])
@pytest.mark.parametrize("topk,topp", [(0.5, 0.0), (0.9, 0.0), (1.0, 0.0), (0.0, 1.0), (0.3, 0.99)])
def test_mask_with_underflowing_probabilities(s, topk, topp):
    # Very wide score ranges: most of a row's probabilities are exactly 0 in
    # double or lie more than 255 binades below its largest, so the
    # selection's threshold falls among keys of mixed binades (and among
    # exact zeros, which tie and go to the lower indices).
    Q, K, _ = synth.make_qkv(1, 2, 4096, 64, grid=None, s=s, seed=123)
    _check(Q, K, 64, 64, topk, topp, what=f"s={s} k={topk} p={topp}")
