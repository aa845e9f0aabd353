"""GPU block-sparse attention vs the double-precision oracle on the same
(oracle-computed) block mask."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_pooled_b200 import synth
from parity import assert_outputs, sample_rows

pytestmark = pytest.mark.gpu


def _gpu_attn(Q, K, V, idx, cnt, bq, bk, with_lse=True):
    from block_sparse_attention_pooled_b200 import sparge

    dev = torch.device("cuda")
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    idx_d = torch.as_tensor(idx, dtype=torch.int32).to(dev)
    cnt_d = torch.as_tensor(cnt, dtype=torch.int32).to(dev)
    B, H, N, d = Q.shape
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev) if with_lse else None
    O = sparge.sparge_attn_fwd(Qd, Kd, Vd, idx_d, cnt_d, bq, bk, lse=lse)
    torch.cuda.synchronize()
    assert sparge.device_status() == 0
    return O.float().cpu().numpy(), (lse.cpu().numpy() if with_lse else None)


def _check_rows(Q, K, V, idx, cnt, bq, bk, rows=None):
    B, H, N, d = Q.shape
    O, lse = _gpu_attn(Q, K, V, idx, cnt, bq, bk)
    ref, ref_lse = oracle.attention_rows(Q, K, V, bq, bk, idx, cnt, mode="sparse", rows=rows)
    got = O.reshape(-1, d) if rows is None else O.reshape(-1, d)[rows]
    got_lse = lse.reshape(-1) if rows is None else lse.reshape(-1)[rows]
    errs = assert_outputs(got, ref, "sparse attention")
    fin = np.isfinite(ref_lse)
    np.testing.assert_allclose(got_lse[fin], ref_lse[fin], atol=2e-3, rtol=1e-4)
    assert np.all(np.isneginf(got_lse[~fin]))
    return errs


@pytest.mark.parametrize("N,d,bq,bk", [(4096, 64, 64, 64), (1000, 128, 128, 64), (1000, 64, 64, 64),
                                        (777, 128, 64, 128), (130, 64, 128, 128), (64, 128, 128, 64),
                                        (1, 128, 128, 64), (2000, 128, 128, 128)])
def test_attn_random_masks(N, d, bq, bk):
    Q, K, V = synth.make_qkv(1, 2, N, d, grid=None, s=1.5, seed=N * 3 + d)
    nqb, nkb = -(-N // bq), -(-N // bk)
    idx, cnt = synth.random_mask(1, 2, nqb, nkb, min(nkb, 9), seed=N)
    _check_rows(Q, K, V, idx.numpy(), cnt.numpy(), bq, bk)


def test_attn_all_blocks_kept_equals_dense():
    N, d, bq, bk = 1500, 128, 128, 64
    Q, K, V = synth.make_qkv(1, 2, N, d, grid=None, s=1.0, seed=7)
    nqb, nkb = -(-N // bq), -(-N // bk)
    idx = np.tile(np.arange(nkb, dtype=np.int32), (1, 2, nqb, 1))
    cnt = np.full((1, 2, nqb), nkb, np.int32)
    O, _ = _gpu_attn(Q, K, V, idx, cnt, bq, bk)
    ref, _ = oracle.attention_rows(Q, K, V, bq, bk, mode="dense")
    assert_outputs(O.reshape(-1, d), ref, "dense via all blocks")


def test_attn_empty_rows_are_zero():
    N, d, bq, bk = 512, 128, 128, 64
    Q, K, V = synth.make_qkv(1, 1, N, d, grid=None, s=1.0, seed=8)
    idx = np.zeros((1, 1, 4, 8), np.int32)
    cnt = np.array([[[0, 3, 0, 8]]], np.int32)
    idx[0, 0, 1, :3] = [0, 4, 7]
    idx[0, 0, 3, :] = np.arange(8)
    O, lse = _gpu_attn(Q, K, V, idx, cnt, bq, bk)
    assert np.all(O[0, 0, :128] == 0) and np.all(O[0, 0, 256:384] == 0)
    assert np.all(np.isneginf(lse[0, 0, :128]))
    _check_rows(Q, K, V, idx, cnt, bq, bk)


def test_attn_peaked_scores_rescale_path():
    # Large score spread forces the online softmax to move its reference max.
    N, d, bq, bk = 1024, 128, 128, 64
    Q, K, V = synth.make_qkv(1, 2, N, d, grid=None, s=4.0, seed=9)
    nqb, nkb = N // bq, N // bk
    idx = np.tile(np.arange(nkb, dtype=np.int32), (1, 2, nqb, 1))
    cnt = np.full((1, 2, nqb), nkb, np.int32)
    _check_rows(Q, K, V, idx, cnt, bq, bk)


def test_attn_long_rows_at_the_block_limit():
    # 4096 key blocks per row (the library's maximum) with a ragged last
    # block: one query block keeps every block (4096 kept-list entries, read
    # 32 at a time), one keeps a scattered half, the rest keep a few.
    N, d, bq, bk = 64 * 4096 - 17, 64, 128, 64
    Q, K, V = synth.make_qkv(1, 1, N, d, grid=None, s=1.5, seed=4096)
    nqb, nkb = -(-N // bq), -(-N // bk)
    idx, cnt = (np.asarray(a) for a in synth.random_mask(1, 1, nqb, nkb, 6, seed=11))
    idx[0, 0, 0] = np.arange(nkb, dtype=np.int32)
    cnt[0, 0, 0] = nkb
    half = np.sort(np.random.default_rng(5).choice(nkb, nkb // 2, replace=False)).astype(np.int32)
    idx[0, 0, nqb - 1, : nkb // 2] = half
    cnt[0, 0, nqb - 1] = nkb // 2
    rows = np.concatenate([np.arange(0, 128, 5), np.arange((nqb - 1) * bq, N, 7), np.arange(700 * bq, 700 * bq + 64, 9)])
    _check_rows(Q, K, V, idx, cnt, bq, bk, rows=rows.astype(np.int64))


@pytest.mark.parametrize("name", ["tiny", "480p"])
def test_attn_workload_oracle_mask(name):
    w = synth.WORKLOADS[name]
    Q, K, V, _ = synth.make_workload(w)
    idx, cnt, _ = oracle.mask(Q, K, w.bq, w.bk, w.topk, w.topp)
    rows = None if name == "tiny" else sample_rows(w.B, w.H, w.N, w.bq, 96, seed=1)
    max_abs, mean_rel = _check_rows(Q, K, V, idx, cnt, w.bq, w.bk, rows=rows)
    print(f"{name}: max-abs {max_abs:.2e} mean-rel-L1 {mean_rel:.2e}")


def test_attn_is_deterministic():
    N, d = 3000, 128
    Q, K, V = synth.make_qkv(1, 2, N, d, grid=None, s=2.0, seed=10)
    idx, cnt = synth.random_mask(1, 2, -(-N // 128), -(-N // 64), 12, seed=3)
    a, _ = _gpu_attn(Q, K, V, idx.numpy(), cnt.numpy(), 128, 64)
    b, _ = _gpu_attn(Q, K, V, idx.numpy(), cnt.numpy(), 128, 64)
    assert np.array_equal(a, b)
