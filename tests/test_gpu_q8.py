"""Low-bit sparse branch (int8 Q/K codes, e4m3 P and V codes) on the GPU
against the CPU oracle's definition of the same computation.

The oracle takes the plain two-pass definition (the row's integer log2
reference is the ceiling of the max over all of its kept keys); the kernel
moves its reference lazily while it walks the key tiles. The two agree
exactly wherever 2^(x - m) stays in e4m3's normal range and differ by
subnormal rounding below it, so the outputs are held to the general
bars (max-abs 2e-2, mean relative L1 5e-3)."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_pooled_b200 import synth
from parity import assert_outputs, sample_rows

pytestmark = pytest.mark.gpu


def _run(Q, K, V, kv_idx, kv_cnt, bq, bk):
    from block_sparse_attention_pooled_b200 import sparge

    dev = torch.device("cuda")
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    shape = sparge.make_shape(Qd, bq, bk)
    ws = torch.empty(sparge.workspace_bytes(sparge.OP_ATTN_Q8, shape), dtype=torch.uint8, device=dev)
    O = sparge.sparge_attn_fwd_q8(Qd, Kd, Vd, torch.as_tensor(kv_idx).to(dev), torch.as_tensor(kv_cnt).to(dev),
                                  bq, bk, workspace=ws)
    torch.cuda.synchronize()
    assert sparge.device_status() == 0
    return O, ws, shape


@pytest.mark.parametrize("N,bq,bk", [(4096, 128, 64), (1000, 64, 64), (1000, 128, 128), (777, 64, 128)])
def test_q8_codes_match_oracle(N, bq, bk):
    from block_sparse_attention_pooled_b200 import sparge

    Q, K, V = synth.make_qkv(1, 2, N, 128, grid=None, s=2.0, seed=N)
    kv_idx, kv_cnt = synth.random_mask(1, 2, -(-N // bq), -(-N // bk), 3, seed=1)
    _, ws, shape = _run(Q, K, V, kv_idx, kv_cnt, bq, bk)
    q8, k8, v8, sq, sk, sv = (t.cpu() for t in sparge.quant_q8_workspace_views(ws, shape))
    o_q8, o_sq, o_k8, o_sk, o_v8, o_sv = oracle.quant_q8(Q, K, V, bq, bk)
    np.testing.assert_array_equal(sq.numpy(), o_sq)
    np.testing.assert_array_equal(sk.numpy(), o_sk)
    np.testing.assert_array_equal(sv.numpy(), o_sv)
    np.testing.assert_array_equal(q8.numpy(), o_q8)
    np.testing.assert_array_equal(k8.numpy(), o_k8)
    np.testing.assert_array_equal(v8.view(torch.float8_e4m3fn).to(torch.float64).numpy(), o_v8)


@pytest.mark.parametrize("N,bq,bk,mask", [(4096, 128, 64, "oracle"), (1000, 64, 64, "random"),
                                          (1000, 128, 128, "random"), (777, 64, 128, "oracle"),
                                          (4096, 128, 64, "all")])
def test_q8_attention_matches_oracle(N, bq, bk, mask):
    B, H, d = 1, 2, 128
    Q, K, V = synth.make_qkv(B, H, N, d, grid=None, s=2.0, seed=N + bq)
    nqb, nkb = -(-N // bq), -(-N // bk)
    if mask == "oracle":
        kv_idx, kv_cnt, _ = oracle.mask(Q, K, bq, bk, 0.1, 0.9)
    elif mask == "all":
        kv_idx = np.tile(np.arange(nkb, dtype=np.int32), (B, H, nqb, 1))
        kv_cnt = np.full((B, H, nqb), nkb, np.int32)
    else:
        kv_idx, kv_cnt = (np.asarray(a) for a in synth.random_mask(B, H, nqb, nkb, 4, seed=3))
    O, _, _ = _run(Q, K, V, kv_idx, kv_cnt, bq, bk)
    ref = oracle.attention_q8_rows(Q, K, V, bq, bk, kv_idx, kv_cnt)
    got = O.float().cpu().numpy().reshape(-1, d).astype(np.float64)
    max_abs, mean_rel = assert_outputs(got, ref)
    print(f"q8 N={N} bq={bq} bk={bk} mask={mask}: max-abs {max_abs:.2e}, mean-rel-L1 {mean_rel:.2e}")


def test_q8_long_rows_at_the_block_limit():
    # 4096 key blocks per row (the library's maximum), ragged last block: V's
    # channel scales reduce 256 chunk maxima; one query block keeps every
    # key block, the last a scattered half, the rest a few.
    N, bq, bk = 64 * 4096 - 17, 128, 64
    Q, K, V = synth.make_qkv(1, 1, N, 128, grid=None, s=2.0, seed=4099)
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx, kv_cnt = (np.asarray(a) for a in synth.random_mask(1, 1, nqb, nkb, 5, seed=14))
    kv_idx[0, 0, 0] = np.arange(nkb, dtype=np.int32)
    kv_cnt[0, 0, 0] = nkb
    half = np.sort(np.random.default_rng(7).choice(nkb, nkb // 2, replace=False)).astype(np.int32)
    kv_idx[0, 0, nqb - 1, : nkb // 2] = half
    kv_cnt[0, 0, nqb - 1] = nkb // 2
    O, _, _ = _run(Q, K, V, kv_idx, kv_cnt, bq, bk)
    rows = np.concatenate([np.arange(0, 128, 17), np.arange((nqb - 1) * bq, N, 19),
                           np.arange(900 * bq, 900 * bq + 128, 23)]).astype(np.int64)
    ref = oracle.attention_q8_rows(Q, K, V, bq, bk, kv_idx, kv_cnt, rows)
    got = O.float().cpu().numpy().reshape(-1, 128)[rows].astype(np.float64)
    assert_outputs(got, ref)


def test_q8_480p_sampled_rows():
    w = synth.WORKLOADS["480p"]
    Q, K, V, _ = synth.make_workload(w, heads=[(0, 0), (0, 5)])
    kv_idx, kv_cnt, _ = oracle.mask(Q, K, w.bq, w.bk, w.topk, w.topp)
    O, _, _ = _run(Q, K, V, kv_idx, kv_cnt, w.bq, w.bk)
    rows = sample_rows(Q.shape[0], Q.shape[1], w.N, w.bq, 96, seed=4)
    ref = oracle.attention_q8_rows(Q, K, V, w.bq, w.bk, kv_idx, kv_cnt, rows)
    got = O.float().cpu().numpy().reshape(-1, w.d)[rows].astype(np.float64)
    assert_outputs(got, ref)


def test_q8_is_deterministic():
    Q, K, V = synth.make_qkv(1, 2, 2048, 128, grid=None, s=2.0, seed=9)
    kv_idx, kv_cnt, _ = oracle.mask(Q, K, 128, 64, 0.1, 0.9)
    a, _, _ = _run(Q, K, V, kv_idx, kv_cnt, 128, 64)
    b, _, _ = _run(Q, K, V, kv_idx, kv_cnt, 128, 64)
    assert torch.equal(a, b)
