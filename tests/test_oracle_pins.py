"""Pins for the CPU oracle against facts that do not come from the oracle itself.

Each test ties one oracle function to a library routine it does not call, a
closed form, an invariant, hand-derived golden values or exact brute force.
Sources of the rules: SpargeAttention2 article (arXiv:2602.13515) sections 1
and 4; SLA2 article (arXiv:2602.12675) sections 1 and 2.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from block_sparse_attention_pooled_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "select_rows.json")


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def _rand_qkv(B, H, N, d, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    q = _bf16(torch.randn(B, H, N, d, generator=g) * scale)
    k = _bf16(torch.randn(B, H, N, d, generator=g) * scale)
    v = _bf16(torch.randn(B, H, N, d, generator=g))
    return q, k, v


def _block_bool_mask(kv_idx, kv_cnt, N, bq, bk):
    """[B,H,N,N] boolean key mask expanded from block lists (test-side helper)."""
    B, H, nqb, nkb = kv_idx.shape
    m = np.zeros((B, H, N, N), bool)
    for b in range(B):
        for h in range(H):
            for I in range(nqb):
                for e in range(int(kv_cnt[b, h, I])):
                    J = int(kv_idx[b, h, I, e])
                    m[b, h, I * bq:(I + 1) * bq, J * bk:(J + 1) * bk] = True
    return m


def _phi_torch(x):
    return F.elu(x) + 1.0


# ----------------------------------------------------------------------------- pooling
def test_pool_full_blocks_match_avg_pool(oracle_mod):
    q, _, _ = _rand_qkv(1, 2, 256, 16, 1)
    got = oracle_mod.pool(q, 64)
    x = q.double().reshape(2, 256, 16).transpose(1, 2)  # (BH, d, N)
    ref = F.avg_pool1d(x, kernel_size=64, stride=64).transpose(1, 2).reshape(1, 2, 4, 16)
    np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


def test_pool_ragged_block_averages_valid_rows_only(oracle_mod):
    # N = 70 with blocks of 64: the last block holds rows 64..69 only.
    x = torch.zeros(1, 1, 70, 4)
    x[0, 0, :64] = 3.0
    x[0, 0, 64:] = torch.arange(6, dtype=torch.float32)[:, None]  # rows 0..5 -> mean 2.5
    got = oracle_mod.pool(_bf16(x), 64)
    assert got.shape == (1, 1, 2, 4)
    np.testing.assert_array_equal(got[0, 0, 0], 3.0)
    np.testing.assert_array_equal(got[0, 0, 1], 2.5)


# ----------------------------------------------------------------------------- block scores
def test_block_probs_match_torch_softmax(oracle_mod):
    g = torch.Generator().manual_seed(3)
    qb = torch.randn(1, 2, 5, 16, generator=g, dtype=torch.float64) * 2
    kb = torch.randn(1, 2, 9, 16, generator=g, dtype=torch.float64) * 2
    got = oracle_mod.block_probs(qb.numpy(), kb.numpy())
    ref = torch.softmax(qb @ kb.transpose(-1, -2) / math.sqrt(16), dim=-1)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(got.sum(-1), 1.0, atol=1e-12)


# ----------------------------------------------------------------------------- selection
def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_select_golden_rows(oracle_mod, case):
    P = np.array([float(Fraction(p)) for p in case["P"]])
    r = oracle_mod.select_row(P, case["topk"], case["topp"])
    assert r["kc"] == case["kc"]
    assert r["pc"] == case["pc"]
    assert r["kept"].tolist() == case["kept"]


def _brute_select(P_frac, topk, topp):
    """Exact selection by brute force: ranks from pairwise comparison, running
    sums in exact rational arithmetic."""
    n = len(P_frac)
    rank = [sum(1 for i in range(n) if P_frac[i] > P_frac[j] or (P_frac[i] == P_frac[j] and i < j))
            for j in range(n)]
    order = sorted(range(n), key=lambda j: rank[j])
    kc = min(n, math.ceil(Fraction(topk).limit_denominator(10**9) * n)) if topk > 0 else 0
    pc = 0
    if topp > 0:
        pc = n
        run = Fraction(0)
        for m in range(1, n + 1):
            run += P_frac[order[m - 1]]
            if run >= Fraction(topp):
                pc = m
                break
    m = max(kc, pc, 1)
    return sorted(order[:m]), kc, pc


def test_select_matches_exact_brute_force():
    import oracle

    rng = np.random.default_rng(7)
    for trial in range(400):
        n = int(rng.integers(1, 9))
        # Dyadic weights with frequent ties, normalised exactly.
        w = rng.integers(0, 5, size=n)
        if w.sum() == 0:
            w[0] = 1
        tot = int(w.sum())
        # Scale to a power-of-two denominator so doubles hold the values exactly.
        den = 1 << 12
        num = [int(x) * den // tot for x in w]
        P_frac = [Fraction(x, den) for x in num]
        P = np.array([float(x) for x in P_frac])
        topk = float(rng.choice([0.0, 0.125, 0.25, 0.5, 1.0]))
        topp = float(rng.choice([0.0, 0.25, 0.5, 0.75, 0.875, 1.0]))
        kept, kc, pc = _brute_select(P_frac, topk, topp)
        r = oracle.select_row(P, topk, topp)
        assert (r["kc"], r["pc"]) == (kc, pc), (P_frac, topk, topp)
        assert r["kept"].tolist() == kept, (P_frac, topk, topp)


def test_select_invariants_random_rows(oracle_mod):
    rng = np.random.default_rng(11)
    for trial in range(200):
        n = int(rng.integers(1, 300))
        P = rng.dirichlet(np.full(n, float(rng.choice([0.05, 1.0, 20.0]))))
        topk, topp = float(rng.uniform(0, 0.3)), float(rng.uniform(0, 1))
        r = oracle_mod.select_row(P, topk, topp)
        kept = set(r["kept"].tolist())
        order = r["order"].tolist()
        assert r["kept"].tolist() == sorted(kept)  # ascending, unique
        assert set(order[: r["kc"]]) <= kept  # mask contains the Top-k set
        assert set(order[: r["pc"]]) <= kept  # mask contains the Top-p set
        assert len(kept) == max(r["kc"], r["pc"], 1)
        if r["pc"] > 0 and r["pc"] < n:
            assert r["cum"][r["pc"]] >= topp > r["cum"][r["pc"] - 1]


# ----------------------------------------------------------------------------- attention
def test_dense_matches_sdpa(oracle_mod):
    q, k, v = _rand_qkv(1, 2, 200, 16, 21, scale=1.5)
    O, lse = oracle_mod.attention_rows(q, k, v, 64, 32, mode="dense")
    ref = F.scaled_dot_product_attention(q.double(), k.double(), v.double())
    np.testing.assert_allclose(O.reshape(1, 2, 200, 16), ref.numpy(), rtol=0, atol=1e-12)
    s = (q.double() @ k.double().transpose(-1, -2)) / math.sqrt(16)
    np.testing.assert_allclose(lse.reshape(1, 2, 200), torch.logsumexp(s, -1).numpy(), atol=1e-12)


@pytest.mark.parametrize("N,bq,bk", [(200, 64, 32), (256, 128, 64), (130, 128, 64)])
def test_sparse_matches_masked_sdpa(oracle_mod, N, bq, bk):
    q, k, v = _rand_qkv(1, 2, N, 16, 22, scale=1.5)
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx, kv_cnt = synth.random_mask(1, 2, nqb, nkb, nkb, seed=N)
    # masked SDPA needs at least one key per row: give empty rows block 0
    empty = kv_cnt == 0
    kv_cnt[empty] = 1
    kv_idx[..., 0][empty] = 0
    O, lse = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode="sparse")
    m = torch.from_numpy(_block_bool_mask(kv_idx.numpy(), kv_cnt.numpy(), N, bq, bk))
    ref = F.scaled_dot_product_attention(q.double(), k.double(), v.double(), attn_mask=m)
    np.testing.assert_allclose(O.reshape(1, 2, N, 16), ref.numpy(), rtol=0, atol=1e-12)
    s = (q.double() @ k.double().transpose(-1, -2)) / math.sqrt(16)
    s = s.masked_fill(~m, -math.inf)
    np.testing.assert_allclose(lse.reshape(1, 2, N), torch.logsumexp(s, -1).numpy(), atol=1e-12)


def test_all_blocks_kept_equals_dense(oracle_mod):
    N, bq, bk = 200, 64, 32
    q, k, v = _rand_qkv(1, 1, N, 8, 23, scale=2.0)
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx = np.tile(np.arange(nkb, dtype=np.int32), (1, 1, nqb, 1))
    kv_cnt = np.full((1, 1, nqb), nkb, np.int32)
    Os, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode="sparse")
    Od, _ = oracle_mod.attention_rows(q, k, v, bq, bk, mode="dense")
    np.testing.assert_allclose(Os, Od, rtol=0, atol=1e-12)
    # and the mask itself keeps all blocks when k = 1
    idx, cnt, _ = oracle_mod.mask(q, k, bq, bk, 1.0, 0.0)
    assert (cnt == nkb).all()
    idx, cnt, _ = oracle_mod.mask(q, k, bq, bk, 0.0, 1.0)
    assert (cnt >= 1).all()


def test_constant_v_and_zero_q_closed_forms(oracle_mod):
    N, bq, bk, d = 150, 64, 32, 8
    q, k, _ = _rand_qkv(1, 1, N, d, 24, scale=2.0)
    v = _bf16(torch.full((1, 1, N, d), 0.75))
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx, kv_cnt = synth.random_mask(1, 1, nqb, nkb, 2, seed=3)
    alpha = np.array([0.3], np.float32)
    for mode in ("sparse", "linear", "sla2", "dense"):
        O, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, alpha, mode=mode)
        rows_nonempty = []
        for i in range(N):
            c = int(kv_cnt[0, 0, i // bq])
            kept_keys = sum(min(bk, N - int(J) * bk) for J in kv_idx[0, 0, i // bq, :c])
            sparse_ok = kept_keys > 0
            linear_ok = kept_keys < N
            expect = 0.75
            if mode == "sparse" and not sparse_ok:
                expect = 0.0
            if mode == "linear" and not linear_ok:
                expect = 0.0
            if mode == "sla2":
                expect = 0.3 * (0.75 if sparse_ok else 0.0) + 0.7 * (0.75 if linear_ok else 0.0)
            np.testing.assert_allclose(O[i], expect, atol=1e-12)
    # Q = 0: uniform weights, the mean of V over the kept valid keys.
    q0 = _bf16(torch.zeros(1, 1, N, d))
    _, _, v = _rand_qkv(1, 1, N, d, 25)
    O, _ = oracle_mod.attention_rows(q0, k, v, bq, bk, kv_idx, kv_cnt, mode="sparse")
    vd = v.double().numpy()[0, 0]
    for i in range(N):
        c = int(kv_cnt[0, 0, i // bq])
        keys = [j for J in kv_idx[0, 0, i // bq, :c] for j in range(int(J) * bk, min(N, int(J) * bk + bk))]
        expect = vd[keys].mean(0) if keys else np.zeros(d)
        np.testing.assert_allclose(O[i], expect, atol=1e-12)


def test_empty_row_gives_zero_and_neg_inf_lse(oracle_mod):
    q, k, v = _rand_qkv(1, 1, 64, 8, 26)
    kv_idx = np.zeros((1, 1, 1, 1), np.int32)
    kv_cnt = np.zeros((1, 1, 1), np.int32)
    O, lse = oracle_mod.attention_rows(q, k, v, 64, 64, kv_idx, kv_cnt, mode="sparse")
    assert np.all(O == 0) and np.all(np.isneginf(lse))


def test_linear_branch_matches_associative_form(oracle_mod):
    # Empty mask: the complement is every key, and the normalised linear
    # attention equals phi(Q) (phi(K)^T V) / (phi(Q) . sum_j phi(k_j)).
    N, d = 130, 16
    q, k, v = _rand_qkv(1, 2, N, d, 27, scale=1.5)
    kv_idx = np.zeros((1, 2, 2, 3), np.int32)
    kv_cnt = np.zeros((1, 2, 2), np.int32)
    O, _ = oracle_mod.attention_rows(q, k, v, 128, 64, kv_idx, kv_cnt, mode="linear")
    pq, pk = _phi_torch(q.double()), _phi_torch(k.double())
    num = pq @ (pk.transpose(-1, -2) @ v.double())
    den = pq @ pk.sum(-2, keepdim=True).transpose(-1, -2)
    np.testing.assert_allclose(O.reshape(1, 2, N, d), (num / den).numpy(), rtol=1e-12, atol=1e-12)


def test_linear_branch_matches_masked_quadratic_form(oracle_mod):
    N, bq, bk, d = 200, 64, 32, 8
    q, k, v = _rand_qkv(1, 2, N, d, 28, scale=1.2)
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx, kv_cnt = synth.random_mask(1, 2, nqb, nkb, nkb - 1, seed=9)
    O, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode="linear")
    keep = torch.from_numpy(_block_bool_mask(kv_idx.numpy(), kv_cnt.numpy(), N, bq, bk))
    W = (_phi_torch(q.double()) @ _phi_torch(k.double()).transpose(-1, -2)) * (~keep)
    ref = (W @ v.double()) / W.sum(-1, keepdim=True)
    np.testing.assert_allclose(O.reshape(1, 2, N, d), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_phi_is_elu_plus_one(oracle_mod):
    # With one key outside the kept set, O_l = v of that key regardless of phi,
    # so use two keys and a scalar feature: weights phi(q) phi(k_j).
    xs = [-3.0, -0.5, 0.0, 0.25, 2.0]
    for x in xs:
        q = _bf16(torch.tensor([x]).reshape(1, 1, 1, 1).expand(1, 1, 2, 1).contiguous())
        k = _bf16(torch.tensor([x, 1.0]).reshape(1, 1, 2, 1))
        v = _bf16(torch.tensor([1.0, 0.0]).reshape(1, 1, 2, 1))
        kv_idx = np.zeros((1, 1, 1, 2), np.int32)
        kv_cnt = np.zeros((1, 1, 1), np.int32)
        O, _ = oracle_mod.attention_rows(q, k, v, 2, 1, kv_idx, kv_cnt, mode="linear")
        ph = float(F.elu(torch.tensor(float(q[0, 0, 0, 0]), dtype=torch.float64)) + 1)
        pk0 = float(F.elu(torch.tensor(float(k[0, 0, 0, 0]), dtype=torch.float64)) + 1)
        pk1 = float(F.elu(torch.tensor(1.0, dtype=torch.float64)) + 1)
        expect = ph * pk0 / (ph * pk0 + ph * pk1)
        np.testing.assert_allclose(O[0, 0], expect, atol=1e-14)


def test_sla2_mix_endpoints_and_linearity(oracle_mod):
    N, bq, bk, d = 192, 64, 32, 8
    q, k, v = _rand_qkv(1, 3, N, d, 29, scale=1.3)
    nqb, nkb = N // bq, N // bk
    kv_idx, kv_cnt = synth.random_mask(1, 3, nqb, nkb, 3, seed=4)
    Os, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode="sparse")
    Ol, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode="linear")
    a1, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, np.ones(3, np.float32), mode="sla2")
    a0, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, np.zeros(3, np.float32), mode="sla2")
    np.testing.assert_array_equal(a1, Os)
    np.testing.assert_array_equal(a0, Ol)
    al = np.array([0.6, 0.75, 1.0], np.float32)
    am, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, al, mode="sla2")
    w = np.repeat(al.astype(np.float64), N)[:, None]
    np.testing.assert_allclose(am, w * Os + (1 - w) * Ol, atol=1e-14)


def test_key_permutation_within_block_is_invisible(oracle_mod):
    N, bq, bk, d = 128, 64, 32, 8
    q, k, v = _rand_qkv(1, 1, N, d, 30, scale=1.5)
    kv_idx, kv_cnt = synth.random_mask(1, 1, 2, 4, 3, seed=6)
    perm = torch.cat([torch.randperm(bk, generator=torch.Generator().manual_seed(J)) + J * bk for J in range(4)])
    kp, vp = k[:, :, perm].contiguous(), v[:, :, perm].contiguous()
    for mode in ("sparse", "linear"):
        a, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode=mode)
        b, _ = oracle_mod.attention_rows(q, kp, vp, bq, bk, kv_idx, kv_cnt, mode=mode)
        np.testing.assert_allclose(a, b, atol=1e-12)


def test_sampled_rows_equal_full_rows(oracle_mod):
    q, k, v = _rand_qkv(1, 2, 160, 8, 31)
    kv_idx, kv_cnt = synth.random_mask(1, 2, 3, 5, 3, seed=8)
    full, lse = oracle_mod.attention_rows(q, k, v, 64, 32, kv_idx, kv_cnt, mode="sparse")
    rows = np.array([319, 0, 200, 17, 160], np.int64)
    part, lse_p = oracle_mod.attention_rows(q, k, v, 64, 32, kv_idx, kv_cnt, mode="sparse", rows=rows)
    np.testing.assert_array_equal(part, full[rows])
    np.testing.assert_array_equal(lse_p, lse[rows])


def test_invalid_arguments_are_rejected(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.select_row(np.array([0.5, 0.5]), 1.5, 0.5)
    q, k, v = _rand_qkv(1, 1, 64, 8, 32)
    kv_idx = np.full((1, 1, 1, 1), 5, np.int32)  # block index out of range
    kv_cnt = np.ones((1, 1, 1), np.int32)
    with pytest.raises(ValueError):
        oracle_mod.attention_rows(q, k, v, 64, 64, kv_idx, kv_cnt, mode="sparse")


# ----------------------------------------------------------------------------- low-bit sparse branch
def _e4m3_torch(x):
    """fp8 e4m3 rounding through torch's own cast (values already in fp32, |x| <= 448)."""
    t = torch.as_tensor(np.asarray(x), dtype=torch.float64).to(torch.float32).clamp(-448, 448)
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_rounding_matches_torch_float8(oracle_mod):
    x = np.concatenate([np.linspace(-448, 448, 40001), np.exp2(np.linspace(-12, 8.8, 5001)),
                        -np.exp2(np.linspace(-12, 8.8, 5001)), [0.0, 2.0 ** -10, 3 * 2.0 ** -11, 1.0625, 1.1875]])
    x = x.astype(np.float32).astype(np.float64)  # the GPU rounds fp32 values
    np.testing.assert_array_equal(oracle_mod.e4m3(x), _e4m3_torch(x))
    # saturation instead of overflow
    np.testing.assert_array_equal(oracle_mod.e4m3(np.array([500.0, -1e6, 449.0])), [448.0, -448.0, 448.0])


def test_q8_quantisation_closed_forms(oracle_mod):
    # A block whose max |x| is 127 * 2^-3 and whose values are multiples of 2^-3:
    # the scale is exactly 2^3 and every code is the integer x * 8.
    d, N = 8, 64
    vals = (torch.arange(N * d, dtype=torch.float32).reshape(N, d) % 255 - 127) / 8.0
    Q = _bf16(vals.reshape(1, 1, N, d))
    K = _bf16(-vals.reshape(1, 1, N, d))
    V = _bf16(torch.ones(1, 1, N, d))
    q8, sq, k8, sk, v8, sv = oracle_mod.quant_q8(Q, K, V, 64, 64)
    assert sq[0, 0, 0] == 8.0 and sk[0, 0, 0] == 8.0
    np.testing.assert_array_equal(q8[0, 0], (vals * 8).numpy().astype(np.int8))
    np.testing.assert_array_equal(k8[0, 0], (-vals * 8).numpy().astype(np.int8))
    # V all ones: the channel max maps to 448 exactly.
    np.testing.assert_array_equal(v8, 448.0)
    np.testing.assert_allclose(sv, 448.0)
    # Ties go to even: x * s = k + 1/2 with amax fixing s = 127 / 2.
    Qt = _bf16(torch.tensor([2.0, 5.0 / 127.0, 3.0 / 127.0, 1.0 / 127.0]).reshape(1, 1, 1, 4))
    q8t, sqt, *_ = oracle_mod.quant_q8(Qt, Qt, Qt, 64, 64)
    expect = np.rint(Qt.float().numpy() * np.float32(127.0 / 2.0))
    np.testing.assert_array_equal(q8t.reshape(-1), expect.reshape(-1).astype(np.int8))


def test_q8_constant_v_and_identical_keys(oracle_mod):
    B, H, N, d, bq, bk = 1, 2, 256, 16, 64, 64
    q, k, v = _rand_qkv(B, H, N, d, 40, scale=1.5)
    kv_idx, kv_cnt = (np.asarray(a) for a in synth.random_mask(B, H, N // bq, N // bk, 3, seed=12))
    # V constant per channel: the output is that constant times sum(p)/sum(e),
    # the e4m3-rounded weights over the unrounded normaliser, so within the
    # format's relative rounding of 2^-4 (and the same factor in every channel).
    c = torch.linspace(-2.0, 3.0, d)
    vc = _bf16(c.expand(B, H, N, d).clone())
    out = oracle_mod.attention_q8_rows(q, k, vc, bq, bk, kv_idx, kv_cnt)
    nonempty = np.repeat(kv_cnt.reshape(-1) > 0, bq)  # rows of empty blocks keep nothing: 0
    assert nonempty.any() and not nonempty.all()
    const = vc[0, 0, 0].float().numpy().astype(np.float64)
    ratio = out[nonempty] / const
    np.testing.assert_allclose(ratio, ratio[:, :1].repeat(d, axis=1), rtol=1e-6)  # fp32 channel scales
    assert np.all(np.abs(ratio - 1.0) <= 2.0 ** -4)
    np.testing.assert_array_equal(out[~nonempty], 0.0)
    # All keys identical: every kept key gets the same weight e4m3(e) over the
    # normaliser's e, so the output is the mean of the e4m3-coded values over
    # the kept keys times one factor within 2^-4 of 1, the same in every channel.
    kc = _bf16(k[:, :, :1].expand(B, H, N, d).clone())
    out = oracle_mod.attention_q8_rows(q, kc, v, bq, bk, kv_idx, kv_cnt)
    sv = np.float32(448.0) / np.abs(v.float().numpy()).max(axis=2)  # [B,H,d], fp32
    v8 = _e4m3_torch((v.float().numpy() * sv[:, :, None, :]).astype(np.float64)) / sv[:, :, None, :]
    for b in range(B):
        for h in range(H):
            for i in range(N):
                I = i // bq
                row = out[(b * H + h) * N + i]
                if kv_cnt[b, h, I] == 0:
                    np.testing.assert_array_equal(row, 0.0)
                    continue
                keys = np.concatenate([np.arange(J * bk, (J + 1) * bk) for J in kv_idx[b, h, I, :kv_cnt[b, h, I]]])
                mean = v8[b, h, keys].mean(axis=0)
                big = np.abs(mean) > 1e-3
                ratio = row[big] / mean[big]
                np.testing.assert_allclose(ratio, ratio[0], rtol=1e-9)
                assert abs(ratio[0] - 1.0) <= 2.0 ** -4


def test_q8_scaling_v_by_two_scales_output_exactly(oracle_mod):
    q, k, v = _rand_qkv(1, 1, 192, 16, 41, scale=2.0)
    kv_idx, kv_cnt = synth.random_mask(1, 1, 3, 3, 2, seed=13)
    a = oracle_mod.attention_q8_rows(q, k, v, 64, 64, kv_idx, kv_cnt)
    b = oracle_mod.attention_q8_rows(q, k, _bf16(v.float() * 2.0), 64, 64, kv_idx, kv_cnt)
    np.testing.assert_array_equal(b, 2.0 * a)


def test_q8_close_to_exact_sparse_attention(oracle_mod):
    # Within the error that 8-bit Q/K codes and e4m3 P/V allow: each e4m3
    # value carries up to 2^-4 relative error and each int8 code half a step
    # of the block's max / 127; on these inputs the outputs stay within a few
    # percent of the exact sparse branch (mean relative L1).
    q, k, v = _rand_qkv(1, 2, 512, 64, 42, scale=1.0)
    kv_idx, kv_cnt, _ = oracle_mod.mask(q, k, 64, 64, 0.25, 0.9)
    rows = np.arange(0, 1024, 7)
    a = oracle_mod.attention_q8_rows(q, k, v, 64, 64, kv_idx, kv_cnt, rows)
    e, _ = oracle_mod.attention_rows(q, k, v, 64, 64, kv_idx, kv_cnt, mode="sparse", rows=rows)
    rel = np.abs(a - e).sum() / np.abs(e).sum()
    assert rel < 0.06, rel
    assert rel > 1e-4  # the quantisation is really applied


def test_q8_dominant_late_block_keeps_the_codes_in_range(oracle_mod):
    # The row's largest scores sit in the LAST kept block, about 2^12 above
    # those of the first kept block. The integer reference must be the max
    # over every kept key: a reference taken from the first block alone would
    # put 2^(x - m) of the late keys far above e4m3's largest value (448),
    # saturate them and collapse the output. Against exact sparse attention
    # the result must stay within the 8-bit error budget.
    N, d, bq, bk = 256, 64, 64, 64
    g = torch.Generator().manual_seed(43)
    q = torch.randn(1, 1, N, d, generator=g)
    k = torch.randn(1, 1, N, d, generator=g) * 0.3
    v = torch.randn(1, 1, N, d, generator=g)
    # keys of block 3 point along their query block's mean direction
    u = q[0, 0, :bq].mean(0)
    u = u / u.norm()
    k[0, 0, 3 * bk:] = u * 16.0 + 0.05 * torch.randn(bk, d, generator=g)
    q[0, 0, :bq] = q[0, 0, :bq] + 8.0 * u
    q, k, v = _bf16(q), _bf16(k), _bf16(v)
    kv_idx = np.zeros((1, 1, 4, 4), np.int32)
    kv_idx[0, 0, 0, :2] = [0, 3]  # first block weak, last block dominant
    kv_cnt = np.array([[[2, 0, 0, 0]]], np.int32)
    rows = np.arange(bq)
    a = oracle_mod.attention_q8_rows(q, k, v, bq, bk, kv_idx, kv_cnt, rows)
    e, lse = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode="sparse", rows=rows)
    # the late block really dominates: its keys carry almost all the weight
    s = (q[0, 0, :bq].double() @ k[0, 0].double().T / math.sqrt(d)).numpy()
    late = np.exp(s[:, 3 * bk:] - lse[:, None]).sum(1)
    assert late.min() > 0.999
    assert (s[:, 3 * bk:].max(1) - s[:, :bk].max(1)).min() * math.log2(math.e) > 12
    rel = np.abs(a - e).sum() / np.abs(e).sum()
    assert rel < 0.06, rel


def test_q8_output_does_not_depend_on_the_kept_list_order(oracle_mod):
    # The definition has no walk order: a reversed kept list gives the same
    # output up to the order of the double sums.
    q, k, v = _rand_qkv(1, 1, 512, 32, 44, scale=2.0)
    kv_idx, kv_cnt = (np.asarray(x) for x in synth.random_mask(1, 1, 8, 8, 5, seed=14))
    rev = kv_idx.copy()
    for I in range(8):
        c = kv_cnt[0, 0, I]
        rev[0, 0, I, :c] = kv_idx[0, 0, I, :c][::-1]
    a = oracle_mod.attention_q8_rows(q, k, v, 64, 64, kv_idx, kv_cnt)
    b = oracle_mod.attention_q8_rows(q, k, v, 64, 64, rev, kv_cnt)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------- learnt router
def _router_inputs(seed, H=2, N=2048, d=64, s=1.5):
    Q, K, V = synth.make_qkv(1, H, N, d, grid=(2, 32, 32), s=s, seed=seed)
    return Q, K


def test_router_identity_projection_is_the_plain_mask(oracle_mod):
    Q, K = _router_inputs(50)
    I = np.tile(np.eye(64, dtype=np.float32), (2, 1, 1))
    a = oracle_mod.mask(Q, K, 64, 64, 0.1, 0.9)
    b = oracle_mod.mask_router(Q, K, 64, 64, I, I, 0.1, 0.9)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_router_probabilities_match_projected_softmax(oracle_mod):
    Q, K = _router_inputs(51)
    g = np.random.default_rng(5)
    Wq = g.standard_normal((2, 64, 32)).astype(np.float32) / 8
    Wk = g.standard_normal((2, 64, 32)).astype(np.float32) / 8
    _, _, P = oracle_mod.mask_router(Q, K, 64, 64, Wq, Wk, 0.1, 0.9)
    qb = oracle_mod.pool(Q, 64)[0]  # [H, Nqb, d]
    kb = oracle_mod.pool(K, 64)[0]
    for h in range(2):
        z = (qb[h] @ Wq[h].astype(np.float64)) @ (kb[h] @ Wk[h].astype(np.float64)).T / math.sqrt(32)
        ref = torch.softmax(torch.from_numpy(z), dim=-1).numpy()
        np.testing.assert_allclose(P[0, h], ref, rtol=1e-10, atol=1e-15)


def test_router_orthogonal_projection_keeps_the_probabilities(oracle_mod):
    Q, K = _router_inputs(52)
    R = np.linalg.qr(np.random.default_rng(6).standard_normal((64, 64)))[0].astype(np.float32)
    W = np.stack([R, R])
    _, _, P0 = oracle_mod.mask(Q, K, 64, 64, 0.1, 0.9)
    _, _, P1 = oracle_mod.mask_router(Q, K, 64, 64, W, W, 0.1, 0.9)
    np.testing.assert_allclose(P1, P0, rtol=1e-5, atol=1e-9)  # R R^T = I up to the fp32 rounding of R


def test_router_power_of_two_rescaling_is_exact(oracle_mod):
    Q, K = _router_inputs(53)
    g = np.random.default_rng(7)
    Wq = g.standard_normal((2, 64, 64)).astype(np.float32) / 8
    Wk = g.standard_normal((2, 64, 64)).astype(np.float32) / 8
    # Doubling Wq and halving Wk scales every product by exactly 2 and 1/2.
    a = oracle_mod.mask_router(Q, K, 64, 64, Wq, Wk, 0.1, 0.9)
    b = oracle_mod.mask_router(Q, K, 64, 64, Wq * 2, Wk / 2, 0.1, 0.9)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_router_generator_is_a_scaled_partial_isometry():
    # The stand-in router weights: seeded, fp32 [H, d, dr], and without their
    # perturbation a partial isometry times the stated gain.
    for d, dr in ((128, 64), (64, 128), (128, 128)):
        Wq, Wk = synth.make_router(3, d, dr, seed=2)
        assert Wq.shape == (3, d, dr) and Wq.dtype == torch.float32
        a, b = synth.make_router(3, d, dr, seed=2)
        assert torch.equal(a, Wq) and torch.equal(b, Wk)
        gain = (max(d, dr) / min(d, dr)) ** 0.25
        base = (Wq.double() + Wk.double()).numpy() / (2 * gain)  # perturbations average out partly
        for h in range(3):
            gram = base[h].T @ base[h] if dr <= d else base[h] @ base[h].T
            assert np.abs(gram - np.eye(min(d, dr))).max() < 0.1


# ----------------------------------------------------------------------------- gradients
def _bwd_case(N, bq, bk, d, seed, max_keep=None, keep_nonempty=True):
    q, k, v = _rand_qkv(1, 2, N, d, seed, scale=1.5)
    g = torch.Generator().manual_seed(seed + 1)
    dO = _bf16(torch.randn(1, 2, N, d, generator=g))
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx, kv_cnt = synth.random_mask(1, 2, nqb, nkb, nkb if max_keep is None else max_keep, seed=seed)
    if keep_nonempty:
        empty = kv_cnt == 0
        kv_cnt[empty] = 1
        kv_idx[..., 0][empty] = 0
    return q, k, v, dO, kv_idx, kv_cnt


def _autograd(fn, q, k, v, dO, extra=()):
    leaves = [t.double().requires_grad_(True) for t in (q, k, v)] + [t.requires_grad_(True) for t in extra]
    O = fn(*leaves)
    (O * dO.double()).sum().backward()
    return O.detach(), [t.grad for t in leaves]


def _kgrad(x, nkb, bk):
    """[1,H,N,d] key-side gradient as the oracle's [H*nkb, bk, d] block layout."""
    _, H, N, d = x.shape
    out = torch.zeros(H, nkb * bk, d, dtype=torch.float64)
    out[:, :N] = x[0]
    return out.reshape(H * nkb, bk, d).numpy()


@pytest.mark.parametrize("N,bq,bk", [(200, 64, 32), (130, 128, 64)])
def test_sparse_gradients_match_sdpa_autograd(oracle_mod, N, bq, bk):
    d = 16
    q, k, v, dO, kv_idx, kv_cnt = _bwd_case(N, bq, bk, d, 40 + N)
    m = torch.from_numpy(_block_bool_mask(kv_idx.numpy(), kv_cnt.numpy(), N, bq, bk))
    O, (gq, gk, gv) = _autograd(lambda a, b, c: F.scaled_dot_product_attention(a, b, c, attn_mask=m), q, k, v, dO)
    O_or, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode="sparse")
    np.testing.assert_allclose(O_or.reshape(O.shape), O.numpy(), rtol=0, atol=1e-12)
    dQ, dK, dV, _ = oracle_mod.attention_bwd(q, k, v, dO, bq, bk, kv_idx, kv_cnt, mode="sparse")
    nkb = -(-N // bk)
    np.testing.assert_allclose(dQ.reshape(gq.shape), gq.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dK, _kgrad(gk, nkb, bk), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dV, _kgrad(gv, nkb, bk), rtol=0, atol=1e-11)


def test_linear_gradients_match_autograd(oracle_mod):
    N, bq, bk, d = 200, 64, 32, 8
    q, k, v, dO, kv_idx, kv_cnt = _bwd_case(N, bq, bk, d, 44, max_keep=6, keep_nonempty=False)
    # one row keeps everything: its complement is empty, O_l = 0 and no gradient
    nkb = -(-N // bk)
    kv_idx[0, 1, 1, :nkb] = torch.arange(nkb, dtype=torch.int32)
    kv_cnt[0, 1, 1] = nkb
    keep = torch.from_numpy(_block_bool_mask(kv_idx.numpy(), kv_cnt.numpy(), N, bq, bk))

    def lin(a, b, c):
        W = (_phi_torch(a) @ _phi_torch(b).transpose(-1, -2)) * (~keep)
        den = W.sum(-1, keepdim=True)
        return torch.where(den > 0, (W @ c) / torch.where(den > 0, den, torch.ones_like(den)), torch.zeros_like(a))

    O, (gq, gk, gv) = _autograd(lin, q, k, v, dO)
    O_or, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode="linear")
    np.testing.assert_allclose(O_or.reshape(O.shape), O.numpy(), rtol=0, atol=1e-12)
    dQ, dK, dV, _ = oracle_mod.attention_bwd(q, k, v, dO, bq, bk, kv_idx, kv_cnt, mode="linear")
    np.testing.assert_allclose(dQ.reshape(gq.shape), gq.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dK, _kgrad(gk, nkb, bk), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dV, _kgrad(gv, nkb, bk), rtol=0, atol=1e-11)


def test_mix_gradients_match_autograd_including_alpha(oracle_mod):
    N, bq, bk, d = 200, 64, 32, 8
    q, k, v, dO, kv_idx, kv_cnt = _bwd_case(N, bq, bk, d, 45, max_keep=5)
    alpha = torch.tensor([0.7, 0.25], dtype=torch.float32)
    keep = torch.from_numpy(_block_bool_mask(kv_idx.numpy(), kv_cnt.numpy(), N, bq, bk))
    nkb = -(-N // bk)

    def mix(a, b, c, al):
        Os = F.scaled_dot_product_attention(a, b, c, attn_mask=keep)
        W = (_phi_torch(a) @ _phi_torch(b).transpose(-1, -2)) * (~keep)
        Ol = (W @ c) / W.sum(-1, keepdim=True)
        w = al.view(1, 2, 1, 1)
        return w * Os + (1 - w) * Ol

    O, (gq, gk, gv, ga) = _autograd(mix, q, k, v, dO, extra=(alpha.double(),))
    O_or, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, alpha=alpha, mode="sla2")
    np.testing.assert_allclose(O_or.reshape(O.shape), O.numpy(), rtol=0, atol=1e-12)
    dQ, dK, dV, da = oracle_mod.attention_bwd(q, k, v, dO, bq, bk, kv_idx, kv_cnt, alpha=alpha, mode="sla2",
                                              want_dalpha=True)
    np.testing.assert_allclose(dQ.reshape(gq.shape), gq.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dK, _kgrad(gk, nkb, bk), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dV, _kgrad(gv, nkb, bk), rtol=0, atol=1e-11)
    np.testing.assert_allclose(da, ga.numpy(), rtol=1e-12, atol=1e-11)


def test_sparse_gradient_invariants(oracle_mod):
    # Softmax rows sum to one, so each row's dS sums to zero: the key gradients of a
    # head sum to zero, and the value gradients sum to the sum of dO over the rows.
    N, bq, bk, d = 1000, 128, 64, 64
    q, k, v, dO, kv_idx, kv_cnt = _bwd_case(N, bq, bk, d, 46, max_keep=5)
    _, dK, dV, _ = oracle_mod.attention_bwd(q, k, v, dO, bq, bk, kv_idx, kv_cnt, mode="sparse", rows=[])
    nkb = -(-N // bk)
    dK = dK.reshape(2, nkb * bk, d)
    dV = dV.reshape(2, nkb * bk, d)
    scale = np.abs(dK).sum(1)
    assert np.all(np.abs(dK.sum(1)) <= 1e-12 * scale + 1e-300)
    np.testing.assert_allclose(dV.sum(1), dO.double().numpy()[0].sum(1), rtol=1e-12, atol=1e-10)


def test_dalpha_is_do_dot_branch_difference(oracle_mod):
    N, bq, bk, d = 300, 64, 64, 16
    q, k, v, dO, kv_idx, kv_cnt = _bwd_case(N, bq, bk, d, 47, max_keep=3)
    alpha = torch.tensor([0.9, 0.6], dtype=torch.float32)
    Os, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode="sparse")
    Ol, _ = oracle_mod.attention_rows(q, k, v, bq, bk, kv_idx, kv_cnt, mode="linear")
    ref = (dO.double().numpy().reshape(2, N, d) * (Os - Ol).reshape(2, N, d)).sum((1, 2))
    _, _, _, da = oracle_mod.attention_bwd(q, k, v, dO, bq, bk, kv_idx, kv_cnt, alpha=alpha, mode="sla2",
                                           rows=[], kblocks=[], want_dalpha=True)
    np.testing.assert_allclose(da, ref, rtol=1e-12)


def test_sampled_gradients_equal_full_gradients(oracle_mod):
    N, bq, bk, d = 500, 128, 64, 32
    q, k, v, dO, kv_idx, kv_cnt = _bwd_case(N, bq, bk, d, 48, max_keep=4)
    alpha = torch.tensor([0.8, 0.7], dtype=torch.float32)
    for mode in ("sparse", "sla2"):
        al = alpha if mode == "sla2" else None
        full = oracle_mod.attention_bwd(q, k, v, dO, bq, bk, kv_idx, kv_cnt, alpha=al, mode=mode)
        rows = np.array([0, 17, 499, 500 + 250, 999])
        kb = np.array([1, 7, 8 + 3])
        part = oracle_mod.attention_bwd(q, k, v, dO, bq, bk, kv_idx, kv_cnt, alpha=al, mode=mode, rows=rows,
                                        kblocks=kb)
        np.testing.assert_array_equal(part[0], full[0][rows])
        np.testing.assert_array_equal(part[1], full[1][kb])
        np.testing.assert_array_equal(part[2], full[2][kb])
