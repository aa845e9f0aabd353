"""GPU sparse + linear mix (sla2_attn_fwd) vs the double-precision oracle on
the same (oracle-computed or seeded) block mask."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_pooled_b200 import synth
from parity import assert_outputs, sample_rows

pytestmark = pytest.mark.gpu


def _gpu_sla2(Q, K, V, idx, cnt, alpha, bq, bk):
    from block_sparse_attention_pooled_b200 import sparge

    dev = torch.device("cuda")
    O = sparge.sla2_attn_fwd(Q.to(dev), K.to(dev), V.to(dev), torch.as_tensor(idx, dtype=torch.int32).to(dev),
                             torch.as_tensor(cnt, dtype=torch.int32).to(dev),
                             torch.as_tensor(alpha, dtype=torch.float32).to(dev), bq, bk)
    torch.cuda.synchronize()
    assert sparge.device_status() == 0
    return O.float().cpu().numpy()


def _check(Q, K, V, idx, cnt, alpha, bq, bk, rows=None):
    B, H, N, d = Q.shape
    O = _gpu_sla2(Q, K, V, idx, cnt, alpha, bq, bk)
    ref, _ = oracle.attention_rows(Q, K, V, bq, bk, idx, cnt, np.asarray(alpha, np.float32), mode="sla2", rows=rows)
    got = O.reshape(-1, d) if rows is None else O.reshape(-1, d)[rows]
    return assert_outputs(got, ref, "sla2")


@pytest.mark.parametrize("N,bq,bk,max_keep", [(1000, 128, 64, 6), (777, 64, 64, 5), (2000, 128, 128, 4),
                                              (777, 64, 128, 4), (1000, 128, 128, 5),
                                               (130, 128, 64, 3), (64, 64, 64, 1), (4100, 128, 64, 20)])
def test_sla2_random_masks(N, bq, bk, max_keep):
    Q, K, V = synth.make_qkv(1, 3, N, 128, grid=None, s=1.5, seed=N + bq)
    nqb, nkb = -(-N // bq), -(-N // bk)
    idx, cnt = synth.random_mask(1, 3, nqb, nkb, min(nkb, max_keep), seed=N)
    alpha = np.array([0.6, 0.85, 1.0], np.float32)
    _check(Q, K, V, idx.numpy(), cnt.numpy(), alpha, bq, bk)


def test_sla2_alpha_endpoints():
    from block_sparse_attention_pooled_b200 import sparge

    N, bq, bk = 1500, 128, 64
    Q, K, V = synth.make_qkv(1, 2, N, 128, grid=None, s=1.5, seed=3)
    idx, cnt = synth.random_mask(1, 2, -(-N // bq), -(-N // bk), 7, seed=5)
    cnt = torch.clamp(cnt, min=1)
    for h in range(2):
        for I in range(cnt.shape[-1]):
            c = int(cnt[0, h, I])
            if len(set(idx[0, h, I, :c].tolist())) != c:
                idx[0, h, I, :c] = torch.arange(c)
    # alpha = 1: exactly the pure sparse kernel's output
    O1 = _gpu_sla2(Q, K, V, idx, cnt, np.ones(2, np.float32), bq, bk)
    dev = torch.device("cuda")
    Os = sparge.sparge_attn_fwd(Q.to(dev), K.to(dev), V.to(dev), idx.to(dev), cnt.to(dev), bq, bk)
    assert np.array_equal(O1, Os.float().cpu().numpy())
    # alpha = 0: pure linear branch over the complement
    O0 = _gpu_sla2(Q, K, V, idx, cnt, np.zeros(2, np.float32), bq, bk)
    ref, _ = oracle.attention_rows(Q, K, V, bq, bk, idx, cnt, mode="linear")
    assert_outputs(O0.reshape(-1, 128), ref, "linear branch")


def test_sla2_empty_and_full_rows():
    N, bq, bk = 512, 128, 64
    Q, K, V = synth.make_qkv(1, 1, N, 128, grid=None, s=1.0, seed=11)
    idx = np.zeros((1, 1, 4, 8), np.int32)
    cnt = np.array([[[0, 3, 8, 1]]], np.int32)
    idx[0, 0, 1, :3] = [0, 4, 7]
    idx[0, 0, 2, :] = np.arange(8)  # every block kept: linear part is 0
    idx[0, 0, 3, 0] = 7             # the ragged-free last block only
    _check(Q, K, V, idx, cnt, np.array([0.7], np.float32), bq, bk)


def _neighbour_masks(H, nqb, nkb, seed):
    """Kept lists for query blocks 2c and 2c + 1 with every relation two
    ascending lists can have: identical, nested either way, interleaved with a
    shared part, disjoint, one or both empty, one complete."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 7])))
    idx = np.zeros((1, H, nqb, nkb), np.int32)
    cnt = np.zeros((1, H, nqb), np.int32)

    def pick(pool, k):
        return np.sort(rng.choice(pool, size=min(k, len(pool)), replace=False))

    kinds = 9
    for h in range(H):
        for c in range((nqb + 1) // 2):
            kind = (c + h) % kinds
            base = pick(np.arange(nkb), int(rng.integers(1, nkb + 1)))
            if kind == 0:
                a, b = base, base
            elif kind == 1:
                a, b = pick(base, max(1, len(base) // 2)), base
            elif kind == 2:
                a, b = base, pick(base, max(1, len(base) // 2))
            elif kind == 3:
                rest = np.setdiff1d(np.arange(nkb), base)
                a = np.union1d(pick(base, len(base) // 2 + 1), pick(rest, 3))
                b = np.union1d(pick(base, len(base) // 2 + 1), pick(rest, 3))
            elif kind == 4:
                perm = rng.permutation(nkb)
                a, b = np.sort(perm[: nkb // 3]), np.sort(perm[nkb // 3: nkb // 3 + nkb // 4])
            elif kind == 5:
                a, b = np.array([], np.int64), base
            elif kind == 6:
                a, b = base, np.array([], np.int64)
            elif kind == 7:
                a, b = np.arange(nkb), base
            else:
                a, b = np.array([], np.int64), np.array([], np.int64)
            for I, lst in ((2 * c, a), (2 * c + 1, b)):
                if I < nqb:
                    idx[0, h, I, :len(lst)] = lst
                    cnt[0, h, I] = len(lst)
    return idx, cnt


@pytest.mark.parametrize("N,bq,bk", [(1100, 128, 64), (1300, 64, 64), (2200, 128, 128), (900, 64, 128)])
def test_sla2_neighbouring_blocks_share_key_blocks(N, bq, bk):
    # One CTA takes query blocks 2c and 2c + 1 and walks the union of their
    # lists; every relation between the two lists, odd block counts and a
    # ragged last key block.
    H = 9
    Q, K, V = synth.make_qkv(1, H, N, 128, grid=None, s=1.5, seed=N + bk)
    nqb, nkb = -(-N // bq), -(-N // bk)
    idx, cnt = _neighbour_masks(H, nqb, nkb, seed=N)
    alpha = np.linspace(0.55, 0.95, H).astype(np.float32)
    _check(Q, K, V, idx, cnt, alpha, bq, bk)


@pytest.mark.parametrize("B,H,N,bq,bk", [(2, 350, 100, 64, 64), (1, 900, 64, 64, 64), (3, 200, 200, 128, 128)])
def test_sla2_many_short_heads(B, H, N, bq, bk):
    # The summary kernel splits all heads' 64-key tiles evenly over its
    # persistent grid: with short heads one CTA's run crosses three or more
    # heads, so its two TMEM accumulators are each reused after release.
    Q, K, V = synth.make_qkv(B, H, N, 128, grid=None, s=1.5, seed=N + H)
    nqb, nkb = -(-N // bq), -(-N // bk)
    idx, cnt = synth.random_mask(B, H, nqb, nkb, nkb, seed=H)
    alpha = np.linspace(0.6, 1.0, H).astype(np.float32)
    _check(Q, K, V, idx.numpy(), cnt.numpy(), alpha, bq, bk)


def test_sla2_long_rows_at_the_block_limit():
    # 4096 key blocks per row (the library's maximum), ragged last block: the
    # first query block keeps every block (empty complement, O_l = 0), the
    # last keeps a scattered half, the rest a few (complements of ~262k keys).
    N, bq, bk = 64 * 4096 - 17, 128, 64
    Q, K, V = synth.make_qkv(1, 1, N, 128, grid=None, s=1.5, seed=4098)
    nqb, nkb = -(-N // bq), -(-N // bk)
    idx, cnt = (np.asarray(a) for a in synth.random_mask(1, 1, nqb, nkb, 5, seed=13))
    idx[0, 0, 0] = np.arange(nkb, dtype=np.int32)
    cnt[0, 0, 0] = nkb
    half = np.sort(np.random.default_rng(6).choice(nkb, nkb // 2, replace=False)).astype(np.int32)
    idx[0, 0, nqb - 1, : nkb // 2] = half
    cnt[0, 0, nqb - 1] = nkb // 2
    rows = np.concatenate([np.arange(0, 128, 17), np.arange((nqb - 1) * bq, N, 19),
                           np.arange(900 * bq, 900 * bq + 128, 23)]).astype(np.int64)
    _check(Q, K, V, idx, cnt, np.array([0.75], np.float32), bq, bk, rows=rows)


@pytest.mark.parametrize("name", ["sla2_480p", "720p"])
def test_sla2_workload_oracle_mask(name):
    w = synth.WORKLOADS[name]
    if name == "720p":
        heads = [(0, 0), (0, 17), (0, 39)]
        Q, K, V, _ = synth.make_workload(w, heads=heads)
        alpha = synth.make_alpha(w.H, w.seed, True).numpy()[[h for _, h in heads]]
    else:
        Q, K, V, alpha = synth.make_workload(w)
        alpha = alpha.numpy()
    idx, cnt, _ = oracle.mask(Q, K, w.bq, w.bk, w.topk, w.topp)
    B, H = Q.shape[:2]
    rows = sample_rows(B, H, w.N, w.bq, 48, seed=2)
    max_abs, mean_rel = _check(Q, K, V, idx, cnt, alpha, w.bq, w.bk, rows=rows)
    print(f"{name}: max-abs {max_abs:.2e} mean-rel-L1 {mean_rel:.2e}")


def test_sla2_is_deterministic():
    N = 3000
    Q, K, V = synth.make_qkv(1, 2, N, 128, grid=None, s=2.0, seed=12)
    idx, cnt = synth.random_mask(1, 2, -(-N // 128), -(-N // 64), 10, seed=7)
    a = _gpu_sla2(Q, K, V, idx, cnt, np.array([0.7, 0.9], np.float32), 128, 64)
    b = _gpu_sla2(Q, K, V, idx, cnt, np.array([0.7, 0.9], np.float32), 128, 64)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("kind", ["random", "windows"])
def test_sla2_many_query_tiles(kind):
    # Many query tiles over many heads, with masks whose neighbouring rows
    # change a lot (random) or by a few blocks at a time (sliding windows).
    B, H, N, d, bq, bk = 1, 96, 8192, 128, 128, 64
    g = torch.Generator().manual_seed(31)
    Q, K, V = ((torch.randn(B, H, N, d, generator=g) * s).to(torch.bfloat16) for s in (1.5, 1.5, 1.0))
    nqb, nkb = N // bq, N // bk
    if kind == "random":
        idx, cnt = (np.asarray(a) for a in synth.random_mask(B, H, nqb, nkb, 8, seed=5))
    else:
        idx = np.zeros((B, H, nqb, nkb), np.int32)
        cnt = np.zeros((B, H, nqb), np.int32)
        for h in range(H):
            for I in range(nqb):
                w = sorted({(2 * I + k + h) % nkb for k in range(6)})
                idx[0, h, I, :len(w)] = w
                cnt[0, h, I] = len(w)
    alpha = np.linspace(0.6, 0.95, H).astype(np.float32)
    rows = sample_rows(B, H, N, bq, 64, seed=3)
    max_abs, mean_rel = _check(Q, K, V, idx, cnt, alpha, bq, bk, rows=rows)
    print(f"{kind}: max-abs {max_abs:.2e} mean-rel-L1 {mean_rel:.2e}")
