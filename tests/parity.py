"""Comparison helpers shared by the GPU parity tests.

The bars: masks bit-exact except blocks whose probability lies within 1e-6
(relative) of the row's selection threshold, or rows whose Top-p running sum
lies within 1e-6 of p at the boundary; outputs within max-abs 2e-2 and mean
relative L1 5e-3 of the double-precision oracle on the same mask.
"""
import numpy as np

import oracle

MAX_ABS = 2e-2
MEAN_REL_L1 = 5e-3
AMBIG_REL = 1e-6


def compare_masks(g_idx, g_cnt, o_idx, o_cnt, P, topk, topp):
    """Returns (n_rows, n_mismatched_rows, n_ambiguous_rows); raises on a
    mismatch outside the ambiguity rule. Arrays are numpy; P is the oracle's
    double-precision probability array."""
    g_idx = np.asarray(g_idx).reshape(-1, g_idx.shape[-1])
    o_idx = np.asarray(o_idx).reshape(-1, o_idx.shape[-1])
    g_cnt = np.asarray(g_cnt).reshape(-1)
    o_cnt = np.asarray(o_cnt).reshape(-1)
    P = np.asarray(P).reshape(-1, P.shape[-1])
    nkb = P.shape[1]
    cols = np.arange(nkb)[None, :]
    valid_g = cols < g_cnt[:, None]
    valid_o = cols < o_cnt[:, None]
    same = (g_cnt == o_cnt) & np.all(np.where(valid_o, g_idx == o_idx, True), axis=1)
    bad_rows = np.nonzero(~same)[0]
    n_amb = 0
    for r in bad_rows:
        gs = set(g_idx[r, : g_cnt[r]].tolist())
        os_ = set(o_idx[r, : o_cnt[r]].tolist())
        sel = oracle.select_row(P[r], topk, topp)
        m = sel["m"]
        order = sel["order"]
        t = P[r, order[m - 1]]
        allowed = set(np.nonzero(np.abs(P[r] - t) <= AMBIG_REL * t)[0].tolist())
        cum = sel["cum"]
        if topp > 0:
            # Every Top-p count whose boundary lies within the tolerance of p
            # is a correct answer for some rounding of the running sums.
            ok_pc = [c for c in range(1, nkb + 1)
                     if cum[c] >= topp - AMBIG_REL and cum[c - 1] < topp + AMBIG_REL]
            if cum[nkb] < topp + AMBIG_REL:
                ok_pc.append(nkb)
            ms = [max(sel["kc"], c, 1) for c in ok_pc] + [m]
            allowed |= set(int(j) for j in order[min(ms):max(ms)])
        diff = gs ^ os_
        if not diff <= allowed:
            raise AssertionError(
                f"mask row {r}: GPU keeps {sorted(gs)[:20]}... ({len(gs)}), oracle {sorted(os_)[:20]}... "
                f"({len(os_)}); unexplained blocks {sorted(diff - allowed)[:10]}, threshold {t}")
        n_amb += 1
    return len(g_cnt), len(bad_rows), n_amb


def check_mask_outputs(gpu, ora, topk, topp):
    """Checks a GPU mask (kv_idx, kv_cnt, probs as float, row thresholds as
    float) against the oracle's (kv_idx, kv_cnt, P in double): kept sets under
    the ambiguity rule, probabilities to float rounding, and, on the rows whose
    kept sets agree, the threshold = the smallest kept probability (the last
    kept block in the (P desc, index asc) order). Returns compare_masks'
    counts."""
    g_idx, g_cnt, g_P, g_thr = gpu
    o_idx, o_cnt, o_P = ora
    # float rounding (2^-24 relative) of a double that differs from the
    # oracle's by a few double rounding units
    np.testing.assert_allclose(g_P, o_P, rtol=1.2e-7, atol=1e-45)
    n, bad, amb = compare_masks(g_idx, g_cnt, o_idx, o_cnt, o_P, topk, topp)
    nkb = o_P.shape[-1]
    oi = o_idx.reshape(-1, nkb)
    oc = o_cnt.reshape(-1)
    gi = g_idx.reshape(-1, nkb)
    gc = g_cnt.reshape(-1)
    P = o_P.reshape(-1, nkb)
    cols = np.arange(nkb)[None, :]
    valid = cols < oc[:, None]
    same = (gc == oc) & np.all(np.where(valid, gi == oi, True), axis=1)
    kept_P = np.where(valid, np.take_along_axis(P, np.clip(oi, 0, nkb - 1), axis=1), np.inf)
    t = kept_P.min(axis=1)
    np.testing.assert_allclose(g_thr.reshape(-1)[same], t[same], rtol=1.2e-7, atol=1e-45)
    return n, bad, amb


def output_errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.abs(ref).sum())
    mean_rel = float(err.sum() / denom) if denom > 0 else float(err.sum())
    return max_abs, mean_rel


def assert_outputs(got, ref, what=""):
    max_abs, mean_rel = output_errors(got, ref)
    assert max_abs <= MAX_ABS and mean_rel <= MEAN_REL_L1, f"{what}: max-abs {max_abs:.3e}, mean-rel-L1 {mean_rel:.3e}"
    return max_abs, mean_rel


def sample_rows(B, H, N, bq, n, seed):
    """Flat row ids: n random rows plus the first and last rows of the first
    and last query blocks of a few heads (the ragged tail included)."""
    rng = np.random.default_rng(seed)
    rows = set(rng.integers(0, B * H * N, size=n).tolist())
    for bh in {0, B * H - 1, (B * H) // 2}:
        for i in (0, bq - 1, N - 1, max(0, N - 2), (N - 1) // bq * bq):
            rows.add(bh * N + i)
    return np.array(sorted(rows), np.int64)
