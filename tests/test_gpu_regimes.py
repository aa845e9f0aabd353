"""The mask-regime report (Top-k alone, Top-p alone and their union against
dense attention, SpargeAttention2 article section 1) on a reduced sweep
workload: its dense reference agrees with the oracle's dense attention, the
union keeps at least what each rule keeps, and a mask that keeps everything
reproduces the dense output exactly."""
import numpy as np
import pytest
import torch

import bench
from block_sparse_attention_pooled_b200 import synth
from parity import MAX_ABS, MEAN_REL_L1

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["sweep_flat", "sweep_peaked"])
def test_regime_rows_on_two_heads(name):
    w = synth.WORKLOADS[name]
    Q, K, V = synth.make_qkv(1, 2, w.N, w.d, w.grid, w.s, w.seed)
    settings = [("top-k", 0.05, 0.0), ("top-p", 0.0, 0.9), ("hybrid", 0.05, 0.9), ("all", 1.0, 0.0)]
    rows, check = bench.regime_rows(w, Q, K, V, settings, torch.device("cuda"), check_rows=32)
    assert check["max_abs"] <= MAX_ABS and check["mean_rel_l1"] <= MEAN_REL_L1, check
    r = {x["rule"]: x for x in rows}
    # The union of two prefixes of one order is the longer prefix, row by row.
    assert r["hybrid"]["kept_fraction"] >= max(r["top-k"]["kept_fraction"], r["top-p"]["kept_fraction"]) - 1e-12
    assert r["hybrid"]["mean_kept_blocks"] >= max(r["top-k"]["mean_kept_blocks"], r["top-p"]["mean_kept_blocks"])
    assert r["all"]["kept_fraction"] == 1.0
    assert r["all"]["rel_l1_vs_dense"] == 0.0 and r["all"]["max_abs_vs_dense"] == 0.0
    assert abs(r["all"]["cos_sim_vs_dense"] - 1.0) < 1e-12
    for x in rows:
        # flat attention averages V over many keys, so a sparse output can sit
        # several times the dense output's (small) norm away from it
        assert np.isfinite(x["rel_l1_vs_dense"]) and x["rel_l1_vs_dense"] >= 0.0
        assert -1.0 <= x["cos_sim_vs_dense"] <= 1.0
    print(name, [(x["rule"], round(x["kept_fraction"], 4), round(x["rel_l1_vs_dense"], 4)) for x in rows])
