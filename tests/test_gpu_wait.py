"""Bounded device waits: a kernel that waits on a barrier nothing arrives on
gives up after its limit, frees its tensor memory and returns; the host then
reads the self-test's site code through sparge_device_status and the context
keeps working (a mask computed right after matches the oracle)."""
import time

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_pooled_b200 import synth
from parity import compare_masks

pytestmark = pytest.mark.gpu


def test_wait_gives_up_reports_its_site_and_leaves_the_context_usable():
    from block_sparse_attention_pooled_b200 import sparge

    assert sparge.device_status() == 0
    flag = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    sparge.selftest_wait(5000, gave_up=flag)  # 5 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert flag.item() == 1  # every role gave up its wait
    assert 0.004 < elapsed < 5.0, elapsed  # it waited about its limit, then returned
    assert sparge.device_status() == sparge.SITE_SELFTEST
    assert sparge.device_status() == 0  # reading the word clears it
    # The same process keeps launching the library's kernels (tensor memory
    # was freed: the attention kernels allocate it again).
    Q, K, V = synth.make_qkv(1, 2, 1000, 128, grid=(1, 20, 50), s=2.0, seed=1)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    idx, cnt = sparge.sparge_mask(Qd, Kd, 128, 64, 0.1, 0.9)
    O = sparge.sparge_attn_fwd(Qd, Kd, Vd, idx, cnt, 128, 64)
    torch.cuda.synchronize()
    assert sparge.device_status() == 0
    o_idx, o_cnt, o_P = oracle.mask(Q, K, 128, 64, 0.1, 0.9)
    compare_masks(idx.cpu().numpy(), cnt.cpu().numpy(), o_idx, o_cnt, o_P, 0.1, 0.9)
    assert torch.isfinite(O.float()).all()


def test_two_waits_in_a_row_report_the_first_site_once():
    from block_sparse_attention_pooled_b200 import sparge

    sparge.selftest_wait(2000)
    sparge.selftest_wait(2000)
    assert sparge.device_status() == sparge.SITE_SELFTEST
    assert sparge.device_status() == 0
