"""Failure detection on the GPU without a fault: the fused IKBO launch's bounded completion-flag
wait is made to run out, and the test checks that the kernel reports it and returns.

The fused launch ("ROCS：面向请求的大规模推荐计算共享" review, §2.4: the request and candidate
GEMMs in one persistent kernel) lets a candidate tile's epilogue wait for the completion flags of
the request tiles whose Z rows it gathers.  A test hook (rocs_test_withhold_ikbo_flag, off by
default) keeps one request tile from publishing its flag and shortens the wait budget to about
2 ms.  Nothing faults, traps or spins without a limit: every wait in the kernel is bounded and the
abort path drains the CTA's copies and MMAs before it releases tensor memory.
"""
import time

import numpy as np
import pytest
import torch

import synth
from oracle import rocs_oracle as O
from tests.gpu_util import check_bf16, dev, dev_i32, host, stream

pytestmark = pytest.mark.gpu

BUDGET_CYCLES = 4_000_000      # about 2 ms at the B200's 1.97 GHz SM clock


@pytest.fixture(scope="module")
def R():
    from request_candidate_sharing_b200 import rocs
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    h = rocs.Rocs(0)
    yield h
    h.rocs_test_withhold_ikbo_flag(-1)
    h.close()


def test_fused_ikbo_flag_wait_runs_out(R):
    from request_candidate_sharing_b200 import rocs
    # 130 requests = two 128-request blocks of the Z GEMM; d_C_out = 64 is one column tile, so flag
    # b is request block b.  Requests 0..127 own candidate rows 0..383 (three full candidate tiles);
    # requests 128 and 129 own rows 384..493, the fourth tile, which gathers from block 1 only.
    counts = np.asarray([3] * 128 + [50, 60], np.int32)
    case = synth.LinearCase("flag_timeout", counts, 64, 64, 32, 64, "relu", True, 5)
    x = synth.linear_inputs(case)
    _, m = O.segments(case.counts)
    desc = rocs.IkboDesc(case.B_R, case.B_C, 64, 64, 32, 64, rocs.ROCS_BF16, rocs.ROCS_BF16, rocs.ACT["relu"])
    nb = R.rocs_linear_ikbo_workspace(desc)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    t = {k: dev(x[k]) for k in ("X_R", "X_C", "W_RR", "W_CR", "W_CC")}
    bR, bC, md = dev(x["b_R"], torch.float32), dev(x["b_C"], torch.float32), dev_i32(m)

    def call():
        YR = torch.full((case.B_R, 32), float("nan"), dtype=torch.bfloat16, device="cuda")
        YC = torch.full((case.B_C, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        R.rocs_linear_ikbo(desc, t["X_R"], t["X_C"], md, t["W_RR"], t["W_CR"], t["W_CC"], bR, bC, YR, YC, ws, nb,
                           stream())
        torch.cuda.synchronize()
        return YR, YC, time.perf_counter() - t0, R.rocs_get_device_status(stream())

    R.rocs_set_ikbo_fused(1)
    YR0, YC0, _, st0 = call()
    assert st0 == rocs.ROCS_OK

    try:
        R.rocs_test_withhold_ikbo_flag(1, BUDGET_CYCLES)
        YR1, YC1, dt, st1 = call()
    finally:
        R.rocs_test_withhold_ikbo_flag(-1)
    assert st1 == rocs.ROCS_ERR_DEVICE_TIMEOUT
    assert dt < 0.5, f"the timed-out launch took {dt:.3f} s: the shortened budget was not applied"
    # the candidates that gather from the withheld block are untouched; every row that was
    # written holds the right value
    assert torch.isnan(YC1[384:]).all()
    written = ~torch.isnan(YC1).any(dim=1)
    assert written[:384].any()
    assert torch.equal(YC1[written], YC0[written])
    assert torch.equal(YR1, YR0)
    assert R.rocs_get_device_status(stream()) == rocs.ROCS_OK      # the status word was cleared

    # the kernel returned and left the context usable: the next call runs normally
    YR2, YC2, _, st2 = call()
    assert st2 == rocs.ROCS_OK
    assert torch.equal(YR2, YR0) and torch.equal(YC2, YC0)
    rR, rC = O.glm_linear(x["X_R"], x["X_C"], m, x["W_RR"], x["W_CR"], x["W_CC"], x["b_R"], x["b_C"], "relu")
    check_bf16(host(YR2), rR, out_bf16=True, what="Y_R")
    check_bf16(host(YC2), rC, out_bf16=True, what="Y_C")


def test_withhold_hook_argument_checks(R):
    from request_candidate_sharing_b200 import rocs
    for bad in ((-2, 0), (0, 10), (0, 10 ** 11)):
        with pytest.raises(rocs.RocsError) as e:
            R.rocs_test_withhold_ikbo_flag(*bad)
        assert e.value.status == rocs.ROCS_ERR_INVALID_ARG
    R.rocs_test_withhold_ikbo_flag(-1, 0)
