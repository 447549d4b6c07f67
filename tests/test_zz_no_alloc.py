"""The no-allocation IKBO linear (rocs_linear_ikbo_noalloc), for callers that cannot allocate
device memory -- not even a workspace -- because their host plans every device buffer up front.

Its scratch is a built-in device array shared by all calls, so the test makes two calls in a row
with different inputs (a stale or uncleared scratch would show in the second) and compares each
with rocs_linear_ikbo on the same inputs.  Collected last, so a run that stops at the first
failure has run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import rocs_oracle as O
from tests.gpu_util import check_bf16, check_fp32, dev, dev_i32, host, stream

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    from request_candidate_sharing_b200 import rocs
    h = rocs.Rocs(0)
    yield h
    h.close()


def _both(R, case, x, m, dtype_in, dtype_out):
    from request_candidate_sharing_b200 import rocs
    tdt = torch.bfloat16 if dtype_in == rocs.ROCS_BF16 else torch.float32
    odt = torch.bfloat16 if dtype_out == rocs.ROCS_BF16 else torch.float32
    d = rocs.IkboDesc(case.B_R, case.B_C, case.d_R_in, case.d_C_in, case.d_R_out, case.d_C_out, dtype_in,
                      dtype_out, rocs.ACT[case.act])
    t = {k: dev(v, tdt) for k, v in x.items() if k.startswith(("X", "W"))}
    bR, bC = dev(x["b_R"], torch.float32), dev(x["b_C"], torch.float32)
    mi = dev_i32(m)
    outs = []
    for variant in ("workspace", "noalloc"):
        YR = torch.full((case.B_R, case.d_R_out), float("nan"), dtype=odt, device="cuda")
        YC = torch.full((case.B_C, case.d_C_out), float("nan"), dtype=odt, device="cuda")
        if variant == "workspace":
            nb = R.rocs_linear_ikbo_workspace(d)
            ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
            R.rocs_linear_ikbo(d, t["X_R"], t["X_C"], mi, t["W_RR"], t["W_CR"], t["W_CC"], bR, bC, YR, YC, ws, nb,
                               stream())
        else:
            R.rocs_linear_ikbo_noalloc(d, t["X_R"], t["X_C"], mi, t["W_RR"], t["W_CR"], t["W_CC"], bR, bC, YR, YC,
                                       stream())
        assert R.rocs_get_device_status(stream()) == 0
        outs.append((host(YR), host(YC)))
    return outs


@pytest.mark.parametrize("dtype_in", [0, 1])
def test_noalloc_matches_workspace_entry_point_two_calls(R, dtype_in):
    from request_candidate_sharing_b200 import rocs
    for call, (counts, d, seed) in enumerate([([40, 0, 300, 7], 512, 11), ([129, 3], 256, 12)]):
        case = synth.LinearCase(f"noalloc{call}", np.asarray(counts, np.int32), d, d, d, d, "relu",
                                dtype_in == 1, seed)
        x = synth.linear_inputs(case)
        _, m = O.segments(case.counts)
        dtype_out = rocs.ROCS_F32
        (wR, wC), (nR, nC) = _both(R, case, x, m, dtype_in, dtype_out)
        # same kernels in the same order: identical results
        assert np.array_equal(wR, nR) and np.array_equal(wC, nC)
        rR, rC = O.glm_linear(x["X_R"], x["X_C"], m, x["W_RR"], x["W_CR"], x["W_CC"], x["b_R"], x["b_C"], "relu")
        if dtype_in == 0:
            check_fp32(nR, rR, what="Y_R")
            check_fp32(nC, rC, what="Y_C")
        else:
            check_bf16(nR, rR, what="Y_R")
            check_bf16(nC, rC, what="Y_C")


def test_noalloc_rejects_sizes_beyond_its_scratch(R):
    from request_candidate_sharing_b200 import rocs
    d = rocs.IkboDesc(512, 0, 64, 64, 0, 4096, rocs.ROCS_BF16, rocs.ROCS_F32, 0)   # 2,097,152 > 1,048,576
    with pytest.raises(rocs.RocsError) as e:
        R.rocs_linear_ikbo_noalloc(d, 16, None, None, None, 16, None, None, 16, None, None, stream())
    assert e.value.status == rocs.ROCS_ERR_UNSUPPORTED and "scratch" in str(e.value)
    d = rocs.IkboDesc(4, 8, 100, 64, 0, 64, rocs.ROCS_BF16, rocs.ROCS_F32, 0)      # needs the alignment fix
    with pytest.raises(rocs.RocsError) as e:
        R.rocs_linear_ikbo_noalloc(d, 16, 16, 16, None, 16, 16, None, 16, None, 16, stream())
    assert e.value.status == rocs.ROCS_ERR_UNSUPPORTED
