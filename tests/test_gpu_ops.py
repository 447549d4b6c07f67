"""GPU parity of each librocs entry point against the float64 oracle, through the C ABI.

Sizes span several tiles and ragged tails; edge cases: empty requests, one-candidate requests,
rows not multiple of 16 bytes (alignment fix), partial N tiles.  Bounds: bit-exact for the
segment bookkeeping and for small-integer inputs (every summation order exact); fp32 path max
relative error 1e-4; bf16 path relative L2 5e-3 and max abs 2e-2 (+ half an output ulp when
the output itself is bf16).
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import rocs_oracle as O
from tests.gpu_util import (check_bf16, check_fp32, dev, dev_i32, host, sample_candidates, stream)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    from request_candidate_sharing_b200 import rocs
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    h = rocs.Rocs(0)
    yield h
    h.close()


def _status_ok(R):
    assert R.rocs_get_device_status(stream()) == 0


# ---------------------------------------------------------------------------------------------
# a0
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("counts", [[3, 0, 5, 1], [64] * 4, [0], [1],
                                    synth.model_cfg3().counts.tolist(), synth.model_cfg5().counts.tolist(),
                                    [7] * 3000])
def test_segments_bit_exact(R, counts):
    from request_candidate_sharing_b200 import rocs
    counts = np.asarray(counts, np.int32)
    off_ref, m_ref = O.segments(counts)
    B_C = int(counts.sum())
    off = torch.full((len(counts) + 1,), -7, dtype=torch.int32, device="cuda")
    m = torch.full((max(B_C, 1),), -7, dtype=torch.int32, device="cuda")
    R.rocs_segments_from_counts(dev_i32(counts), len(counts), off, m, B_C, stream())
    _status_ok(R)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    if B_C:
        assert np.array_equal(m.cpu().numpy(), m_ref)


def test_segments_count_mismatch_sets_status(R):
    from request_candidate_sharing_b200 import rocs
    counts = np.array([3, 4], np.int32)
    off = torch.zeros(3, dtype=torch.int32, device="cuda")
    m = torch.full((5,), -1, dtype=torch.int32, device="cuda")
    R.rocs_segments_from_counts(dev_i32(counts), 2, off, m, 5, stream())
    assert R.rocs_get_device_status(stream()) == rocs.ROCS_ERR_COUNTS
    assert np.all(m.cpu().numpy()[:3] == 0)      # only slots inside [0, B_C) written
    assert R.rocs_get_device_status(stream()) == 0   # status cleared


# ---------------------------------------------------------------------------------------------
# a1-a3 IKBO linear
# ---------------------------------------------------------------------------------------------
def _run_linear(R, case, x, m, dtype_in, dtype_out):
    from request_candidate_sharing_b200 import rocs
    tdt = torch.bfloat16 if dtype_in == rocs.ROCS_BF16 else torch.float32
    odt = torch.bfloat16 if dtype_out == rocs.ROCS_BF16 else torch.float32
    d = rocs.IkboDesc(case.B_R, case.B_C, case.d_R_in, case.d_C_in, case.d_R_out, case.d_C_out, dtype_in,
                      dtype_out, rocs.ACT[case.act])
    ws_bytes = R.rocs_linear_ikbo_workspace(d)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    t = {k: dev(v, tdt) for k, v in x.items() if k.startswith(("X", "W"))}
    bR, bC = dev(x["b_R"], torch.float32), dev(x["b_C"], torch.float32)
    YR = torch.full((case.B_R, case.d_R_out), float("nan"), dtype=odt, device="cuda")
    YC = torch.full((max(case.B_C, 1), case.d_C_out), float("nan"), dtype=odt, device="cuda")
    R.rocs_linear_ikbo(d, t["X_R"], t["X_C"], dev_i32(m), t["W_RR"], t["W_CR"], t["W_CC"], bR, bC, YR, YC, ws,
                       ws_bytes, stream())
    _status_ok(R)
    return YR, YC[:case.B_C]


def test_linear_fp32_cfg1(R):
    from request_candidate_sharing_b200 import rocs
    case = synth.linear_cfg1()
    x = synth.linear_inputs(case)
    _, m = O.segments(case.counts)
    YR, YC = _run_linear(R, case, x, m, rocs.ROCS_F32, rocs.ROCS_F32)
    rR, rC = O.glm_linear(x["X_R"], x["X_C"], m, x["W_RR"], x["W_CR"], x["W_CC"], x["b_R"], x["b_C"], case.act)
    check_fp32(host(YR), rR, what="Y_R")
    check_fp32(host(YC), rC, what="Y_C")


@pytest.mark.parametrize("dtype_in", [0, 1])
@pytest.mark.parametrize("shape", [
    # (counts, d_R_in, d_C_in, d_R_out, d_C_out): tails in M, N and K; empty request
    ([70, 0, 190], 192, 320, 136, 264),
    ([1, 2, 3], 64, 64, 32, 32),
    ([129], 100, 36, 40, 300),        # K not a multiple of 8 -> alignment fix on the bf16 path
    ([5, 300], 512, 512, 0, 512),     # no request output (scoring-head form)
])
@pytest.mark.parametrize("out_dtype", [0, 1])
def test_linear_integer_inputs_bit_exact(R, dtype_in, shape, out_dtype):
    """Small integers: every product and partial sum is exact in fp32, so GPU == oracle bit for bit;
    a bf16 output is then the oracle's value rounded to nearest even.  The output widths give the
    bf16 store path odd chunk counts (136 -> 5 chunks of 32, 32 -> 1), boxes clipped at N (264, 40)
    and rows that are not 16-byte multiples (300: element stores)."""
    from request_candidate_sharing_b200 import rocs
    counts, dRi, dCi, dRo, dCo = shape
    case = synth.LinearCase("int", np.asarray(counts, np.int32), dRi, dCi, dRo, dCo, "relu", dtype_in == 1, 7)
    x = synth.linear_inputs(case, integer=3)
    _, m = O.segments(case.counts)
    if dtype_in == rocs.ROCS_F32 and out_dtype == rocs.ROCS_BF16:
        with pytest.raises(rocs.RocsError, match="fp32 path writes fp32 outputs"):   # host-checked
            _run_linear(R, case, x, m, dtype_in, out_dtype)
        return
    YR, YC = _run_linear(R, case, x, m, dtype_in, out_dtype)
    rR, rC = O.glm_linear(x["X_R"], x["X_C"], m, x["W_RR"] if dRo else None, x["W_CR"], x["W_CC"],
                          x["b_R"] if dRo else None, x["b_C"], "relu")
    expect = (lambda a: synth.bf16_round(a.astype(np.float32))) if out_dtype == 1 else (lambda a: a)
    if dRo:
        assert np.array_equal(host(YR), expect(rR))
    assert np.array_equal(host(YC), expect(rC))


@pytest.mark.parametrize("out_dtype", [0, 1])
@pytest.mark.parametrize("N,d", [(64, 512), (17, 1024), (3, 256)])
def test_linear_bf16_random(R, out_dtype, N, d):
    from request_candidate_sharing_b200 import rocs
    case = synth.linear_cfg2(N, d, B_R=9)
    x = synth.linear_inputs(case)
    _, m = O.segments(case.counts)
    YR, YC = _run_linear(R, case, x, m, rocs.ROCS_BF16, out_dtype)
    rR, rC = O.glm_linear(x["X_R"], x["X_C"], m, x["W_RR"], x["W_CR"], x["W_CC"], x["b_R"], x["b_C"], "relu")
    check_bf16(host(YR), rR, out_bf16=out_dtype == 1, what="Y_R")
    check_bf16(host(YC), rC, out_bf16=out_dtype == 1, what="Y_C")
    if out_dtype == 0:   # fp32 outputs: only accumulation-order error remains
        check_fp32(host(YC), rC, rel=1e-4, what="Y_C fp32")


def test_linear_glm_invariant_and_row_independence_gpu(R):
    from request_candidate_sharing_b200 import rocs
    case = synth.linear_cfg2(64, 512, B_R=6)
    x = synth.linear_inputs(case)
    _, m = O.segments(case.counts)
    YR1, YC1 = _run_linear(R, case, x, m, rocs.ROCS_BF16, rocs.ROCS_BF16)
    x2 = dict(x)
    x2["X_C"] = synth.bf16_round(x["X_C"] * -2.0 + 0.5)
    YR2, _ = _run_linear(R, case, x2, m, rocs.ROCS_BF16, rocs.ROCS_BF16)
    assert torch.equal(YR1, YR2)
    x3 = dict(x)
    x3["X_C"] = x["X_C"].copy()
    x3["X_C"][100] = synth.bf16_round(x3["X_C"][100] + 1.0)
    _, YC3 = _run_linear(R, case, x3, m, rocs.ROCS_BF16, rocs.ROCS_BF16)
    keep = torch.ones(case.B_C, dtype=torch.bool, device="cuda")
    keep[100] = False
    assert torch.equal(YC1[keep], YC3[keep]) and not torch.equal(YC1[100], YC3[100])


def test_linear_bad_request_index_sets_status(R):
    from request_candidate_sharing_b200 import rocs
    case = synth.linear_cfg2(64, 512, B_R=2)
    x = synth.linear_inputs(case)
    _, m = O.segments(case.counts)
    m = m.copy()
    m[5] = 99
    d = rocs.IkboDesc(case.B_R, case.B_C, 512, 512, 512, 512, rocs.ROCS_BF16, rocs.ROCS_F32, 1)
    nb = R.rocs_linear_ikbo_workspace(d)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    t = {k: dev(v) for k, v in x.items() if k.startswith(("X", "W"))}
    YR = torch.zeros(2, 512, device="cuda")
    YC = torch.full((case.B_C, 512), -5.0, device="cuda")
    R.rocs_linear_ikbo(d, t["X_R"], t["X_C"], dev_i32(m), t["W_RR"], t["W_CR"], t["W_CC"],
                       dev(x["b_R"], torch.float32), dev(x["b_C"], torch.float32), YR, YC, ws, nb, stream())
    assert R.rocs_get_device_status(stream()) == rocs.ROCS_ERR_INDEX
    assert torch.all(YC[5] == -5.0)       # the bad row is skipped, not written
    assert not torch.all(YC[4] == -5.0)


@pytest.mark.parametrize("N,d", [(N, d) for N in synth.CFG2_N for d in synth.CFG2_D])
def test_linear_cfg2_every_point_sampled(R, N, d):
    """Every IKBO sweep point at full size: 256 requests x N candidates, d_in = d_out = d, bf16 in
    and out, ReLU.  The GPU runs the whole batch (up to 262,144 candidates at K = 4096); the oracle
    checks every request output and four candidates of each request, its first and last among
    them.  The candidate batch is the seeded draw the sweep in bench.py times."""
    from request_candidate_sharing_b200 import rocs
    from tests.gpu_util import dev_normal_bf16
    case = synth.linear_cfg2(N, d)
    rows = sample_candidates(case.counts, 4)
    x = synth.linear_inputs(case, cand_rows=rows[:1])
    _, m = O.segments(case.counts)
    XC, x_rows = dev_normal_bf16(case.seed, "X_C", (case.B_C, d), keep_rows=rows)
    assert np.array_equal(x_rows[:1], x["X_C"])        # the same seeded draw as the oracle's generator
    x["X_C"] = x_rows
    rt = torch.from_numpy(rows).cuda()
    desc = rocs.IkboDesc(case.B_R, case.B_C, d, d, d, d, rocs.ROCS_BF16, rocs.ROCS_BF16, rocs.ACT[case.act])
    nb = R.rocs_linear_ikbo_workspace(desc)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    t = {k: dev(x[k]) for k in ("X_R", "W_RR", "W_CR", "W_CC")}
    YR = torch.full((case.B_R, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    YC = torch.full((case.B_C, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    R.rocs_linear_ikbo(desc, t["X_R"], XC, dev_i32(m), t["W_RR"], t["W_CR"], t["W_CC"],
                       dev(x["b_R"], torch.float32), dev(x["b_C"], torch.float32), YR, YC, ws, nb, stream())
    _status_ok(R)
    assert not torch.isnan(YC).any(), "candidate rows left unwritten"
    rR, rC = O.glm_linear(x["X_R"], x["X_C"], m[rows], x["W_RR"], x["W_CR"], x["W_CC"], x["b_R"], x["b_C"], "relu")
    check_bf16(host(YR), rR, out_bf16=True, what="Y_R")
    check_bf16(host(YC[rt]), rC, out_bf16=True, what="Y_C sample")


@pytest.mark.parametrize("counts,dRo,dCo,act,perm", [
    ([70, 0, 190, 33] * 80, 136, 384, "relu", False),    # 320 requests: three request row blocks, two N tiles
    ([300] * 6, 0, 256, "gelu", False),                   # no request output; one request block
    ([5, 1, 0, 200, 64] * 60, 64, 96, "none", True),      # candidates not grouped by request
])
def test_linear_fused_launch_matches_two_launches(R, counts, dRo, dCo, act, perm):
    """The one-launch IKBO form (request tiles publish completion flags, candidate epilogues wait
    for the Z tiles they gather) gives the same bits as the request and candidate launches."""
    from request_candidate_sharing_b200 import rocs
    case = synth.LinearCase("fused", np.asarray(counts, np.int32), 192, 128, dRo, dCo, act, True, 11)
    x = synth.linear_inputs(case)
    _, m = O.segments(case.counts)
    if perm:   # the ABI takes any candidate order: shuffle rows and their request indices together
        order = np.random.default_rng(3).permutation(case.B_C)
        m = m[order].copy()
        x = dict(x)
        x["X_C"] = x["X_C"][order].copy()
    try:
        R.rocs_set_ikbo_fused(0)
        YR0, YC0 = _run_linear(R, case, x, m, rocs.ROCS_BF16, rocs.ROCS_BF16)
        R.rocs_set_ikbo_fused(1)
        YR1, YC1 = _run_linear(R, case, x, m, rocs.ROCS_BF16, rocs.ROCS_BF16)
    finally:
        R.rocs_set_ikbo_fused(1)
    if dRo:
        assert torch.equal(YR0, YR1)
    assert torch.equal(YC0, YC1)
    rows = sample_candidates(case.counts, 2) if not perm else np.arange(0, case.B_C, 97)
    _, rC = O.glm_linear(x["X_R"], x["X_C"][rows], m[rows], x["W_RR"] if dRo else None, x["W_CR"], x["W_CC"],
                         x["b_R"] if dRo else None, x["b_C"], act)
    check_bf16(host(YC1[torch.from_numpy(rows).cuda()]), rC, out_bf16=True, what="Y_C fused")


def test_linear_short_k_many_candidates(R):
    """d = 256 with 159,840 candidates (K = 256: four k blocks per tile, so the gather epilogue and
    its prefetch of the next chunk's Z row dominate); ragged last tile.  Oracle on a sample, every
    row against a float32 torch evaluation of the same formula."""
    from request_candidate_sharing_b200 import rocs
    case = synth.linear_cfg2(999, 256, B_R=160)
    x = synth.linear_inputs(case)
    _, m = O.segments(case.counts)
    YR, YC = _run_linear(R, case, x, m, rocs.ROCS_BF16, rocs.ROCS_F32)
    rows = sample_candidates(case.counts, 2)
    rR, rC = O.glm_linear(x["X_R"], x["X_C"][rows], m[rows], x["W_RR"], x["W_CR"], x["W_CC"], x["b_R"], x["b_C"],
                          "relu")
    check_bf16(host(YR), rR, out_bf16=False, what="Y_R")
    check_fp32(host(YC[torch.from_numpy(rows).cuda()]), rC, rel=1e-4, what="Y_C sample")
    t = {k: torch.from_numpy(np.asarray(v, np.float32)).cuda() for k, v in x.items()}
    z = t["X_R"] @ t["W_CR"].T + t["b_C"]
    ref = torch.relu(t["X_C"] @ t["W_CC"].T + z[torch.from_numpy(m.astype(np.int64)).cuda()])
    err = (YC - ref).abs().max().item()
    assert err <= 1e-3 * ref.abs().max().item(), err


# ---------------------------------------------------------------------------------------------
# FP8-weight (W8A16) IKBO linear
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("w_bf16", [0, 1])
def test_quantize_weights_fp8_bit_exact(R, w_bf16):
    """Per-channel E4M3 quantisation: bytes and scales equal the oracle's exactly."""
    from oracle import fp8
    from request_candidate_sharing_b200 import rocs
    g = np.random.default_rng(5)
    W = (g.standard_normal((300, 1000)) * np.exp(2 * g.standard_normal((300, 1)))).astype(np.float32)
    W[3] = 0.0
    W[7, ::3] = 1e-30
    W[9, 5] = 3e30
    if w_bf16:
        W = synth.bf16_round(W)
    Q_ref, s_ref = fp8.quantize_rows(W)
    Q = torch.empty((300, 1000), dtype=torch.uint8, device="cuda")
    sc = torch.empty(300, dtype=torch.float32, device="cuda")
    R.rocs_quantize_weights_fp8(dev(W, torch.bfloat16 if w_bf16 else torch.float32),
                                rocs.ROCS_BF16 if w_bf16 else rocs.ROCS_F32, 300, 1000, Q, sc, stream())
    _status_ok(R)
    assert np.array_equal(sc.cpu().numpy(), s_ref)
    assert np.array_equal(Q.cpu().numpy(), Q_ref)


def _run_w8(R, case, x, q, m, out_dtype):
    from request_candidate_sharing_b200 import rocs
    d = rocs.IkboDesc(case.B_R, case.B_C, case.d_R_in, case.d_C_in, case.d_R_out, case.d_C_out, rocs.ROCS_BF16,
                      out_dtype, rocs.ACT[case.act])
    nb = R.rocs_linear_ikbo_w8_workspace(d)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    odt = torch.bfloat16 if out_dtype == rocs.ROCS_BF16 else torch.float32
    YR = torch.full((case.B_R, max(case.d_R_out, 1)), float("nan"), dtype=odt, device="cuda")
    YC = torch.full((max(case.B_C, 1), case.d_C_out), float("nan"), dtype=odt, device="cuda")
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in q.items()}
    R.rocs_linear_ikbo_w8(d, dev(x["X_R"], torch.bfloat16), dev(x["X_C"], torch.bfloat16), dev_i32(m),
                          t.get("Q_RR"), t["Q_CR"], t["Q_CC"], t.get("s_RR"), t["s_CR"], t["s_CC"],
                          dev(x["b_R"], torch.float32), dev(x["b_C"], torch.float32), YR, YC, ws, nb, stream())
    _status_ok(R)
    return YR[:, :case.d_R_out], YC[:case.B_C]


@pytest.mark.parametrize("counts,dRi,dCi,dRo,dCo,out", [
    ([16], 1280, 1280, 2560, 2560, 1),               # the pages' (1, 16, 1280, 2560): small M on both sides
    ([8], 1280, 1280, 640, 640, 0),                  # (1, 8, 1280, 640), fp32 out
    ([40, 0, 23], 96, 200, 64, 136, 1),              # small M, candidate K not a multiple of 32 (expanded)
    ([300] * 5 + [7], 256, 512, 128, 384, 1),        # B_C > 64: expanded weights on the tcgen05 GEMM
    ([1] * 60 + [0] * 30, 512, 256, 0, 256, 0),     # B_R > 64 (expanded) with a small candidate side
    ([130, 5, 300] * 50, 256, 384, 72, 200, 1),      # 150 requests, 21,750 candidates: several M tiles, a ragged
                                                     # N tile, two and three weight tiles of 128 k bytes on the
                                                     # FP8 tensor-core path
    ([3] * 7, 4096, 4096, 1024, 384, 0),             # long K (64 k blocks), fp32 out
])
@pytest.mark.parametrize("tc", [0, 1])
def test_linear_ikbo_w8(R, counts, dRi, dCi, dRo, dCo, out, tc):
    """W8A16 IKBO linear against the oracle's early-broadcast evaluation with the effective weights
    q * s, on both paths: the default one (the weight-streaming kernel for sides of at most 64 rows,
    the expanded-weight GEMM otherwise) and, with tc = 1, the FP8-operand tensor-core GEMM wherever
    both input widths are multiples of 128."""
    from oracle import fp8
    case = synth.LinearCase("w8", np.asarray(counts, np.int32), dRi, dCi, dRo, dCo, "gelu", True, 13)
    x = synth.linear_inputs(case)
    _, m = O.segments(case.counts)
    q = {}
    for k in ("RR", "CR", "CC"):
        if k == "RR" and dRo == 0:
            continue
        q["Q_" + k], q["s_" + k] = fp8.quantize_rows(x["W_" + k])
    try:
        R.rocs_set_w8_tensor_cores(tc)
        YR, YC = _run_w8(R, case, x, q, m, out)
    finally:
        R.rocs_set_w8_tensor_cores(0)
    rR, rC = fp8.w8_glm_linear(x["X_R"], x["X_C"], m, q.get("Q_RR"), q.get("s_RR"), q["Q_CR"], q["s_CR"], q["Q_CC"],
                               q["s_CC"], x["b_R"] if dRo else None, x["b_C"], "gelu")
    if dRo:
        check_bf16(host(YR.float()), rR, out_bf16=out == 1, what="Y_R")
    check_bf16(host(YC.float()), rC, out_bf16=out == 1, what="Y_C")


# ---------------------------------------------------------------------------------------------
# a6 group LayerNorm
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("io", [0, 1])
@pytest.mark.parametrize("w1,w2,res,rows", [(2048, 2048, True, 37), (1024, 1024, True, 300), (256, 0, True, 1000),
                                            (100, 28, False, 9), (4096, 0, False, 3),
                                            # >= 16384 contiguous rows: the streaming (bulk-copy ring) path,
                                            # ragged against its row blocks and CTA ranges
                                            (1024, 1024, True, 20011), (256, 0, True, 40001),
                                            (512, 0, False, 16384)])
def test_group_layernorm(R, io, w1, w2, res, rows):
    g = np.random.default_rng(w1 + w2 + rows)
    tdt = torch.bfloat16 if io == 1 else torch.float32
    rnd = (lambda a: synth.bf16_round(a)) if io == 1 else (lambda a: a)
    X1 = rnd((g.standard_normal((rows, w1)) * 2 + 0.3).astype(np.float32))
    X2 = rnd(g.standard_normal((rows, w2)).astype(np.float32))
    Rr = rnd(g.standard_normal((rows, w1 + w2)).astype(np.float32)) if res else None
    gam = (1 + g.uniform(-0.1, 0.1, w1 + w2)).astype(np.float32)
    bet = g.uniform(-0.1, 0.1, w1 + w2).astype(np.float32)
    Y = torch.empty((rows, w1 + w2), dtype=tdt, device="cuda")
    R.rocs_group_layernorm(dev(X1, tdt), w1, dev(X2, tdt) if w2 else None, w2, dev(Rr, tdt) if res else None, rows,
                           dev(gam, torch.float32), dev(bet, torch.float32), 1e-5, Y, io, stream())
    _status_ok(R)
    x = np.concatenate([X1, X2], 1).astype(np.float64) + (Rr if res else 0)
    ref = O.group_layernorm(x, gam, bet)
    if io == 0:
        check_fp32(host(Y), ref, what="LN fp32")
    else:
        check_bf16(host(Y), ref, out_bf16=True, what="LN bf16")


# ---------------------------------------------------------------------------------------------
# a4 masked FM and token LCB
# ---------------------------------------------------------------------------------------------
def _glm_small(counts, seed=3):
    case = synth.model_cfg3(B_R=len(counts), counts=counts, seed=seed)
    return case, synth.model_inputs(case), synth.model_weights(case)


@pytest.mark.parametrize("counts", [[3, 0, 17, 1, 40], [130, 64]])
def test_fm_masked(R, counts):
    case, x, W = _glm_small(counts)
    g = case.glm
    _, m = O.segments(case.counts)
    FR = torch.empty((case.B_R, g.n_R * g.n_R), device="cuda")
    FC = torch.empty((case.B_C, g.n_C * (g.n_R + g.n_C)), device="cuda")
    R.rocs_fm_masked(dev(x["E_R"]), dev(x["E_C"]), dev_i32(m), case.B_R, case.B_C, g.n_R, g.n_C, g.D, FR, FC, 0,
                     stream())
    _status_ok(R)
    rR, rC = O.fm_masked(x["E_R"], x["E_C"], m)
    check_fp32(host(FR), rR, what="F_R")
    check_fp32(host(FC), rC, what="F_C")


def test_fm_integer_exact(R):
    counts = np.array([2, 5], np.int32)
    _, m = O.segments(counts)
    ER = synth.small_ints(1, "ER", (2, 32, 128), 2)
    EC = synth.small_ints(1, "EC", (7, 16, 128), 2)
    FR = torch.empty((2, 1024), device="cuda")
    FC = torch.empty((7, 768), device="cuda")
    R.rocs_fm_masked(dev(ER), dev(EC), dev_i32(m), 2, 7, 32, 16, 128, FR, FC, 0, stream())
    rR, rC = O.fm_masked(ER, EC, m)
    assert np.array_equal(host(FR), rR) and np.array_equal(host(FC), rC)


@pytest.mark.parametrize("o_R,o_C", [(16, 8), (1, 1)])
def test_token_lcb(R, o_R, o_C):
    case, x, W = _glm_small([4, 0, 33])
    g = case.glm
    _, m = O.segments(case.counts)
    rng = np.random.default_rng(5)
    P_RR = synth.bf16_round(rng.standard_normal((o_R, g.n_R)).astype(np.float32) / 5)
    P_CR = synth.bf16_round(rng.standard_normal((o_C, g.n_R)).astype(np.float32) / 5)
    P_CC = synth.bf16_round(rng.standard_normal((o_C, g.n_C)).astype(np.float32) / 4)
    nb = R.rocs_token_lcb_workspace(case.B_R, o_C, g.D)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    LR = torch.empty((case.B_R, o_R * g.D + 64), device="cuda")   # wider rows: strided output
    LC = torch.empty((case.B_C, o_C * g.D), device="cuda")
    R.rocs_token_lcb(dev(x["E_R"]), dev(x["E_C"]), dev_i32(m), case.B_R, case.B_C, g.n_R, g.n_C, g.D, dev(P_RR),
                     dev(P_CR), dev(P_CC), o_R, o_C, LR, o_R * g.D + 64, LC, o_C * g.D, 0, ws, nb, stream())
    _status_ok(R)
    db = O.DenseBatch(m, case.B_R)
    rR, rC = O.token_lcb_rows(db.broadcast(x["E_R"]), db.with_probe(x["E_C"]), P_RR, P_CR, P_CC)
    check_fp32(host(LR[:, :o_R * g.D]), db.request_out(rR).reshape(case.B_R, -1), what="L_R")
    check_fp32(host(LC), db.cand_out(rC).reshape(case.B_C, -1), what="L_C")


# ---------------------------------------------------------------------------------------------
# a9 cross-attention
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("L,H,dh,counts", [(200, 4, 64, [3, 0, 40, 17]), (1024, 8, 32, [33, 1]),
                                           (5, 2, 32, [16, 2, 0]), (512, 1, 64, [70]),
                                           (1024, 8, 32, [300, 129, 0, 1000]), (200, 4, 64, [517, 2]),
                                           # key blocks with a ragged last one; many one-tile items,
                                           # which the query-tile groups take in turn
                                           (100, 2, 32, [40, 1, 0, 130]), (700, 8, 32, [5] * 40 + [300, 0, 129]),
                                           # one key block per item, hundreds of one-tile items: the
                                           # tile descriptor slots are reused at the fastest pace
                                           (50, 4, 32, [3] * 100 + [129, 1]), (64, 8, 64, [7] * 60)])
def test_cross_attention(R, L, H, dh, counts):
    counts = np.asarray(counts, np.int32)
    off, m = O.segments(counts)
    B_R, n, d = len(counts), int(counts.sum()), H * dh
    g = np.random.default_rng(L + n)
    K = synth.bf16_round(g.standard_normal((B_R, L, d)).astype(np.float32))
    V = synth.bf16_round(g.standard_normal((B_R, L, d)).astype(np.float32))
    Q = synth.bf16_round(g.standard_normal((n, d)).astype(np.float32))
    Ot = torch.full((max(n, 1), d), float("nan"), device="cuda")
    R.rocs_dca_cross_attn(dev(Q), dev(K), dev(V), dev_i32(off), B_R, n, L, H, dh, 1.0 / math.sqrt(dh), Ot, d, 0,
                          stream())
    _status_ok(R)
    ref = O.cross_attn(Q, K, V, m, H)
    check_bf16(host(Ot[:n]), ref, what="cross-attention")


@pytest.mark.parametrize("L,H,dh,counts,ragged", [
    (1024, 8, 32, [33, 1, 0, 300, 129], True),     # staged K/V (tcgen05), ragged key counts
    (200, 4, 64, [3, 0, 40, 17], True),            # staged, d_h 64
    (1536, 8, 32, [70, 5, 200], True),             # L d_h = 49152: streamed through shared memory
    (2048, 4, 64, [9, 130], False),                # long history, every key valid
])
def test_cross_attention_ragged_and_long(R, L, H, dh, counts, ragged):
    """Per-request key counts (a ragged history: keys past kv_len[r] are padding, here filled with
    large values that would dominate any softmax they entered) and histories longer than the
    staged kernel holds, against the oracle on the truncated histories."""
    counts = np.asarray(counts, np.int32)
    off, m = O.segments(counts)
    B_R, n, d = len(counts), int(counts.sum()), H * dh
    g = np.random.default_rng(L + n + 7)
    K = synth.bf16_round(g.standard_normal((B_R, L, d)).astype(np.float32))
    V = synth.bf16_round(g.standard_normal((B_R, L, d)).astype(np.float32))
    Q = synth.bf16_round(g.standard_normal((n, d)).astype(np.float32))
    kv_len = synth.hist_lengths(L, B_R, L, 1) if ragged else None
    if ragged:
        for r in range(B_R):
            K[r, kv_len[r]:] = 64.0
            V[r, kv_len[r]:] = 1e4
    Ot = torch.full((max(n, 1), d), float("nan"), device="cuda")
    R.rocs_dca_cross_attn(dev(Q), dev(K), dev(V), dev_i32(off), B_R, n, L, H, dh, 1.0 / math.sqrt(dh), Ot, d, 0,
                          stream(), kv_len=dev_i32(kv_len) if ragged else None)
    _status_ok(R)
    ref = O.cross_attn(Q, K, V, m, H, kv_len=kv_len)
    check_bf16(host(Ot[:n]), ref, what="ragged/long cross-attention")


def test_cross_attention_bad_length_sets_status(R):
    from request_candidate_sharing_b200 import rocs
    B_R, L, H, dh = 2, 256, 8, 32
    d = H * dh
    off = np.asarray([0, 4, 9], np.int32)
    z = dev(np.zeros((B_R, L, d), np.float32))
    Ot = torch.full((9, d), -2.0, device="cuda")
    R.rocs_dca_cross_attn(dev(np.ones((9, d), np.float32)), z, z, dev_i32(off), B_R, 9, L, H, dh, 0.1, Ot, d, 0,
                          stream(), kv_len=dev_i32(np.asarray([L + 1, 5], np.int32)))
    assert R.rocs_get_device_status(stream()) == rocs.ROCS_ERR_COUNTS
    assert torch.all(Ot[:4] == -2.0) and not torch.all(Ot[4:] == -2.0)


# ---------------------------------------------------------------------------------------------
# candidates in any order: stable sort by request, and the cross-attention over it
# ---------------------------------------------------------------------------------------------
def _sort_case(kind, B_R, B_C, seed=0):
    g = np.random.default_rng(seed)
    if kind == "random":
        return g.integers(0, B_R, B_C).astype(np.int32)
    if kind == "grouped":
        return np.sort(g.integers(0, B_R, B_C)).astype(np.int32)
    if kind == "reversed":
        return np.sort(g.integers(0, B_R, B_C))[::-1].astype(np.int32).copy()
    if kind == "one_request":
        return np.full(B_C, B_R - 1, np.int32)
    if kind == "runs":   # grouped runs that revisit requests, crossing chunk boundaries
        return np.repeat(g.integers(0, B_R, B_C // 700 + 1), 700)[:B_C].astype(np.int32)
    raise ValueError(kind)


@pytest.mark.parametrize("kind,B_R,B_C", [("random", 512, 242464), ("grouped", 512, 100000), ("reversed", 37, 5000),
                                          ("one_request", 3, 4099), ("runs", 64, 50001), ("random", 1, 33),
                                          ("random", 5, 1), ("random", 70000, 300000)])
def test_sort_by_request_bit_exact(R, kind, B_R, B_C):
    """The device counting sort gives the oracle's stable permutation and offsets exactly."""
    m = _sort_case(kind, B_R, B_C)
    perm_ref, off_ref = O.sort_by_request(m, B_R)
    nb = R.rocs_sort_by_request_workspace(B_R, B_C)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    perm = torch.full((B_C,), -7, dtype=torch.int32, device="cuda")
    off = torch.full((B_R + 1,), -7, dtype=torch.int32, device="cuda")
    R.rocs_sort_by_request(dev_i32(m), B_R, B_C, perm, off, ws, nb, stream())
    _status_ok(R)
    assert np.array_equal(perm.cpu().numpy(), perm_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)


def test_sort_by_request_bad_indices(R):
    """Indices outside [0, B_R) sort last in their given order, are not counted in offsets[B_R],
    and set ROCS_ERR_INDEX."""
    from request_candidate_sharing_b200 import rocs
    B_R, B_C = 40, 9000
    m = _sort_case("random", B_R, B_C, seed=4)
    m[[0, 17, 4500, 8999]] = [-1, 40, 1 << 30, -5]
    perm_ref, off_ref = O.sort_by_request(m, B_R)
    nb = R.rocs_sort_by_request_workspace(B_R, B_C)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    perm = torch.empty(B_C, dtype=torch.int32, device="cuda")
    off = torch.empty(B_R + 1, dtype=torch.int32, device="cuda")
    R.rocs_sort_by_request(dev_i32(m), B_R, B_C, perm, off, ws, nb, stream())
    assert R.rocs_get_device_status(stream()) == rocs.ROCS_ERR_INDEX
    assert np.array_equal(perm.cpu().numpy(), perm_ref) and np.array_equal(off.cpu().numpy(), off_ref)
    assert off_ref[-1] == B_C - 4


@pytest.mark.parametrize("L,H,dh,counts,out,extra", [(1024, 8, 32, [33, 1, 0, 300, 129], 0, 8),
                                                     (200, 4, 64, [3, 0, 40, 17], 1, 8),
                                                     (1024, 8, 32, [2000, 16, 700], 1, 2)])
def test_cross_attention_unsorted(R, L, H, dh, counts, out, extra):
    """Query rows in a shuffled order, each with its request index: the result equals the grouped
    call on the same rows bit for bit (after un-shuffling) and the oracle within the bf16 bound.
    Output rows wider than H d_h by `extra`: 8 keeps rows 16-byte aligned (the attention writes
    each row at its caller position), 2 does not (grouped output, then a row scatter)."""
    from request_candidate_sharing_b200 import rocs
    counts = np.asarray(counts, np.int32)
    off, m = O.segments(counts)
    B_R, n, d = len(counts), int(counts.sum()), H * dh
    g = np.random.default_rng(L + n + 1)
    K = synth.bf16_round(g.standard_normal((B_R, L, d)).astype(np.float32))
    V = synth.bf16_round(g.standard_normal((B_R, L, d)).astype(np.float32))
    Q = synth.bf16_round(g.standard_normal((n, d)).astype(np.float32))
    order = g.permutation(n)                 # shuffled position i holds grouped row order[i]
    Qs, ms = Q[order], m[order]
    odt = torch.bfloat16 if out == 1 else torch.float32
    scale = 1.0 / math.sqrt(dh)
    Og = torch.full((n, d), float("nan"), dtype=odt, device="cuda")
    R.rocs_dca_cross_attn(dev(Q), dev(K), dev(V), dev_i32(off), B_R, n, L, H, dh, scale, Og, d, out, stream())
    _status_ok(R)
    nb = R.rocs_dca_cross_attn_unsorted_workspace(B_R, n, H, dh, out)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    Ou = torch.full((n, d + extra), float("nan"), dtype=odt, device="cuda")   # wider rows: ld_O > H d_h
    R.rocs_dca_cross_attn_unsorted(dev(Qs), dev(K), dev(V), dev_i32(ms), B_R, n, L, H, dh, scale, Ou, d + extra, out,
                                   ws, nb, stream())
    _status_ok(R)
    assert torch.equal(Ou[:, :d], Og[torch.from_numpy(order).cuda()])
    assert torch.isnan(Ou[:, d:].float()).all()          # columns past H d_h untouched
    ref = O.cross_attn(Qs, K, V, ms, H)
    check_bf16(host(Ou[:, :d].float()), ref, out_bf16=out == 1, what="unsorted cross-attention")


def test_cross_attention_unsorted_bad_index_rows_untouched(R):
    from request_candidate_sharing_b200 import rocs
    B_R, L, H, dh, n = 3, 256, 8, 32, 500
    d = H * dh
    g = np.random.default_rng(9)
    K = synth.bf16_round(g.standard_normal((B_R, L, d)).astype(np.float32))
    V = synth.bf16_round(g.standard_normal((B_R, L, d)).astype(np.float32))
    Q = synth.bf16_round(g.standard_normal((n, d)).astype(np.float32))
    m = g.integers(0, B_R, n).astype(np.int32)
    m[[5, 77]] = [3, -2]
    nb = R.rocs_dca_cross_attn_unsorted_workspace(B_R, n, H, dh, 0)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    Ou = torch.full((n, d), -3.0, device="cuda")
    R.rocs_dca_cross_attn_unsorted(dev(Q), dev(K), dev(V), dev_i32(m), B_R, n, L, H, dh, 1.0 / math.sqrt(dh), Ou, d, 0,
                                   ws, nb, stream())
    assert R.rocs_get_device_status(stream()) == rocs.ROCS_ERR_INDEX
    assert torch.all(Ou[5] == -3.0) and torch.all(Ou[77] == -3.0)
    ok = np.setdiff1d(np.arange(n), [5, 77])
    ref = O.cross_attn(Q[ok], K, V, m[ok], H)
    check_bf16(host(Ou[torch.from_numpy(ok).cuda()]), ref, what="valid rows")


# ---------------------------------------------------------------------------------------------
# a7 DCA encoder
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("L,lengths", [(256, [256, 1, 100]), (1536, [1536, 700])])
def test_dca_encode_ragged_and_long(R, L, lengths):
    """Ragged histories (each request keeps its first lengths[r] rows; the padding rows hold NaN,
    so a leak into any history row would show) and a history longer than the staged attention
    kernels hold (streamed).  History rows of S and K/V against the oracle."""
    from request_candidate_sharing_b200 import rocs
    lengths = np.asarray(lengths, np.int32)
    case = synth.model_cfg4(B_R=len(lengths), counts=[1] * len(lengths))
    case.dca.L = L
    a = case.dca
    W = synth.model_weights(case)
    x = synth.model_inputs(case)
    Hn = x["H"].copy()
    for r, Lr in enumerate(lengths):
        Hn[r, Lr:] = np.nan
    Wd = {k: dev(v, torch.float32 if ("ln." in k) else torch.bfloat16) for k, v in W.items()}
    desc = rocs.DcaDesc(case.B_R, a.L, a.d, a.H, a.layers)
    nb = R.rocs_dca_encode_workspace(desc)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    S = torch.empty((a.layers, case.B_R, a.L, a.d), dtype=torch.bfloat16, device="cuda")
    KV = torch.empty((a.layers, 4, case.B_R, a.L, a.d), dtype=torch.bfloat16, device="cuda")
    R.rocs_dca_encode(desc, dev(Hn), [rocs.dca_layer_weights(Wd, l) for l in range(a.layers)], S, KV, ws, nb,
                      stream(), lengths=dev_i32(lengths))
    _status_ok(R)
    Ss, KVs = O.dca_encode(x["H"], W, a.layers, a.H, lengths)
    for l in range(a.layers):
        for r, Lr in enumerate(lengths):
            check_bf16(host(S[l, r, :Lr]), Ss[l][r, :Lr], out_bf16=True, what=f"S_{l} request {r}")
            for i in range(4):
                check_bf16(host(KV[l, i, r, :Lr]), KVs[l][i][r, :Lr], out_bf16=True, what=f"KV_{l}_{i} request {r}")


def test_dca_encode(R):
    from request_candidate_sharing_b200 import rocs
    case = synth.model_cfg4(B_R=3, counts=[1, 1, 1])
    a = case.dca
    W = synth.model_weights(case)
    x = synth.model_inputs(case)
    Wd = {k: dev(v, torch.float32 if ("ln." in k) else torch.bfloat16) for k, v in W.items()}
    desc = rocs.DcaDesc(case.B_R, a.L, a.d, a.H, a.layers)
    nb = R.rocs_dca_encode_workspace(desc)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    S = torch.empty((a.layers, case.B_R, a.L, a.d), dtype=torch.bfloat16, device="cuda")
    KV = torch.empty((a.layers, 4, case.B_R, a.L, a.d), dtype=torch.bfloat16, device="cuda")
    R.rocs_dca_encode(desc, dev(x["H"]), [rocs.dca_layer_weights(Wd, l) for l in range(a.layers)], S, KV, ws, nb,
                      stream())
    _status_ok(R)
    Ss, KVs = O.dca_encode(x["H"], W, a.layers, a.H)
    for l in range(a.layers):
        check_bf16(host(S[l]), Ss[l], out_bf16=True, what=f"S_{l}")
        for i in range(4):
            check_bf16(host(KV[l, i]), KVs[l][i], out_bf16=True, what=f"KV_{l}_{i}")
