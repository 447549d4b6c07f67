"""Out-of-bounds writes, caught with guard bands (GPU).

Every output and workspace buffer of each entry point is placed inside a larger allocation whose
bytes before and after it hold a sentinel pattern; after the call those bands must be unchanged.
Shapes are chosen with ragged tails (rows not a multiple of the 128-row tiles, columns not a
multiple of the 32- and 256-wide epilogue chunks, history lengths not a multiple of the 128-key
blocks), which is where a kernel's last tile or its TMA store box could reach past the end of a
row or of the buffer.  This is the test-side stand-in for a memory checker, which is not
available on these GPUs.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import rocs_oracle as O
from tests.gpu_util import dev, dev_i32, stream

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (a multiple of 256: the buffer keeps its alignment)
SENTINEL = 0xA5


class Guarded:
    """A device tensor of `shape` and `dtype` inside sentinel bands of GUARD bytes."""

    def __init__(self, shape, dtype, fill=float("nan")):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((2 * GUARD + ((n + 255) // 256) * 256,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(*shape)
        if dtype.is_floating_point:
            self.t.fill_(fill)

    def check(self, what):
        before = self.raw[:GUARD]
        after = self.raw[GUARD + self.n:]
        assert bool((before == SENTINEL).all()), f"{what}: write before the buffer"
        assert bool((after == SENTINEL).all()), f"{what}: write after the buffer"


@pytest.fixture(scope="module")
def R():
    from request_candidate_sharing_b200 import rocs
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    h = rocs.Rocs(0)
    yield h
    h.close()


def _ok(R):
    assert R.rocs_get_device_status(stream()) == 0


@pytest.mark.parametrize("dtype_in,dtype_out,fused", [(1, 1, 1), (1, 0, 1), (1, 1, 0), (0, 0, 1)])
def test_linear_ikbo_stays_in_bounds(R, dtype_in, dtype_out, fused):
    from request_candidate_sharing_b200 import rocs
    counts = np.asarray([70, 0, 190, 33, 1], np.int32)          # 294 candidates: a ragged 128-row tile
    case = synth.LinearCase("guard", counts, 192, 136, 72, 200, "relu", dtype_in == 1, 3)   # N tails
    x = synth.linear_inputs(case)
    _, m = O.segments(case.counts)
    tdt = torch.bfloat16 if dtype_in == 1 else torch.float32
    odt = torch.bfloat16 if dtype_out == 1 else torch.float32
    d = rocs.IkboDesc(case.B_R, case.B_C, case.d_R_in, case.d_C_in, case.d_R_out, case.d_C_out, dtype_in, dtype_out,
                      rocs.ACT["relu"])
    nb = R.rocs_linear_ikbo_workspace(d)
    ws = Guarded((max(nb, 16),), torch.uint8)
    YR, YC = Guarded((case.B_R, case.d_R_out), odt), Guarded((case.B_C, case.d_C_out), odt)
    t = {k: dev(v, tdt) for k, v in x.items() if k.startswith(("X", "W"))}
    try:
        R.rocs_set_ikbo_fused(fused)
        R.rocs_linear_ikbo(d, t["X_R"], t["X_C"], dev_i32(m), t["W_RR"], t["W_CR"], t["W_CC"], dev(x["b_R"], torch.float32),
                           dev(x["b_C"], torch.float32), YR.t, YC.t, ws.t, nb, stream())
        _ok(R)
    finally:
        R.rocs_set_ikbo_fused(1)
    for g, w in ((YR, "Y_R"), (YC, "Y_C"), (ws, "workspace")):
        g.check(w)
    assert not torch.isnan(YC.t.float()).any() and not torch.isnan(YR.t.float()).any()


@pytest.mark.parametrize("tc", [0, 1])
def test_linear_ikbo_w8_stays_in_bounds(R, tc):
    from oracle import fp8
    from request_candidate_sharing_b200 import rocs
    counts = np.asarray([40, 0, 23, 150], np.int32)
    case = synth.LinearCase("guard8", counts, 256, 384, 72, 200, "gelu", True, 5)
    x = synth.linear_inputs(case)
    _, m = O.segments(case.counts)
    q = {}
    for k in ("RR", "CR", "CC"):
        q["Q_" + k], q["s_" + k] = fp8.quantize_rows(x["W_" + k])
    d = rocs.IkboDesc(case.B_R, case.B_C, case.d_R_in, case.d_C_in, case.d_R_out, case.d_C_out, rocs.ROCS_BF16,
                      rocs.ROCS_BF16, rocs.ACT["gelu"])
    try:
        R.rocs_set_w8_tensor_cores(tc)
        nb = R.rocs_linear_ikbo_w8_workspace(d)
        ws = Guarded((max(nb, 16),), torch.uint8)
        YR, YC = Guarded((case.B_R, case.d_R_out), torch.bfloat16), Guarded((case.B_C, case.d_C_out), torch.bfloat16)
        tq = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in q.items()}
        R.rocs_linear_ikbo_w8(d, dev(x["X_R"]), dev(x["X_C"]), dev_i32(m), tq["Q_RR"], tq["Q_CR"], tq["Q_CC"], tq["s_RR"],
                              tq["s_CR"], tq["s_CC"], dev(x["b_R"], torch.float32), dev(x["b_C"], torch.float32), YR.t,
                              YC.t, ws.t, nb, stream())
        _ok(R)
    finally:
        R.rocs_set_w8_tensor_cores(0)
    for g, w in ((YR, "Y_R"), (YC, "Y_C"), (ws, "workspace")):
        g.check(w)


@pytest.mark.parametrize("io", [0, 1])
@pytest.mark.parametrize("w1,w2,rows", [(2048, 2048, 20011), (256, 0, 37), (1000, 24, 3)])
def test_group_layernorm_stays_in_bounds(R, io, w1, w2, rows):
    from request_candidate_sharing_b200 import rocs
    dt = torch.bfloat16 if io == 1 else torch.float32
    g = torch.Generator(device="cuda").manual_seed(1)
    X1 = torch.randn(rows, w1, device="cuda", generator=g).to(dt)
    X2 = torch.randn(rows, w2, device="cuda", generator=g).to(dt) if w2 else None
    res = torch.randn(rows, w1 + w2, device="cuda", generator=g).to(dt)
    gamma = torch.ones(w1 + w2, device="cuda")
    beta = torch.zeros(w1 + w2, device="cuda")
    Y = Guarded((rows, w1 + w2), dt)
    R.rocs_group_layernorm(X1, w1, X2, w2, res, rows, gamma, beta, 1e-5, Y.t, rocs.ROCS_BF16 if io else rocs.ROCS_F32,
                           stream())
    _ok(R)
    Y.check("Y")


def test_fm_and_token_lcb_stay_in_bounds(R):
    from request_candidate_sharing_b200 import rocs
    counts = np.asarray([3, 0, 17, 1, 40], np.int32)
    case = synth.model_cfg3(B_R=len(counts), counts=counts)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    g = case.glm
    _, m = O.segments(case.counts)
    ER, EC, mi = dev(x["E_R"]), dev(x["E_C"]), dev_i32(m)
    FR = Guarded((case.B_R, g.n_R * g.n_R), torch.float32)
    FC = Guarded((case.B_C, g.n_C * (g.n_R + g.n_C)), torch.float32)
    R.rocs_fm_masked(ER, EC, mi, case.B_R, case.B_C, g.n_R, g.n_C, g.D, FR.t, FC.t, rocs.ROCS_F32, stream())
    _ok(R)
    FR.check("F_R")
    FC.check("F_C")
    nb = R.rocs_token_lcb_workspace(case.B_R, g.lcb_out_C, g.D)
    ws = Guarded((max(nb, 16),), torch.uint8)
    LR = Guarded((case.B_R, g.lcb_out_R * g.D), torch.float32)
    LC = Guarded((case.B_C, g.lcb_out_C * g.D), torch.float32)
    Pw = {k: dev(W["glm0.lcb." + k]) for k in ("P_RR", "P_CR", "P_CC")}
    R.rocs_token_lcb(ER, EC, mi, case.B_R, case.B_C, g.n_R, g.n_C, g.D, Pw["P_RR"], Pw["P_CR"], Pw["P_CC"],
                     g.lcb_out_R, g.lcb_out_C, LR.t, g.lcb_out_R * g.D, LC.t, g.lcb_out_C * g.D, rocs.ROCS_F32, ws.t, nb,
                     stream())
    _ok(R)
    for buf, w in ((LR, "L_R"), (LC, "L_C"), (ws, "workspace")):
        buf.check(w)


@pytest.mark.parametrize("L,H,dh,counts,ragged", [(1024, 8, 32, [33, 1, 0, 130], False),
                                                   (200, 4, 64, [3, 0, 140, 17], False),
                                                   (1536, 8, 32, [5, 70], False),
                                                   (1024, 8, 32, [129, 2, 40], True)])
def test_cross_attention_stays_in_bounds(R, L, H, dh, counts, ragged):
    from request_candidate_sharing_b200 import rocs
    counts = np.asarray(counts, np.int32)
    B_R, B_C, d = len(counts), int(counts.sum()), H * dh
    gen = torch.Generator(device="cuda").manual_seed(2)
    Q = torch.randn(B_C, d, device="cuda", generator=gen).to(torch.bfloat16)
    K = torch.randn(B_R * L, d, device="cuda", generator=gen).to(torch.bfloat16)
    V = torch.randn(B_R * L, d, device="cuda", generator=gen).to(torch.bfloat16)
    off, _ = O.segments(counts)
    kv_len = dev_i32(np.asarray([L, 77, 1, 500][:B_R], np.int32)) if ragged else None
    Og = Guarded((B_C, d), torch.float32)
    R.rocs_dca_cross_attn(Q, K, V, dev_i32(off), B_R, B_C, L, H, dh, 1.0 / math.sqrt(dh), Og.t, d, rocs.ROCS_F32,
                          stream(), kv_len=kv_len)
    _ok(R)
    Og.check("O")
    assert not torch.isnan(Og.t).any()


def test_sort_and_segments_stay_in_bounds(R):
    from request_candidate_sharing_b200 import rocs
    counts = np.asarray([3, 0, 5, 1, 700], np.int32)
    B_R, B_C = len(counts), int(counts.sum())
    off = Guarded((B_R + 1,), torch.int32)
    mi = Guarded((B_C,), torch.int32)
    R.rocs_segments_from_counts(dev_i32(counts), B_R, off.t, mi.t, B_C, stream())
    _ok(R)
    off.check("offsets")
    mi.check("req_idx")
    keys = np.random.default_rng(4).integers(-1, B_R + 1, size=3001).astype(np.int32)
    nb = R.rocs_sort_by_request_workspace(B_R, len(keys))
    ws = Guarded((max(nb, 16),), torch.uint8)
    perm = Guarded((len(keys),), torch.int32)
    offs = Guarded((B_R + 1,), torch.int32)
    R.rocs_sort_by_request(dev_i32(keys), B_R, len(keys), perm.t, offs.t, ws.t, nb, stream())
    assert R.rocs_get_device_status(stream()) == rocs.ROCS_ERR_INDEX      # the invalid keys are reported
    for buf, w in ((perm, "perm"), (offs, "offsets"), (ws, "workspace")):
        buf.check(w)


def test_forward_stays_in_bounds(R):
    """The end-to-end forward with every output and the workspace guarded: ragged candidate counts
    (a one-candidate request, a 20-candidate one) and a history of 256."""
    from request_candidate_sharing_b200 import rocs
    from tests.test_gpu_forward import FP32_KEYS
    case = synth.model_cfg5(B_R=3, counts=[4, 1, 20], L=256)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    md = rocs.model_desc(case)
    Wd = {k: dev(v, torch.float32 if k.endswith(FP32_KEYS) else torch.bfloat16) for k, v in W.items()}
    g, a = case.glm, case.dca
    mw = rocs.model_weights(Wd, g.layers, a.layers, True)
    xin = {k: dev(v) for k, v in x.items()}
    counts = dev_i32(case.counts)
    inp = rocs.Inputs(counts.data_ptr(), rocs.ptr(xin.get("E_R")), rocs.ptr(xin.get("E_C")), rocs.ptr(xin.get("H")),
                      None, None, None)
    B_R, B_C = case.B_R, case.B_C
    outs = {"offsets": Guarded((B_R + 1,), torch.int32), "req_idx": Guarded((B_C,), torch.int32),
            "E_R": Guarded((B_R, g.n_R, g.D), torch.float32), "E_C": Guarded((B_C, g.n_C, g.D), torch.float32),
            "S": Guarded((a.layers, B_R, a.L, a.d), torch.bfloat16),
            "A_R": Guarded((a.layers, B_R, a.d), torch.float32), "A_C": Guarded((a.layers, B_C, a.d), torch.float32),
            "score": Guarded((B_C,), torch.float32)}
    o = rocs.Outputs(*[outs[k].t.data_ptr() for k in ("offsets", "req_idx", "E_R", "E_C", "S", "A_R", "A_C", "score")])
    nb = R.rocs_forward_workspace(md)
    ws = Guarded((nb,), torch.uint8)
    try:
        R.rocs_set_graph_replay(0)
        R.rocs_forward(md, mw, inp, o, ws.t, nb, stream())
        _ok(R)
    finally:
        R.rocs_set_graph_replay(1)
    for k, buf in outs.items():
        buf.check(k)
    ws.check("workspace")
    assert not torch.isnan(outs["score"].t).any()
