"""Pins for the oracle's compositions (CPU only).

The oracle's primitives are each pinned on their own (tests/test_oracle.py).  These tests pin how
they are wired together, against per-request / per-candidate loop compositions written
independently in oracle/tiny.py from the same readings:
  * the Wukong layer: FM -> flatten -> two-group MLP (GELU hidden) -> tokens; token-axis LCB;
    concat [FM-block tokens, LCB tokens]; residual add of the layer input; group-local LayerNorm
    ("ROCS：面向请求的大规模推荐计算共享" review, §2.1 Figure 1(d), Figure 2);
  * the DCA query generator [Q^R; Q^C] = MLP_i(LCB_i(.)) and the depth wiring of the DCA path
    (same review, §2.2), with attention outputs appended as one token per group (DCA's own
    query embeddings) or query tokens read from the previous GLM layer's output (end-to-end
    forward), and the candidate scoring head;
  * the FP8-weight two-group linear ("Compute Only Once: UG-Separation ..." review, §三 Stage 4).

Each pin is followed by planted mistakes: the oracle function's source with one plausible error
(an operand order, an operation moved, a weight taken from the wrong block) is executed in place
of the real one on the CPU, and the same comparison must then fail.  This shows that the pin
would catch that mistake.
"""
import inspect
import math
import textwrap

import numpy as np
import pytest

import synth
from oracle import fp8
from oracle import rocs_oracle as O
from oracle import tiny

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")

EXACT = 1e-10       # float64 vectorised oracle vs float64 loops: rounding order only
PLANTED = 1e-4      # a planted mistake must move some output by more than this


def _glm_shape(layers=2):
    # token counts chosen unequal so that every concatenation and reshape is checked:
    # 3 FM-block tokens + 1 LCB token = 4 request tokens, 1 + 1 = 2 candidate tokens
    return synth.GLMShape(n_R=4, n_C=2, D=3, hidden=5, fm_out_R=3, fm_out_C=1,
                          lcb_out_R=1, lcb_out_C=1, layers=layers)


def _case3(counts=(2, 0, 3)):
    return synth.ModelCase("tiny_glm", np.asarray(counts, np.int32), 7, _glm_shape(), None, None)


def _case4(counts=(2, 3)):
    dca = synth.DCAShape(L=3, d=4, H=2, layers=2, q_n_R=3, q_n_C=2, q_dim=4, source="own")
    return synth.ModelCase("tiny_dca", np.asarray(counts, np.int32), 8, None, dca, None)


def _case5(counts=(2, 1, 3)):
    dca = synth.DCAShape(L=3, d=4, H=2, layers=2, q_n_R=4, q_n_C=2, q_dim=3, source="glm")
    return synth.ModelCase("tiny_e2e", np.asarray(counts, np.int32), 9, _glm_shape(), dca, (5, 3))


def _lists(a):
    return np.asarray(a, np.float64).tolist()


def _maxdiff(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def _mutant(module, fname, old, new):
    """`module.fname` with the one source fragment `old` replaced by `new`, compiled against a
    copy of the module's globals (so it still calls the real versions of everything else)."""
    src = textwrap.dedent(inspect.getsource(getattr(module, fname)))
    assert src.count(old) == 1, f"planted mistake: {old!r} not found exactly once in {fname}"
    ns = dict(module.__dict__)
    exec(compile(src.replace(old, new), f"<mutant {fname}>", "exec"), ns)
    return ns[fname]


# ---------------------------------------------------------------------------------------------
# Wukong layer (the GLM stack)
# ---------------------------------------------------------------------------------------------
def _glm_error():
    case = _case3()
    W, x = synth.model_weights(case), synth.model_inputs(case)
    _, m = O.segments(case.counts)
    out = O.forward_cfg3(case, x, W, m)
    ER, EC = _lists(x["E_R"]), _lists(x["E_C"])
    err = 0.0
    for l in range(case.glm.layers):
        ER, EC = tiny.wukong_layer(ER, EC, m.tolist(), W, f"glm{l}.", case.glm)
        oR, oC = out["layers"][l + 1]
        err = max(err, _maxdiff(oR, ER), _maxdiff(oC, EC))
    return err


def test_wukong_layer_matches_loop_composition():
    assert _glm_error() <= EXACT


WUKONG_MISTAKES = {
    "concat order [L, o] in the request group":
        ("[oR.reshape(b, g.fm_out_R, g.D), LR]", "[LR, oR.reshape(b, g.fm_out_R, g.D)]"),
    "concat order [L, o] in the candidate group":
        ("[oC.reshape(b, g.fm_out_C, g.D), LC]", "[LC, oC.reshape(b, g.fm_out_C, g.D)]"),
    "LayerNorm before the residual (request group)":
        ('group_layernorm((catR + ER).reshape(b, -1), W[pre + "lnR.gamma"], W[pre + "lnR.beta"])',
         'group_layernorm(catR.reshape(b, -1), W[pre + "lnR.gamma"], W[pre + "lnR.beta"]) + ER.reshape(b, -1)'),
    "LayerNorm before the residual (candidate group)":
        ('group_layernorm((catC + EC).reshape(b, -1), W[pre + "lnC.gamma"], W[pre + "lnC.beta"])',
         'group_layernorm(catC.reshape(b, -1), W[pre + "lnC.gamma"], W[pre + "lnC.beta"]) + EC.reshape(b, -1)'),
    "no GELU on the MLP hidden layer":
        ('W[pre + "mlp1.b_R"], W[pre + "mlp1.b_C"], "gelu")', 'W[pre + "mlp1.b_R"], W[pre + "mlp1.b_C"], "none")'),
    "request group's LayerNorm parameters on the candidate group":
        ('W[pre + "lnC.gamma"], W[pre + "lnC.beta"]', 'W[pre + "lnR.gamma"][:EC[0].size], W[pre + "lnR.beta"][:EC[0].size]'),
    "token LCB without the request tokens":
        ('token_lcb_rows(ER, EC,', 'token_lcb_rows(0 * ER, EC,'),
}


@pytest.mark.parametrize("mistake", sorted(WUKONG_MISTAKES))
def test_wukong_pin_catches_planted_mistake(mistake, monkeypatch):
    old, new = WUKONG_MISTAKES[mistake]
    monkeypatch.setattr(O, "wukong_layer_rows", _mutant(O, "wukong_layer_rows", old, new))
    monkeypatch.setattr(O.DenseBatch, "check_request_copies", lambda *a, **k: None)
    assert _glm_error() > PLANTED, mistake


# ---------------------------------------------------------------------------------------------
# DCA with its own query embeddings: query generator and depth wiring (appended A tokens)
# ---------------------------------------------------------------------------------------------
def _dca_own_error():
    case = _case4()
    W, x = synth.model_weights(case), synth.model_inputs(case)
    _, m = O.segments(case.counts)
    out = O.forward_cfg4(case, x, W, m)
    state = {"R": _lists(x["Y_R"]), "C": _lists(x["Y_C"])}

    def own_tokens(i, prev):
        if prev is not None:                       # A_{i-1} becomes one more token per group
            aR, aC = prev
            state["R"] = [state["R"][r] + [aR[r]] for r in range(len(aR))]
            state["C"] = [state["C"][c] + [aC[c]] for c in range(len(aC))]
        return state["R"], state["C"]

    A_R, A_C = tiny.dca_depths(_lists(x["H"]), m.tolist(), W, case.dca.layers, case.dca.H, own_tokens)
    err = 0.0
    for i in range(case.dca.layers):
        err = max(err, _maxdiff(out["A_R"][i], A_R[i]), _maxdiff(out["A_C"][i], A_C[i]))
    return err


def test_dca_own_queries_match_loop_composition():
    assert _dca_own_error() <= EXACT


QUERY_GEN_MISTAKES = {
    "no GELU in the query generator's MLP":
        ('W[pre + "mlp1.b_R"], W[pre + "mlp1.b_C"], "gelu")', 'W[pre + "mlp1.b_R"], W[pre + "mlp1.b_C"], "none")'),
    "query LCB ignores the request tokens on the candidate side":
        ('W[pre + "p_CR"]', '0 * W[pre + "p_CR"]'),
    "GELU on the query generator's output":
        ('W[pre + "mlp2.b_R"], W[pre + "mlp2.b_C"], "none")', 'W[pre + "mlp2.b_R"], W[pre + "mlp2.b_C"], "gelu")'),
}

DCA_OWN_MISTAKES = {
    "attention token appended to the wrong group":
        ('state["YR"], aR[:, None, :]', 'state["YR"], aC[:, None, :]'),
    "attention token prepended instead of appended":
        ('[state["YC"], aC[:, None, :]]', '[aC[:, None, :], state["YC"]]'),
}

DEPTH_MISTAKES = {
    "request query against the candidate group's K/V":
        ("cross_attn(QR, K_R, V_R,", "cross_attn(QR, K_C, V_C,"),
    "candidate query against the request group's K/V":
        ("cross_attn(QC, K_C, V_C,", "cross_attn(QC, K_R, V_R,"),
}


@pytest.mark.parametrize("mistake", sorted(QUERY_GEN_MISTAKES))
def test_query_generator_pin_catches_planted_mistake(mistake, monkeypatch):
    old, new = QUERY_GEN_MISTAKES[mistake]
    monkeypatch.setattr(O, "query_gen_rows", _mutant(O, "query_gen_rows", old, new))
    monkeypatch.setattr(O.DenseBatch, "check_request_copies", lambda *a, **k: None)
    assert _dca_own_error() > PLANTED, mistake


@pytest.mark.parametrize("mistake", sorted(DCA_OWN_MISTAKES))
def test_dca_own_wiring_pin_catches_planted_mistake(mistake, monkeypatch):
    old, new = DCA_OWN_MISTAKES[mistake]
    monkeypatch.setattr(O, "forward_cfg4", _mutant(O, "forward_cfg4", old, new))
    monkeypatch.setattr(O.DenseBatch, "check_request_copies", lambda *a, **k: None)
    assert _dca_own_error() > PLANTED, mistake


@pytest.mark.parametrize("mistake", sorted(DEPTH_MISTAKES))
def test_dca_depth_pin_catches_planted_mistake(mistake, monkeypatch):
    old, new = DEPTH_MISTAKES[mistake]
    monkeypatch.setattr(O, "_dca_depths", _mutant(O, "_dca_depths", old, new))
    monkeypatch.setattr(O.DenseBatch, "check_request_copies", lambda *a, **k: None)
    assert _dca_own_error() > PLANTED, mistake


# ---------------------------------------------------------------------------------------------
# end-to-end forward: GLM stack, DCA queries from GLM layer outputs, scoring head
# ---------------------------------------------------------------------------------------------
def _e2e_error():
    case = _case5()
    W, x = synth.model_weights(case), synth.model_inputs(case)
    _, m = O.segments(case.counts)
    mm = m.tolist()
    out = O.forward_cfg5(case, x, W, m)
    g = case.glm
    glm_rows = [(_lists(x["E_R"]), _lists(x["E_C"]))]
    for l in range(g.layers):
        glm_rows.append(tiny.wukong_layer(*glm_rows[-1], mm, W, f"glm{l}.", g))
    # depth i reads GLM layer i's input, i.e. layer i-1's output (depth 0: the input embeddings)
    A_R, A_C = tiny.dca_depths(_lists(x["H"]), mm, W, case.dca.layers, case.dca.H,
                               lambda i, prev: glm_rows[i])
    ER, EC = glm_rows[-1]
    xR = [[v for tok in ER[r] for v in tok] + [v for i in range(case.dca.layers) for v in A_R[i][r]]
          for r in range(case.B_R)]
    xC = [[v for tok in EC[c] for v in tok] + [v for i in range(case.dca.layers) for v in A_C[i][c]]
          for c in range(case.B_C)]
    score = tiny.score_head(xR, xC, mm, W)
    err = _maxdiff(out["score"], score)
    for i in range(case.dca.layers):
        err = max(err, _maxdiff(out["A_R"][i], A_R[i]), _maxdiff(out["A_C"][i], A_C[i]))
    return err


def test_e2e_forward_matches_loop_composition():
    assert _e2e_error() <= EXACT


E2E_MISTAKES = {
    "depth i reads GLM layer i's output instead of its input":
        ("return rows[l]", "return rows[l + 1]"),
    "scoring input [A, Y] instead of [Y, A] (request part)":
        ("[ER.reshape(b, -1)] + A_R", "A_R + [ER.reshape(b, -1)]"),
    "scoring input with the depths in reverse order (candidate part)":
        ("[EC.reshape(b, -1)] + A_C", "[EC.reshape(b, -1)] + A_C[::-1]"),
    "no ReLU after the second scoring layer":
        ('W["score2.b"], "relu")', 'W["score2.b"], "none")'),
    "scoring reads the GLM input instead of the last layer":
        ("ER, EC = rows[-1]", "ER, EC = rows[0]"),
}


@pytest.mark.parametrize("mistake", sorted(E2E_MISTAKES))
def test_e2e_pin_catches_planted_mistake(mistake, monkeypatch):
    old, new = E2E_MISTAKES[mistake]
    monkeypatch.setattr(O, "forward_cfg5", _mutant(O, "forward_cfg5", old, new))
    assert _e2e_error() > PLANTED, mistake


# ---------------------------------------------------------------------------------------------
# FP8-weight two-group linear
# ---------------------------------------------------------------------------------------------
def _e4m3_value(byte):
    """The value of one E4M3 byte from the format: sign, 4 exponent bits (bias 7), 3 mantissa bits,
    exponent field 0 subnormal."""
    s = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    f = byte & 0x7
    return s * (f / 8.0 * 2.0 ** -6 if e == 0 else (1.0 + f / 8.0) * 2.0 ** (e - 7))


def _w8_glm_error(fn):
    g = np.random.default_rng(11)
    B_R, counts, dRi, dCi, dRo, dCo = 3, [2, 0, 3], 6, 5, 4, 7
    _, m = O.segments(np.asarray(counts))
    XR = g.standard_normal((B_R, dRi))
    XC = g.standard_normal((len(m), dCi))
    Q_RR, s_RR = fp8.quantize_rows(g.standard_normal((dRo, dRi)))
    Q_CR, s_CR = fp8.quantize_rows(g.standard_normal((dCo, dRi)) * 3.0)
    Q_CC, s_CC = fp8.quantize_rows(g.standard_normal((dCo, dCi)) * 0.2)
    b_R = g.uniform(-0.1, 0.1, dRo)
    b_C = g.uniform(-0.1, 0.1, dCo)
    YR, YC = fn(XR, XC, m, Q_RR, s_RR, Q_CR, s_CR, Q_CC, s_CC, b_R, b_C, "relu")
    err = 0.0
    for r in range(B_R):
        for o in range(dRo):
            acc = sum(_e4m3_value(int(Q_RR[o, i])) * float(s_RR[o]) * XR[r, i] for i in range(dRi))
            err = max(err, abs(YR[r, o] - max(acc + b_R[o], 0.0)))
    for c in range(len(m)):
        r = int(m[c])
        for o in range(dCo):
            acc = sum(_e4m3_value(int(Q_CR[o, i])) * float(s_CR[o]) * XR[r, i] for i in range(dRi))
            acc += sum(_e4m3_value(int(Q_CC[o, i])) * float(s_CC[o]) * XC[c, i] for i in range(dCi))
            err = max(err, abs(YC[c, o] - max(acc + b_C[o], 0.0)))
    return err


def test_w8_glm_linear_by_hand():
    assert _w8_glm_error(fp8.w8_glm_linear) <= EXACT


W8_MISTAKES = {
    "candidate-block scale on the cross block": ("dequantize_rows(Q_CR, s_CR)", "dequantize_rows(Q_CR, s_CC)"),
    "candidate bias dropped": ("pre + np.asarray(b_C, F64)[None, :]", "pre"),
    "cross block read from the candidate's own row index": ("X_R[m] @", "X_R[np.minimum(np.arange(len(m)), len(X_R) - 1)] @"),
}


@pytest.mark.parametrize("mistake", sorted(W8_MISTAKES))
def test_w8_pin_catches_planted_mistake(mistake):
    old, new = W8_MISTAKES[mistake]
    assert _w8_glm_error(_mutant(fp8, "w8_glm_linear", old, new)) > PLANTED, mistake


def test_tiny_gelu_against_closed_values():
    """GELU(0) = 0, GELU(x) - GELU(-x) = x, and GELU(1) = Phi(1) from the normal table."""
    assert tiny.gelu(0.0) == 0.0
    for v in (0.3, 1.7, -2.2):
        assert abs(tiny.gelu(v) - tiny.gelu(-v) - v) < 1e-15
    assert abs(tiny.gelu(1.0) - 0.8413447460685429) < 1e-15
