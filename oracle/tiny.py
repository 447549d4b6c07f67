"""Pure-Python loop versions of the oracle's operations, for tiny shapes only.

TEST INFRASTRUCTURE ONLY (same import rule as rocs_oracle).  Each function is written from
the definitions on the pages with explicit index loops and no numpy, so that it shares no
vectorised code path with rocs_oracle and a transposed operand or dropped term in either one
shows up when the two are compared.

  [REV] "ROCS：面向请求的大规模推荐计算共享" (liuzhao09.github.io review), §2.1 / §2.2 / §2.4.
"""
from __future__ import annotations

import math


def linear_two_group(XR, XC, m, W_RR, W_CR, W_CC, b_R, b_C):
    """[REV] §2.1 two-group block matrix: y^R_r[j] = sum_k W_RR[j][k] x^R_r[k] + b^R[j];
    y^C_c[j] = sum_k W_CR[j][k] x^R_{m_c}[k] + sum_k W_CC[j][k] x^C_c[k] + b^C[j]."""
    YR = []
    for r in range(len(XR)):
        row = []
        for j in range(len(W_RR)):
            acc = 0.0
            for k in range(len(XR[r])):
                acc += W_RR[j][k] * XR[r][k]
            row.append(acc + b_R[j])
        YR.append(row)
    YC = []
    for c in range(len(XC)):
        r = m[c]
        row = []
        for j in range(len(W_CR)):
            acc = 0.0
            for k in range(len(XR[r])):
                acc += W_CR[j][k] * XR[r][k]
            for k in range(len(XC[c])):
                acc += W_CC[j][k] * XC[c][k]
            row.append(acc + b_C[j])
        YC.append(row)
    return YR, YC


def fm_masked(ER, EC, m):
    """[REV] §2.1 FM equation: request group keeps X^R X^R^T only; candidate group gets
    [X^C X^R^T, X^C X^C^T].  ER[r][t][k], EC[c][t][k]."""
    FR = []
    for r in range(len(ER)):
        out = []
        for i in range(len(ER[r])):
            for j in range(len(ER[r])):
                out.append(sum(ER[r][i][k] * ER[r][j][k] for k in range(len(ER[r][i]))))
        FR.append(out)
    FC = []
    for c in range(len(EC)):
        r = m[c]
        out = []
        for i in range(len(EC[c])):
            for j in range(len(ER[r])):
                out.append(sum(EC[c][i][k] * ER[r][j][k] for k in range(len(EC[c][i]))))
            for j in range(len(EC[c])):
                out.append(sum(EC[c][i][k] * EC[c][j][k] for k in range(len(EC[c][i]))))
        FC.append(out)
    return FR, FC


def token_lcb(ER, EC, m, P_RR, P_CR, P_CC):
    """Token-axis masked mixing: L^R_r[o][d] = sum_t P_RR[o][t] ER[r][t][d];
    L^C_c[o][d] = sum_t P_CR[o][t] ER[m_c][t][d] + sum_t P_CC[o][t] EC[c][t][d]."""
    D = len(ER[0][0]) if ER else 0
    LR = [[[sum(P_RR[o][t] * ER[r][t][d] for t in range(len(ER[r]))) for d in range(D)]
           for o in range(len(P_RR))] for r in range(len(ER))]
    LC = []
    for c in range(len(EC)):
        r = m[c]
        LC.append([[sum(P_CR[o][t] * ER[r][t][d] for t in range(len(ER[r]))) +
                    sum(P_CC[o][t] * EC[c][t][d] for t in range(len(EC[c]))) for d in range(D)]
                   for o in range(len(P_CR))])
    return LR, LC


def layernorm_row(x, gamma, beta, eps=1e-5):
    n = len(x)
    mu = 0.0
    for v in x:
        mu += v
    mu /= n
    var = 0.0
    for v in x:
        var += (v - mu) * (v - mu)
    var /= n
    inv = 1.0 / math.sqrt(var + eps)
    return [(x[i] - mu) * inv * gamma[i] + beta[i] for i in range(n)]


def attention_one_query(q, K, V, H):
    """One query vector q [d] against keys/values K, V [L][d], H heads of width d/H:
    out_h = sum_l softmax_l(q_h . k_{l,h} / sqrt(d_h)) v_{l,h}."""
    d = len(q)
    dh = d // H
    out = [0.0] * d
    for h in range(H):
        lo = h * dh
        scores = []
        for l in range(len(K)):
            s = 0.0
            for e in range(dh):
                s += q[lo + e] * K[l][lo + e]
            scores.append(s / math.sqrt(dh))
        mx = max(scores)
        w = [math.exp(s - mx) for s in scores]
        tot = sum(w)
        for e in range(dh):
            acc = 0.0
            for l in range(len(K)):
                acc += w[l] * V[l][lo + e]
            out[lo + e] = acc / tot
    return out


# ---------------------------------------------------------------------------------------------
# Compositions, written per request and per candidate with the loop primitives above, in the
# order the readings fix.  They never form the broadcast: a request's path reads only its own
# rows, a candidate's path reads its request's rows through m.  Used to pin the oracle's
# vectorised compositions (concatenation order, residual and LayerNorm placement, weight names).
# ---------------------------------------------------------------------------------------------
def gelu(v):
    """Exact GELU x * Phi(x) with Phi from math.erf."""
    return 0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0)))


def _act(rows, f):
    return [[f(v) for v in row] for row in rows]


def _tokens(flat, n_tok, D):
    return [flat[t * D:(t + 1) * D] for t in range(n_tok)]


def _rows(M):
    """A numpy-or-list 2-D weight as nested Python lists of floats."""
    return [[float(v) for v in row] for row in M]


def _vec(v):
    return [float(x) for x in v]


def wukong_layer(ER, EC, m, W, pre, g):
    """One ROCSified Wukong layer ([REV] §2.1 Figure 1(d) and Figure 2): the FM block
    (masked FM, flatten, two-group MLP with a GELU hidden layer, reshape to tokens), the token-axis
    LCB without bias, the per-group concatenation [FM-block tokens, LCB tokens], the residual add
    of the layer input and then the group-local LayerNorm over each group's whole slice.
    ER[r][t][k] and EC[c][t][k] are nested lists; returns (ER', EC') in the same form."""
    FR, FC = fm_masked(ER, EC, m)
    l1 = pre + "mlp1."
    hR, hC = linear_two_group(FR, FC, m, _rows(W[l1 + "W_RR"]), _rows(W[l1 + "W_CR"]),
                              _rows(W[l1 + "W_CC"]), _vec(W[l1 + "b_R"]), _vec(W[l1 + "b_C"]))
    hR, hC = _act(hR, gelu), _act(hC, gelu)
    l2 = pre + "mlp2."
    oR, oC = linear_two_group(hR, hC, m, _rows(W[l2 + "W_RR"]), _rows(W[l2 + "W_CR"]),
                              _rows(W[l2 + "W_CC"]), _vec(W[l2 + "b_R"]), _vec(W[l2 + "b_C"]))
    LR, LC = token_lcb(ER, EC, m, _rows(W[pre + "lcb.P_RR"]), _rows(W[pre + "lcb.P_CR"]),
                       _rows(W[pre + "lcb.P_CC"]))

    def finish(o_flat, n_o, L_tok, E, ln):
        cat = _tokens(o_flat, n_o, g.D) + L_tok
        flat = [cat[t][k] + E[t][k] for t in range(len(E)) for k in range(g.D)]
        y = layernorm_row(flat, _vec(W[ln + "gamma"]), _vec(W[ln + "beta"]))
        return _tokens(y, len(E), g.D)

    ER2 = [finish(oR[r], g.fm_out_R, LR[r], ER[r], pre + "lnR.") for r in range(len(ER))]
    EC2 = [finish(oC[c], g.fm_out_C, LC[c], EC[c], pre + "lnC.") for c in range(len(EC))]
    return ER2, EC2


def query_gen(YR, YC, m, W, pre):
    """The DCA query generator ([REV] §2.2, [Q^R; Q^C] = MLP_i(LCB_i(.))): a token-axis LCB
    down to one token per group, then a two-group MLP d -> d (GELU) -> d.  YR[r][t][k],
    YC[c][t][k]; returns (QR[r][k], QC[c][k])."""
    LR, LC = token_lcb(YR, YC, m, _rows(W[pre + "p_RR"]), _rows(W[pre + "p_CR"]), _rows(W[pre + "p_CC"]))
    tR = [LR[r][0] for r in range(len(LR))]
    tC = [LC[c][0] for c in range(len(LC))]
    l1 = pre + "mlp1."
    hR, hC = linear_two_group(tR, tC, m, _rows(W[l1 + "W_RR"]), _rows(W[l1 + "W_CR"]),
                              _rows(W[l1 + "W_CC"]), _vec(W[l1 + "b_R"]), _vec(W[l1 + "b_C"]))
    hR, hC = _act(hR, gelu), _act(hC, gelu)
    l2 = pre + "mlp2."
    return linear_two_group(hR, hC, m, _rows(W[l2 + "W_RR"]), _rows(W[l2 + "W_CR"]),
                            _rows(W[l2 + "W_CC"]), _vec(W[l2 + "b_R"]), _vec(W[l2 + "b_C"]))


def _matvec(Wm, x):
    return [sum(Wm[j][k] * x[k] for k in range(len(x))) for j in range(len(Wm))]


def encoder_layer(S, Wq, Wk, Wv, Wo, gamma, beta, H):
    """One request's encoder layer LN(S + MHSA(S) W_O^T), LayerNorm per event over d; S[t][k]."""
    Wq, Wk, Wv, Wo = _rows(Wq), _rows(Wk), _rows(Wv), _rows(Wo)
    Q = [_matvec(Wq, s) for s in S]
    K = [_matvec(Wk, s) for s in S]
    V = [_matvec(Wv, s) for s in S]
    out = []
    for t in range(len(S)):
        a = _matvec(Wo, attention_one_query(Q[t], K, V, H))
        out.append(layernorm_row([S[t][k] + a[k] for k in range(len(a))], _vec(gamma), _vec(beta)))
    return out


def dca_depths(Hist, m, W, layers, H, token_source):
    """The DCA path of [REV] §2.2 per request and per candidate: the shared encoder
    S_i = Enc_i(S_{i-1}) and its four projections once per request, then at each depth i the
    query generator on the tokens `token_source(i, A_prev)` returns, the request query against
    the request group's K/V and each candidate's query against its request's candidate-group K/V.
    Returns (A_R[i][r][k], A_C[i][c][k])."""
    A_R, A_C = [], []
    S = [[list(map(float, s)) for s in Hr] for Hr in Hist]
    prev = None
    for i in range(layers):
        e = f"enc{i}."
        S = [encoder_layer(Sr, W[e + "Wq"], W[e + "Wk"], W[e + "Wv"], W[e + "Wo"],
                           W[e + "ln.gamma"], W[e + "ln.beta"], H) for Sr in S]
        kv = f"kv{i}."
        proj = {k: [[_matvec(_rows(W[kv + k]), s) for s in Sr] for Sr in S]
                for k in ("WK_R", "WV_R", "WK_C", "WV_C")}
        YR, YC = token_source(i, prev)
        QR, QC = query_gen(YR, YC, m, W, f"qg{i}.")
        aR = [attention_one_query(QR[r], proj["WK_R"][r], proj["WV_R"][r], H) for r in range(len(S))]
        aC = [attention_one_query(QC[c], proj["WK_C"][m[c]], proj["WV_C"][m[c]], H) for c in range(len(QC))]
        A_R.append(aR)
        A_C.append(aC)
        prev = (aR, aC)
    return A_R, A_C


def score_head(xR, xC, m, W):
    """Candidate scoring head: sigmoid(w3 . ReLU(W2 ReLU(W_CR x^R_{m_c} + W_CC x^C_c + b_C) + b2)
    + b3), the first layer a two-group linear with no request output."""
    _, h1 = linear_two_group(xR, xC, m, [], _rows(W["score1.W_CR"]), _rows(W["score1.W_CC"]), [],
                             _vec(W["score1.b_C"]))
    out = []
    for c in range(len(xC)):
        a1 = [max(v, 0.0) for v in h1[c]]
        a2 = [max(v + b, 0.0) for v, b in zip(_matvec(_rows(W["score2.W"]), a1), _vec(W["score2.b"]))]
        z = _matvec(_rows(W["score3.w"]), a2)[0] + float(W["score3.b"][0])
        out.append(1.0 / (1.0 + math.exp(-z)))
    return out
