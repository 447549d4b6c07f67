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
