"""Float64 CPU oracle of the ROCS forward: the dense early-broadcast model with explicitly
masked weights.

TEST INFRASTRUCTURE ONLY.  Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s
`cpu_baseline` / `--impl reference` legs may import this module.  It shares no code with the
CUDA path (librocs) and imports nothing from it; both sides read the same seeded inputs from
the `synth` module.

Sources (cited by page title and section):
  [REV]  "ROCS：面向请求的大规模推荐计算共享" -- review of arXiv:2607.27744 at liuzhao09.github.io
         §2.1 Generalized Layer Masking (GLM invariant, dependency mask M_ij, masked linear,
         two-group LCB, masked FM, composition closure), §2.2 Deep Cross Attention (shared
         encoder, GLM query generator, grouped cross-attention), §2.3 RRR (amortised cost),
         §2.4 In-Kernel Broadcast Optimization (request map m, Y_i^C = Z_{m_i} + W_CC X_i^C).
  [SUM]  "Meta推出ROCS：推荐系统推理效率提升3倍，零质量损失" -- PaperDaily summary
         (group-local normalisation, two-group form, DCA three steps).

How the oracle evaluates a model (the "dense early-broadcast" model):
  * Every candidate c carries a dense row [x^R_c ; x^C_c] whose request part starts as a
    materialised copy of its request's input, x^R_c = X^R[m_c] (the logical broadcast that
    [REV] §2.4 describes IKBO removing).
  * Every layer applies its FULL weight W~ = M o W with the zero block stored ([REV] §2.1,
    masked linear equation; two-group block matrix), so each candidate's copy of the request
    path is recomputed per candidate exactly as an early-broadcast model would.
  * One extra "probe" row per request, [X^R[r] ; 0], stands for the request evaluated without
    any candidate (f^R in the two-group form of [REV] §2.1 reads x^R only).  A request's
    outputs are read from its probe row; `check_request_copies` asserts that every candidate's
    copy of them agrees (the closure equation of [REV] §2.1).
  * Request-only subgraphs with no candidate input at all (the DCA sequence encoder and its
    K/V projections, [REV] §2.2) are evaluated once per request and then broadcast; the
    closure property makes this the same as evaluating them per candidate.

Readings where the pages are silent (listed with reasons in the design notes): LayerNorm is
biased-variance with eps 1e-5; GELU is the exact erf form; the encoder layer is
LN(S + MHSA(S)) with W_Q, W_K, W_V, W_O and no FFN; cross-attention has no W_Q / W_O and
scale 1/sqrt(d_h); the Wukong layer is E' = GroupLN(concat(MLP(FM(E)), LCB(E)) + E).
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Tuple

import numpy as np
from scipy.special import erf as _erf

F64 = np.float64


# =============================================================================================
# a0: segment bookkeeping -- [REV] §2.4 (request map m: candidate i belongs to request m_i)
# =============================================================================================
def segments(counts: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """offsets[r] = number of candidates of requests 0..r-1; m[c] = r for offsets[r] <= c <
    offsets[r+1].  Candidates are stored grouped by request, requests in ascending order."""
    counts = np.asarray(counts, dtype=np.int64)
    offsets = np.zeros(len(counts) + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    m = np.repeat(np.arange(len(counts), dtype=np.int64), counts)
    return offsets.astype(np.int32), m.astype(np.int32)


def sort_by_request(m: np.ndarray, B_R: int) -> Tuple[np.ndarray, np.ndarray]:
    """Candidates given in any order with their request index m[c] ([REV] §2.4's map), put in
    the grouped layout that `segments` describes: perm[k] is the candidate at grouped position k,
    candidates of one request keep their given order, and offsets[r] is the first position of
    request r.  An index outside [0, B_R) is not a request: such candidates follow every valid
    one, in their given order, and offsets[B_R] counts only the valid ones."""
    m = np.asarray(m, np.int64)
    key = np.where((m >= 0) & (m < B_R), m, B_R)
    perm = np.argsort(key, kind="stable")
    counts = np.bincount(key, minlength=B_R + 1)
    offsets = np.zeros(B_R + 1, np.int64)
    offsets[1:] = np.cumsum(counts[:B_R])
    return perm.astype(np.int32), offsets.astype(np.int32)


# =============================================================================================
# activations
# =============================================================================================
def activation(x: np.ndarray, kind: str) -> np.ndarray:
    if kind == "none":
        return x
    if kind == "relu":
        return np.maximum(x, 0.0)
    if kind == "gelu":   # exact form x * Phi(x) = x/2 * (1 + erf(x / sqrt(2)))
        return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))
    if kind == "sigmoid":
        return 1.0 / (1.0 + np.exp(-x))
    raise ValueError(kind)


# =============================================================================================
# early broadcast: dense rows + one probe row per request
# =============================================================================================
class DenseBatch:
    """Rows 0..n-1 are candidates (request part = copy of their request's input); rows
    n..n+B_R-1 are the per-request probes (candidate part zero)."""

    def __init__(self, m: np.ndarray, B_R: int):
        self.m = np.asarray(m, dtype=np.int64)
        self.n = len(self.m)
        self.B_R = int(B_R)
        self.owner = np.concatenate([self.m, np.arange(self.B_R)])

    def broadcast(self, X_R: np.ndarray) -> np.ndarray:
        """Materialised copy of request rows for every dense row (the logical broadcast)."""
        return np.asarray(X_R, dtype=F64)[self.owner]

    def with_probe(self, X_C: np.ndarray) -> np.ndarray:
        X_C = np.asarray(X_C, dtype=F64)
        return np.concatenate([X_C, np.zeros((self.B_R,) + X_C.shape[1:], F64)], 0)

    def request_out(self, R_rows: np.ndarray) -> np.ndarray:
        return R_rows[self.n:]

    def cand_out(self, C_rows: np.ndarray) -> np.ndarray:
        return C_rows[:self.n]

    def check_request_copies(self, R_rows: np.ndarray, what: str, rtol: float = 0.0) -> None:
        """Closure property ([REV] §2.1): every candidate's copy of the request outputs equals
        the request's own output F^R(X^R).  rtol=0 demands value equality."""
        if self.n == 0 or R_rows.size == 0:
            return
        cand = R_rows[:self.n]
        ref = R_rows[self.n:][self.m]
        if rtol == 0.0:
            ok = np.array_equal(cand, ref)
        else:
            scale = max(1e-300, float(np.max(np.abs(ref))))
            ok = float(np.max(np.abs(cand - ref))) <= rtol * scale
        if not ok:
            raise AssertionError(f"request-side copies disagree across candidates in {what}")


# =============================================================================================
# A2/A3: GLM linear with explicit block-lower-triangular mask -- [REV] §2.1
# =============================================================================================
def masked_weight(W_RR: Optional[np.ndarray], W_CR: np.ndarray, W_CC: np.ndarray) -> np.ndarray:
    """W~ = [[W_RR, 0], [W_CR, W_CC]] as one dense (d_R_out + d_C_out) x (d_R_in + d_C_in)
    matrix with the zero block stored (mask M_ij = 1{j <= i})."""
    d_C_out, d_R_in = W_CR.shape
    d_C_in = W_CC.shape[1]
    d_R_out = 0 if W_RR is None else W_RR.shape[0]
    W = np.zeros((d_R_out + d_C_out, d_R_in + d_C_in), F64)
    if d_R_out:
        W[:d_R_out, :d_R_in] = W_RR
    W[d_R_out:, :d_R_in] = W_CR
    W[d_R_out:, d_R_in:] = W_CC
    return W


def glm_linear_rows(XR: np.ndarray, XC: np.ndarray, W_RR, W_CR, W_CC, b_R, b_C, act: str):
    """Dense rows [x^R ; x^C] -> act(W~ [x^R ; x^C] + [b^R ; b^C]), split back into the
    request slice (d_R_out wide) and the candidate slice (d_C_out wide)."""
    W = masked_weight(W_RR, W_CR, W_CC)
    d_R_out = 0 if W_RR is None else W_RR.shape[0]
    b = np.concatenate([np.zeros(0) if b_R is None else np.asarray(b_R, F64), np.asarray(b_C, F64)])
    X = np.concatenate([np.asarray(XR, F64), np.asarray(XC, F64)], axis=1)
    Y = activation(X @ W.T + b, act)
    return Y[:, :d_R_out], Y[:, d_R_out:]


def glm_linear(X_R, X_C, m, W_RR, W_CR, W_CC, b_R, b_C, act: str = "none"):
    """Two-group GLM linear over a request batch X_R [B_R, d_R_in] and candidate batch
    X_C [n, d_C_in] with request map m [n]: returns (Y_R [B_R, d_R_out], Y_C [n, d_C_out]),
    evaluated as the dense early-broadcast model."""
    db = DenseBatch(m, len(X_R))
    YR, YC = glm_linear_rows(db.broadcast(X_R), db.with_probe(X_C), W_RR, W_CR, W_CC, b_R, b_C, act)
    db.check_request_copies(YR, "glm_linear", rtol=1e-13)
    return db.request_out(YR), db.cand_out(YC)


def glm_linear_decomposed(X_R, X_C, m, W_RR, W_CR, W_CC, b_R, b_C, act: str = "none"):
    """The IKBO reassociation of the same layer ([REV] §2.4, Y_i^C = Z_{m_i} + W_CC X_i^C with
    Z = W_CR X^R computed on the request batch).  Used only to cross-check the dense form."""
    X_R = np.asarray(X_R, F64)
    X_C = np.asarray(X_C, F64)
    Y_R = None if W_RR is None else activation(X_R @ np.asarray(W_RR, F64).T + b_R, act)
    Z = X_R @ np.asarray(W_CR, F64).T + np.asarray(b_C, F64)
    Y_C = activation(Z[np.asarray(m)] + X_C @ np.asarray(W_CC, F64).T, act)
    return Y_R, Y_C


# =============================================================================================
# A4: group-local LayerNorm -- [SUM] (statistics per group, never over the concatenation)
# =============================================================================================
def group_layernorm(X: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float = 1e-5) -> np.ndarray:
    """LayerNorm over the last axis of one group's slice: (x - mean) / sqrt(var + eps) * gamma
    + beta, variance with divisor = width.  Called separately for each group."""
    X = np.asarray(X, F64)
    mu = X.mean(axis=-1, keepdims=True)
    var = ((X - mu) ** 2).mean(axis=-1, keepdims=True)
    return (X - mu) / np.sqrt(var + eps) * np.asarray(gamma, F64) + np.asarray(beta, F64)


# =============================================================================================
# A5: block-masked factorization machine -- [REV] §2.1 (FM equation, Figure 2(c))
# =============================================================================================
def fm_gram_rows(ER: np.ndarray, EC: np.ndarray) -> np.ndarray:
    """Per dense row: stacked tokens T = [E^R ; E^C] ((n_R + n_C) x D), G = T T^T with the
    request-output x candidate-input block set to zero (output group i only reads input groups
    j <= i)."""
    T = np.concatenate([np.asarray(ER, F64), np.asarray(EC, F64)], axis=1)
    G = np.einsum("bik,bjk->bij", T, T)
    n_R = ER.shape[1]
    G[:, :n_R, n_R:] = 0.0
    return G


def fm_masked_rows(ER, EC):
    """(F^R, F^C) flattened row-major: F^R = G[:n_R, :n_R] (n_R x n_R), F^C = G[n_R:, :]
    (n_C x (n_R + n_C), columns ordered [request tokens, candidate tokens])."""
    G = fm_gram_rows(ER, EC)
    n_R = ER.shape[1]
    b = G.shape[0]
    return G[:, :n_R, :n_R].reshape(b, -1), G[:, n_R:, :].reshape(b, -1)


def fm_masked(E_R, E_C, m):
    db = DenseBatch(m, len(E_R))
    FR, FC = fm_masked_rows(db.broadcast(E_R), db.with_probe(E_C))
    db.check_request_copies(FR, "fm_masked")
    return db.request_out(FR), db.cand_out(FC)


# =============================================================================================
# token-axis LCB (Wukong linear compression) as a GLM linear over tokens -- [REV] §2.1
# =============================================================================================
def token_lcb_rows(ER, EC, P_RR, P_CR, P_CC):
    """Mixes tokens with the masked matrix P~ = [[P_RR, 0], [P_CR, P_CC]] (no bias):
    out = P~ [E^R ; E^C], split into request (rows of P_RR) and candidate tokens."""
    P = masked_weight(P_RR, P_CR, P_CC)
    T = np.concatenate([np.asarray(ER, F64), np.asarray(EC, F64)], axis=1)
    out = np.einsum("oi,bid->bod", P, T)
    o_R = 0 if P_RR is None else P_RR.shape[0]
    return out[:, :o_R], out[:, o_R:]


# =============================================================================================
# attention ([REV] §2.2 grouped cross-attention; candidates read a materialised K/V copy)
# =============================================================================================
def mha_rows(Q: np.ndarray, K: np.ndarray, V: np.ndarray, H: int) -> np.ndarray:
    """Q [b, nq, d], K/V [b, L, d]; heads are H contiguous slices of width d/H;
    softmax(q k^T / sqrt(d_h)) v per head, heads concatenated."""
    b, nq, d = Q.shape
    L = K.shape[1]
    dh = d // H
    q = Q.reshape(b, nq, H, dh).transpose(0, 2, 1, 3)
    k = K.reshape(b, L, H, dh).transpose(0, 2, 1, 3)
    v = V.reshape(b, L, H, dh).transpose(0, 2, 1, 3)
    s = np.einsum("bhqe,bhke->bhqk", q, k) / math.sqrt(dh)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    o = np.einsum("bhqk,bhke->bhqe", p, v)
    return o.transpose(0, 2, 1, 3).reshape(b, nq, d)


def cross_attn(Q: np.ndarray, K: np.ndarray, V: np.ndarray, owner: np.ndarray, H: int,
               chunk: int = 64, kv_len: Optional[np.ndarray] = None) -> np.ndarray:
    """Each query row c attends to a materialised copy of K[owner[c]], V[owner[c]]
    (K/V [B_R, L, d], Q [n, d]) -> [n, d].  With kv_len, request r's history is its first
    kv_len[r] rows: its queries attend to those keys only (the rows after them are padding)."""
    Q = np.asarray(Q, F64)
    out = np.empty_like(Q)
    if kv_len is not None:
        owner = np.asarray(owner)
        for r in np.unique(owner):
            idx = np.flatnonzero(owner == r)
            Lr = int(kv_len[r])
            Kr = np.asarray(K[r:r + 1, :Lr], F64)
            Vr = np.asarray(V[r:r + 1, :Lr], F64)
            out[idx] = mha_rows(Q[idx][None], Kr, Vr, H)[0]
        return out
    for s0 in range(0, len(Q), chunk):
        idx = np.asarray(owner[s0:s0 + chunk])
        Kc = np.asarray(K, F64)[idx]          # broadcast copy, [c, L, d]
        Vc = np.asarray(V, F64)[idx]
        out[s0:s0 + chunk] = mha_rows(Q[s0:s0 + chunk, None, :], Kc, Vc, H)[:, 0, :]
    return out


# =============================================================================================
# A8: DCA shared sequence encoder (request-only) -- [REV] §2.2, S_i = Enc_i(S_{i-1})
# =============================================================================================
def encoder_layer(S: np.ndarray, Wq, Wk, Wv, Wo, gamma, beta, H: int,
                  lengths: Optional[np.ndarray] = None) -> np.ndarray:
    """Enc(S) = LN(S + MHSA(S) W_O^T) per request, MHSA with Q = S W_Q^T, K = S W_K^T,
    V = S W_V^T, non-causal, LN per token over d.  With lengths, request r's sequence is its
    first lengths[r] rows; the rows after them are not part of it and come out as NaN."""
    S = np.asarray(S, F64)
    Q = S @ np.asarray(Wq, F64).T
    K = S @ np.asarray(Wk, F64).T
    V = S @ np.asarray(Wv, F64).T
    A = np.full_like(S, np.nan)
    for r in range(S.shape[0]):
        Lr = S.shape[1] if lengths is None else int(lengths[r])
        A[r, :Lr] = mha_rows(Q[r:r + 1, :Lr], K[r:r + 1, :Lr], V[r:r + 1, :Lr], H)[0]
    return group_layernorm(S + A @ np.asarray(Wo, F64).T, gamma, beta)


def dca_encode(Hist: np.ndarray, W: Dict[str, np.ndarray], layers: int, H: int,
               lengths: Optional[np.ndarray] = None):
    """Runs the request-only encoder and the per-depth K/V projections once per request.
    Returns lists S[l] [B_R, L, d] and KV[l] = (K_R, V_R, K_C, V_C) each [B_R, L, d].  With
    lengths (a ragged history), rows past lengths[r] are NaN in every output."""
    S = np.asarray(Hist, F64)
    Ss, KVs = [], []
    for l in range(layers):
        p = f"enc{l}."
        S = encoder_layer(S, W[p + "Wq"], W[p + "Wk"], W[p + "Wv"], W[p + "Wo"],
                          W[p + "ln.gamma"], W[p + "ln.beta"], H, lengths)
        Ss.append(S)
        p = f"kv{l}."
        KVs.append(tuple(S @ np.asarray(W[p + k], F64).T for k in ("WK_R", "WV_R", "WK_C", "WV_C")))
    return Ss, KVs


# =============================================================================================
# A9: DCA GLM query generator -- [REV] §2.2, [Q^R; Q^C] = MLP_i(LCB_i([Y^R; Y^C]))
# =============================================================================================
def query_gen_rows(YR, YC, W: Dict[str, np.ndarray], pre: str):
    """Token-axis LCB to one token per group, then a two-layer GLM-MLP (GELU hidden)."""
    tR, tC = token_lcb_rows(YR, YC, W[pre + "p_RR"], W[pre + "p_CR"], W[pre + "p_CC"])
    tR, tC = tR[:, 0, :], tC[:, 0, :]
    hR, hC = glm_linear_rows(tR, tC, W[pre + "mlp1.W_RR"], W[pre + "mlp1.W_CR"], W[pre + "mlp1.W_CC"],
                             W[pre + "mlp1.b_R"], W[pre + "mlp1.b_C"], "gelu")
    return glm_linear_rows(hR, hC, W[pre + "mlp2.W_RR"], W[pre + "mlp2.W_CR"], W[pre + "mlp2.W_CC"],
                           W[pre + "mlp2.b_R"], W[pre + "mlp2.b_C"], "none")


# =============================================================================================
# A7: Wukong ROCSified layer -- [REV] §2.1 Figure 1(d), Figure 2
# =============================================================================================
def wukong_layer_rows(ER, EC, W: Dict[str, np.ndarray], pre: str, g) -> Tuple[np.ndarray, np.ndarray]:
    """E' = GroupLN(concat(MLP(FM(E)), LCB(E)) + E), every op group-masked."""
    b = ER.shape[0]
    FR, FC = fm_masked_rows(ER, EC)
    hR, hC = glm_linear_rows(FR, FC, W[pre + "mlp1.W_RR"], W[pre + "mlp1.W_CR"], W[pre + "mlp1.W_CC"],
                             W[pre + "mlp1.b_R"], W[pre + "mlp1.b_C"], "gelu")
    oR, oC = glm_linear_rows(hR, hC, W[pre + "mlp2.W_RR"], W[pre + "mlp2.W_CR"], W[pre + "mlp2.W_CC"],
                             W[pre + "mlp2.b_R"], W[pre + "mlp2.b_C"], "none")
    LR, LC = token_lcb_rows(ER, EC, W[pre + "lcb.P_RR"], W[pre + "lcb.P_CR"], W[pre + "lcb.P_CC"])
    catR = np.concatenate([oR.reshape(b, g.fm_out_R, g.D), LR], axis=1)
    catC = np.concatenate([oC.reshape(b, g.fm_out_C, g.D), LC], axis=1)
    nR = group_layernorm((catR + ER).reshape(b, -1), W[pre + "lnR.gamma"], W[pre + "lnR.beta"])
    nC = group_layernorm((catC + EC).reshape(b, -1), W[pre + "lnC.gamma"], W[pre + "lnC.beta"])
    return nR.reshape(ER.shape), nC.reshape(EC.shape)


def glm_stack(E_R, E_C, m, W, g):
    """3-layer (g.layers) GLM stack on the dense batch.  Returns per-layer (E_R, E_C) pairs
    (request outputs from the probes, candidate outputs from candidate rows), with layer 0 the
    inputs, plus the final dense rows."""
    db = DenseBatch(m, len(E_R))
    ER = db.broadcast(E_R)
    EC = db.with_probe(E_C)
    outs = [(np.asarray(E_R, F64), np.asarray(E_C, F64))]
    rows = [(ER, EC)]
    for l in range(g.layers):
        ER, EC = wukong_layer_rows(ER, EC, W, f"glm{l}.", g)
        db.check_request_copies(ER, f"glm layer {l}", rtol=1e-12)
        outs.append((db.request_out(ER), db.cand_out(EC)))
        rows.append((ER, EC))
    return outs, rows, db


# =============================================================================================
# model forwards
# =============================================================================================
def forward_cfg3(case, inputs, W, m):
    """GLM stack only.  Returns {"E_R": [B_R, n_R, D], "E_C": [n, n_C, D]} after the last layer
    and the per-layer list under "layers"."""
    outs, _, _ = glm_stack(inputs["E_R"], inputs["E_C"], m, W, case.glm)
    return {"E_R": outs[-1][0], "E_C": outs[-1][1], "layers": outs}


def _dca_depths(case, inputs, W, db: DenseBatch, query_rows, Ss, KVs):
    """Query generator + grouped cross-attention at every depth ([REV] §2.2).  `query_rows(l)`
    returns the dense (Y^R, Y^C) token rows the depth-l query generator reads; for the "own"
    wiring the attention outputs are appended as one token per group."""
    a = case.dca
    A_R, A_C = [], []
    appended = None
    for l in range(a.layers):
        YR, YC = query_rows(l, appended)
        QR, QC = query_gen_rows(YR, YC, W, f"qg{l}.")
        db.check_request_copies(QR, f"query generator {l}", rtol=1e-12)
        K_R, V_R, K_C, V_C = KVs[l]
        lengths = inputs.get("hist_len")                  # a ragged history, or None
        aR = cross_attn(QR, K_R, V_R, db.owner, a.H, kv_len=lengths)      # request queries, request K/V
        aC = cross_attn(QC, K_C, V_C, db.owner, a.H, kv_len=lengths)      # candidate queries, shared K/V
        db.check_request_copies(aR, f"request cross-attention {l}", rtol=1e-12)
        A_R.append(aR)
        A_C.append(aC)
        appended = (aR, aC)
    return A_R, A_C


def forward_cfg4(case, inputs, W, m):
    """DCA sequence path with its own query embeddings.  Returns S[l], A_R[l] [B_R, d],
    A_C[l] [n, d]."""
    a = case.dca
    db = DenseBatch(m, len(inputs["H"]))
    Ss, KVs = dca_encode(inputs["H"], W, a.layers, a.H, inputs.get("hist_len"))
    state = {"YR": db.broadcast(inputs["Y_R"]), "YC": db.with_probe(inputs["Y_C"])}

    def query_rows(l, appended):
        if appended is not None:
            aR, aC = appended
            state["YR"] = np.concatenate([state["YR"], aR[:, None, :]], axis=1)
            state["YC"] = np.concatenate([state["YC"], aC[:, None, :]], axis=1)
        return state["YR"], state["YC"]

    A_R, A_C = _dca_depths(case, inputs, W, db, query_rows, Ss, KVs)
    return {"S": Ss, "KV": KVs, "A_R": [db.request_out(x) for x in A_R], "A_C": [db.cand_out(x) for x in A_C]}


def forward_cfg5(case, inputs, W, m):
    """End-to-end ranking forward: GLM stack, DCA with queries from GLM layer l-1 outputs, and
    the candidate scoring MLP [Y^R_m, A^R_m | Y^C, A^C] -> 512 -> 256 -> 1 (sigmoid)."""
    g, a = case.glm, case.dca
    outs, rows, db = glm_stack(inputs["E_R"], inputs["E_C"], m, W, g)
    Ss, KVs = dca_encode(inputs["H"], W, a.layers, a.H, inputs.get("hist_len"))

    def query_rows(l, appended):
        return rows[l]

    A_R, A_C = _dca_depths(case, inputs, W, db, query_rows, Ss, KVs)
    ER, EC = rows[-1]
    b = ER.shape[0]
    xR = np.concatenate([ER.reshape(b, -1)] + A_R, axis=1)
    xC = np.concatenate([EC.reshape(b, -1)] + A_C, axis=1)
    _, h1 = glm_linear_rows(xR, xC, None, W["score1.W_CR"], W["score1.W_CC"], None, W["score1.b_C"], "relu")
    h2 = activation(h1 @ np.asarray(W["score2.W"], F64).T + W["score2.b"], "relu")
    s = activation(h2 @ np.asarray(W["score3.w"], F64).T + W["score3.b"], "sigmoid")[:, 0]
    return {"score": db.cand_out(s), "E_R": outs[-1][0], "E_C": outs[-1][1],
            "A_R": [db.request_out(x) for x in A_R], "A_C": [db.cand_out(x) for x in A_C],
            "S": Ss}


def amortised_cost(C_C: float, C_R: float, N: float) -> float:
    """Per-candidate cost with the request side paid once per request ([REV] §2.3):
    C_amort(N) = C_C + C_R / N."""
    return C_C + C_R / N
