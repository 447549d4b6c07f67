"""Seeded synthetic inputs for the ROCS forward (shared by the CUDA path's tests/bench and
by the float64 oracle).

This module draws random numbers and rounds them to the storage precision; it holds none of
the method's arithmetic (no offsets, no request map, no layer math).  Every named tensor has
its own independent stream, so the order in which tensors are drawn does not matter, and the
first axis of a tensor is split into blocks of ``ROW_BLOCK`` rows that each have their own
stream too, so a sampled subset of rows can be regenerated without drawing the whole tensor.

Workload shapes follow the ROCS pages (liuzhao09 review, §2.1-§2.4; longzhangge summary):
hundreds of candidates per request, user histories of hundreds of events.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

ROW_BLOCK = 1024


# ---------------------------------------------------------------------------------------------
# streams and draws
# ---------------------------------------------------------------------------------------------
def _tensor_id(name: str) -> int:
    return zlib.crc32(name.encode("utf-8")) & 0x7FFFFFFF


def stream(seed: int, name: str, block: int = 0) -> np.random.Generator:
    """Independent generator for (seed, tensor name, row block)."""
    return np.random.default_rng(np.random.SeedSequence([int(seed), _tensor_id(name), int(block)]))


def _block(seed, name, shape, kind, a, b, bi) -> np.ndarray:
    """Row block `bi` (rows bi*ROW_BLOCK ... up to ROW_BLOCK of them) of a drawn tensor."""
    n0, inner = shape[0], shape[1:]
    per_row = int(np.prod(inner)) if inner else 1
    r0 = bi * ROW_BLOCK
    nr = min(ROW_BLOCK, n0 - r0)
    g = stream(seed, name, bi)
    if kind == "normal":
        v = g.standard_normal(nr * per_row, dtype=np.float64) * a
    else:
        v = g.uniform(a, b, nr * per_row)
    return v.astype(np.float32).reshape((nr,) + inner)


def _draw(seed, name, shape, kind, a, b, rows=None) -> np.ndarray:
    shape = tuple(int(s) for s in shape)
    n0 = shape[0]
    inner = shape[1:]
    nblocks = (n0 + ROW_BLOCK - 1) // ROW_BLOCK
    if rows is None:
        out = np.empty(shape, dtype=np.float32)
        for bi in range(nblocks):
            r0 = bi * ROW_BLOCK
            out[r0:r0 + ROW_BLOCK] = _block(seed, name, shape, kind, a, b, bi)
        return out
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows),) + inner, dtype=np.float32)
    cache = {}
    for i, r in enumerate(rows):
        bi = int(r) // ROW_BLOCK
        if bi not in cache:
            cache[bi] = _block(seed, name, shape, kind, a, b, bi)
        out[i] = cache[bi][int(r) - bi * ROW_BLOCK]
    return out


def normal_blocks(seed: int, name: str, shape: Sequence[int], std: float = 1.0):
    """Yields (first_row, rows) over the row blocks of `normal(seed, name, shape, std)`, in order,
    so a tensor too large to hold twice on the host can be filled block by block."""
    shape = tuple(int(s) for s in shape)
    for bi in range((shape[0] + ROW_BLOCK - 1) // ROW_BLOCK):
        yield bi * ROW_BLOCK, _block(seed, name, shape, "normal", float(std), None, bi)


def normal(seed: int, name: str, shape: Sequence[int], std: float = 1.0, rows=None) -> np.ndarray:
    """float32 draws of N(0, std^2); `rows` selects a subset of the first axis."""
    return _draw(seed, name, shape, "normal", float(std), None, rows)


def uniform(seed: int, name: str, shape: Sequence[int], lo: float, hi: float, rows=None) -> np.ndarray:
    return _draw(seed, name, shape, "uniform", float(lo), float(hi), rows)


def small_ints(seed: int, name: str, shape: Sequence[int], bound: int) -> np.ndarray:
    """Integers in [-bound, bound] stored as float32 (exact in bf16 for bound <= 256)."""
    g = stream(seed, name, 0)
    return g.integers(-bound, bound + 1, size=tuple(shape)).astype(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even) and return the raw bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    r = (u + np.uint32(0x7FFF) + lsb) >> 16
    nan = np.isnan(a)
    r = r.astype(np.uint16)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Float32 values exactly representable in bfloat16 (round to nearest even)."""
    return (bf16_bits(a).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------------------------
# candidate counts per request (the oracle and the CUDA path derive offsets / request map)
# ---------------------------------------------------------------------------------------------
def counts_fixed(B_R: int, N: int) -> np.ndarray:
    return np.full(B_R, N, dtype=np.int32)


def counts_uniform(seed: int, B_R: int, lo: int, hi: int) -> np.ndarray:
    """Integers drawn uniformly from [lo, hi] inclusive."""
    return stream(seed, "counts", 0).integers(lo, hi + 1, size=B_R).astype(np.int32)


def hist_lengths(seed: int, B_R: int, L: int, lo: int = 1) -> np.ndarray:
    """Ragged history lengths: request r keeps its first lengths[r] of the L rows, uniform on
    [lo, L] (both ends included), with the first request at L and the second at lo when there are
    two or more, so both extremes always occur."""
    g = stream(seed, "hist_len")
    out = g.integers(lo, L + 1, size=B_R).astype(np.int32)
    if B_R >= 2:
        out[0], out[1] = L, lo
    return out


def counts_lognormal(seed: int, B_R: int, median: float, sigma: float, lo: int, hi: int) -> np.ndarray:
    """round(exp(N(ln median, sigma^2))) clipped to [lo, hi]; rounding is floor(x + 0.5)."""
    z = stream(seed, "counts", 0).standard_normal(B_R)
    x = np.exp(np.log(median) + sigma * z)
    return np.clip(np.floor(x + 0.5), lo, hi).astype(np.int32)


# ---------------------------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------------------------
@dataclasses.dataclass
class LinearCase:
    """One 2-group GLM linear layer: Y^R = W_RR X^R + b^R, Y^C = W_CR X^R[m] + W_CC X^C + b^C."""
    name: str
    counts: np.ndarray
    d_R_in: int
    d_C_in: int
    d_R_out: int
    d_C_out: int
    act: str            # "none" | "relu" | "gelu" | "sigmoid"
    bf16: bool
    seed: int

    @property
    def B_R(self):
        return int(len(self.counts))

    @property
    def B_C(self):
        return int(self.counts.sum())


def linear_cfg1() -> LinearCase:
    """Single 2-group linear, fp32: 4 requests x 64 candidates, X^R[4,128], X^C[256,64], out 128."""
    return LinearCase("cfg1", counts_fixed(4, 64), 128, 64, 128, 128, "none", False, 0)


CFG2_N = (64, 256, 1024)
CFG2_D = (512, 1024, 4096)


def linear_cfg2(N: int, d: int, B_R: int = 256) -> LinearCase:
    """IKBO sweep point, bf16 inputs/weights, fp32 accumulate, ReLU on both outputs."""
    return LinearCase(f"cfg2_N{N}_d{d}", counts_fixed(B_R, N), d, d, d, d, "relu", True, 0)


def linear_inputs(case: LinearCase, cand_rows=None, integer: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Inputs of a linear case.  X ~ N(0,1), weights ~ N(0, 1/fan_in) (fan_in = that block's
    input width), biases ~ U(-0.1, 0.1) in fp32.  bf16 cases round X and W once to bf16.
    `cand_rows` draws only those candidate rows of X^C.  `integer=b` draws small integers in
    [-b, b] (biases zero) so that every summation order is exact."""
    s = case.seed
    B_R, B_C = case.B_R, case.B_C
    if integer is not None:
        out = dict(
            X_R=small_ints(s, "X_R", (B_R, case.d_R_in), integer),
            X_C=small_ints(s, "X_C", (B_C, case.d_C_in), integer),
            W_RR=small_ints(s, "W_RR", (case.d_R_out, case.d_R_in), integer),
            W_CR=small_ints(s, "W_CR", (case.d_C_out, case.d_R_in), integer),
            W_CC=small_ints(s, "W_CC", (case.d_C_out, case.d_C_in), integer),
            b_R=np.zeros(case.d_R_out, np.float32),
            b_C=np.zeros(case.d_C_out, np.float32),
        )
        if cand_rows is not None:
            out["X_C"] = out["X_C"][np.asarray(cand_rows)]
        return out
    out = dict(
        X_R=normal(s, "X_R", (B_R, case.d_R_in)),
        X_C=normal(s, "X_C", (B_C, case.d_C_in), rows=cand_rows),
        W_RR=normal(s, "W_RR", (case.d_R_out, case.d_R_in), (1.0 / case.d_R_in) ** 0.5),
        W_CR=normal(s, "W_CR", (case.d_C_out, case.d_R_in), (1.0 / case.d_R_in) ** 0.5),
        W_CC=normal(s, "W_CC", (case.d_C_out, case.d_C_in), (1.0 / case.d_C_in) ** 0.5),
        b_R=uniform(s, "b_R", (case.d_R_out,), -0.1, 0.1),
        b_C=uniform(s, "b_C", (case.d_C_out,), -0.1, 0.1),
    )
    if case.bf16:
        for k in ("X_R", "X_C", "W_RR", "W_CR", "W_CC"):
            out[k] = bf16_round(out[k])
    return out


# ---------------------------------------------------------------------------------------------
# model workloads (GLM stack, DCA, end-to-end)
# ---------------------------------------------------------------------------------------------
@dataclasses.dataclass
class GLMShape:
    n_R: int = 32          # request embeddings (tokens) per request
    n_C: int = 16          # candidate embeddings per candidate
    D: int = 128           # embedding width
    hidden: int = 1024     # GLM-MLP hidden width (both groups)
    fm_out_R: int = 16     # tokens produced by the FM block's MLP, request group
    fm_out_C: int = 8
    lcb_out_R: int = 16    # tokens produced by the token-axis LCB
    lcb_out_C: int = 8
    layers: int = 3

    @property
    def fm_in_R(self):
        return self.n_R * self.n_R

    @property
    def fm_in_C(self):
        return self.n_C * (self.n_R + self.n_C)


@dataclasses.dataclass
class DCAShape:
    L: int = 200           # history length
    d: int = 256
    H: int = 4
    layers: int = 2        # encoder layers = cross-attention depths
    q_n_R: int = 16        # query-generator request embeddings (cfg4 only)
    q_n_C: int = 8
    q_dim: int = 256       # width of the query-generator embeddings
    source: str = "own"    # "own": DCA's own embeddings + appended A tokens; "glm": GLM layer outputs


@dataclasses.dataclass
class ModelCase:
    name: str
    counts: np.ndarray
    seed: int
    glm: Optional[GLMShape]
    dca: Optional[DCAShape]
    scoring: Optional[Tuple[int, int]]   # hidden widths of the scoring MLP (512, 256) -> 1

    @property
    def B_R(self):
        return int(len(self.counts))

    @property
    def B_C(self):
        return int(self.counts.sum())


def model_cfg3(B_R: int = 64, seed: int = 0, counts=None) -> ModelCase:
    """Wukong-style GLM stack, 3 layers; 32 request / 16 candidate embeddings of dim 128;
    ragged candidate counts U[100, 1000] per request."""
    c = counts_uniform(seed, B_R, 100, 1000) if counts is None else np.asarray(counts, np.int32)
    return ModelCase("cfg3", c, seed, GLMShape(), None, None)


def model_cfg4(B_R: int = 32, N: int = 500, seed: int = 0, counts=None) -> ModelCase:
    """DCA path: L=200, d=256, 4 heads, 2 encoder layers; 16 request + 8 candidate query
    embeddings of dim 256; 32 requests x 500 candidates."""
    c = counts_fixed(B_R, N) if counts is None else np.asarray(counts, np.int32)
    return ModelCase("cfg4", c, seed, None, DCAShape(L=200, d=256, H=4, layers=2), None)


def model_cfg5(B_R: int = 512, seed: int = 1, counts=None, L: int = 1024) -> ModelCase:
    """End-to-end ranking forward: GLM stack + DCA (L=1024, d=256, 8 heads, 3 depths, queries
    from GLM layer outputs) + candidate scoring MLP 512-256-1; lognormal counts (median 300,
    range 16-2000)."""
    c = counts_lognormal(seed, B_R, 300.0, 1.0, 16, 2000) if counts is None else np.asarray(counts, np.int32)
    return ModelCase("cfg5", c, seed, GLMShape(),
                     DCAShape(L=L, d=256, H=8, layers=3, q_n_R=32, q_n_C=16, q_dim=128, source="glm"),
                     (512, 256))


def _w(seed, name, out_dim, in_dim):
    return bf16_round(normal(seed, name, (out_dim, in_dim), (1.0 / in_dim) ** 0.5))


def _b(seed, name, n):
    return uniform(seed, name, (n,), -0.1, 0.1)


def _glm_linear_params(seed, pre, d_R_in, d_C_in, d_R_out, d_C_out):
    p = {}
    if d_R_out > 0:
        p[pre + "W_RR"] = _w(seed, pre + "W_RR", d_R_out, d_R_in)
        p[pre + "b_R"] = _b(seed, pre + "b_R", d_R_out)
    p[pre + "W_CR"] = _w(seed, pre + "W_CR", d_C_out, d_R_in)
    p[pre + "W_CC"] = _w(seed, pre + "W_CC", d_C_out, d_C_in)
    p[pre + "b_C"] = _b(seed, pre + "b_C", d_C_out)
    return p


def _ln_params(seed, pre, n):
    return {pre + "gamma": (1.0 + uniform(seed, pre + "gamma", (n,), -0.1, 0.1)).astype(np.float32),
            pre + "beta": uniform(seed, pre + "beta", (n,), -0.1, 0.1)}


def model_weights(case: ModelCase) -> Dict[str, np.ndarray]:
    """All weights of a model case.  Linear weights [out, in] ~ N(0, 1/fan_in) rounded to bf16;
    biases and LayerNorm shift ~ U(-0.1, 0.1), LayerNorm gain 1 + U(-0.1, 0.1), fp32."""
    s = case.seed
    W: Dict[str, np.ndarray] = {}
    g = case.glm
    if g is not None:
        for l in range(g.layers):
            pre = f"glm{l}."
            W.update(_glm_linear_params(s, pre + "mlp1.", g.fm_in_R, g.fm_in_C, g.hidden, g.hidden))
            W.update(_glm_linear_params(s, pre + "mlp2.", g.hidden, g.hidden,
                                        g.fm_out_R * g.D, g.fm_out_C * g.D))
            W[pre + "lcb.P_RR"] = _w(s, pre + "lcb.P_RR", g.lcb_out_R, g.n_R)
            W[pre + "lcb.P_CR"] = _w(s, pre + "lcb.P_CR", g.lcb_out_C, g.n_R)
            W[pre + "lcb.P_CC"] = _w(s, pre + "lcb.P_CC", g.lcb_out_C, g.n_C)
            W.update(_ln_params(s, pre + "lnR.", g.n_R * g.D))
            W.update(_ln_params(s, pre + "lnC.", g.n_C * g.D))
    a = case.dca
    if a is not None:
        d = a.d
        for l in range(a.layers):
            pre = f"enc{l}."
            for k in ("Wq", "Wk", "Wv", "Wo"):
                W[pre + k] = _w(s, pre + k, d, d)
            W.update(_ln_params(s, pre + "ln.", d))
            pre = f"kv{l}."
            for k in ("WK_R", "WV_R", "WK_C", "WV_C"):
                W[pre + k] = _w(s, pre + k, d, d)
            pre = f"qg{l}."
            if a.source == "own":
                nr, nc, qd = a.q_n_R + l, a.q_n_C + l, a.q_dim
            else:
                nr, nc, qd = a.q_n_R, a.q_n_C, a.q_dim
            W[pre + "p_RR"] = _w(s, pre + "p_RR", 1, nr)
            W[pre + "p_CR"] = _w(s, pre + "p_CR", 1, nr)
            W[pre + "p_CC"] = _w(s, pre + "p_CC", 1, nc)
            W.update(_glm_linear_params(s, pre + "mlp1.", qd, qd, d, d))
            W.update(_glm_linear_params(s, pre + "mlp2.", d, d, d, d))
    if case.scoring is not None:
        h1, h2 = case.scoring
        dR = g.n_R * g.D + a.layers * a.d
        dC = g.n_C * g.D + a.layers * a.d
        W.update(_glm_linear_params(s, "score1.", dR, dC, 0, h1))
        W["score2.W"] = _w(s, "score2.W", h2, h1)
        W["score2.b"] = _b(s, "score2.b", h2)
        W["score3.w"] = _w(s, "score3.w", 1, h2)
        W["score3.b"] = _b(s, "score3.b", 1)
    return W


def model_inputs(case: ModelCase, cand_rows=None, req_rows=None) -> Dict[str, np.ndarray]:
    """Inputs ~ N(0,1) rounded to bf16.  E_R [B_R, n_R, D], E_C [B_C, n_C, D] (GLM);
    H [B_R, L, d] history, Y_R [B_R, q_n_R, q_dim], Y_C [B_C, q_n_C, q_dim] (DCA, own queries).
    `cand_rows` / `req_rows` draw subsets of the candidate / request axis."""
    s = case.seed
    out = {}
    g = case.glm
    if g is not None:
        out["E_R"] = bf16_round(normal(s, "E_R", (case.B_R, g.n_R, g.D), rows=req_rows))
        out["E_C"] = bf16_round(normal(s, "E_C", (case.B_C, g.n_C, g.D), rows=cand_rows))
    a = case.dca
    if a is not None:
        out["H"] = bf16_round(normal(s, "H", (case.B_R, a.L, a.d), rows=req_rows))
        if a.source == "own":
            out["Y_R"] = bf16_round(normal(s, "Y_R", (case.B_R, a.q_n_R, a.q_dim), rows=req_rows))
            out["Y_C"] = bf16_round(normal(s, "Y_C", (case.B_C, a.q_n_C, a.q_dim), rows=cand_rows))
    return out
