"""Float64 CPU oracle of FP8-weight (W8A16) linears.

TEST INFRASTRUCTURE ONLY.  Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s oracle legs may
import this module.  It shares no code with the CUDA path (librocs) and imports nothing from it.

Source:
  [UGS]  "Compute Only Once: UG-Separation for Efficient Large Recommendation Models" -- review of
         arXiv:2602.10455 at xllm-io.github.io: §三 (technical architecture, Stage 4: W8A16
         quantization: 8-bit FP8 weights, BF16 activations, dequantisation cost negligible) and
         the W8A16 configuration table of §六 (weight precision FP8, activation precision BF16).

The pages fix the weight format (8-bit floating point) and the activation format (bf16) but not
the scaling or the rounding.  Readings taken here (and listed with the design notes):
  * FP8 means E4M3 in its "finite" form: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
    no infinities, the all-ones pattern is NaN, the largest finite magnitude is 1.75 * 2^8 = 448,
    subnormals 0.mmm * 2^-6 down to 2^-9.
  * One scale per output channel (weight row o): s_o = max_i |w_oi| / 448 computed in float32
    (s_o = 1 for an all-zero row), and q_oi = E4M3(w_oi / s_o) with the division in float32,
    rounded to nearest (ties to even) and saturated to +-448.
  * The effective weight is q_oi * s_o; a W8A16 linear is y = act(x W_eff^T + b) with the scale
    applied to the accumulated dot product, y_o = act(s_o * sum_i q_oi x_i + b_o).
"""
import math
from typing import Tuple

import numpy as np

F64 = np.float64
E4M3_MAX = 448.0


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Values of E4M3 nearest to x (ties to even), saturated to +-448 (NaN stays NaN).  The
    spacing in binade [2^e, 2^(e+1)) is 2^(e-3) for e >= -6; below 2^-6 (subnormals) it is 2^-9."""
    x = np.asarray(x, F64)
    a = np.abs(x)
    out = np.zeros_like(a)
    nz = (a > 0) & np.isfinite(a)
    e = np.floor(np.log2(np.where(nz, a, 1.0)))
    e = np.maximum(e, -6.0)                      # subnormal range shares the 2^-6 binade's spacing
    q = np.exp2(e - 3.0)
    r = np.rint(np.where(nz, a, 0.0) / q) * q    # a / q is exact (q a power of two); rint: ties to even
    r = np.minimum(r, E4M3_MAX)                  # saturation
    out = np.where(nz, r, 0.0)
    out = np.where(np.isinf(a), E4M3_MAX, out)
    out = np.copysign(out, x)
    return np.where(np.isnan(x), np.nan, out)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Bit patterns (uint8) of E4M3 values v (each exactly representable, |v| <= 448)."""
    v = np.asarray(v, F64)
    a = np.abs(v)
    sign = (np.signbit(v)).astype(np.uint8) << 7
    bits = np.zeros(a.shape, np.uint8)
    normal = a >= 2.0 ** -6
    e = np.floor(np.log2(np.where(normal, a, 1.0)))
    m_norm = np.rint((np.where(normal, a, 1.0) / np.exp2(e) - 1.0) * 8.0)
    bits = np.where(normal, ((e + 7).astype(np.int64) << 3) | m_norm.astype(np.int64), bits)
    m_sub = np.rint(a / 2.0 ** -9)
    bits = np.where(~normal, m_sub.astype(np.int64), bits)
    out = (bits.astype(np.uint8) | sign).astype(np.uint8)
    return np.where(np.isnan(v), np.uint8(0x7F), out).astype(np.uint8)


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    """Values of E4M3 bit patterns (uint8)."""
    b = np.asarray(b, np.uint8).astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    E = (b >> 3) & 0xF
    M = b & 0x7
    val = np.where(E == 0, M / 8.0 * 2.0 ** -6, (1.0 + M / 8.0) * np.exp2(E - 7.0))
    val = np.where((E == 15) & (M == 7), np.nan, val)
    return s * val


def quantize_rows(W: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-output-channel E4M3 quantisation of W [out, in] (float32 arithmetic for the scale and
    the division, as the readings above fix).  Returns (bytes [out, in] uint8, scales [out] f32)."""
    W = np.asarray(W, np.float32)
    amax = np.max(np.abs(W), axis=1) if W.shape[1] else np.zeros(W.shape[0], np.float32)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    ratio = (W / s[:, None]).astype(np.float32)           # IEEE float32 division
    q = e4m3_round(ratio.astype(F64))
    return e4m3_encode(q), s


def dequantize_rows(Q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Effective weights q_oi * s_o in float64."""
    return e4m3_decode(Q) * np.asarray(s, F64)[:, None]


def w8_linear(X: np.ndarray, Q: np.ndarray, s: np.ndarray, b, act: str = "none") -> np.ndarray:
    """y_o = act(s_o * sum_i q_oi x_i + b_o) for every row x of X (float64)."""
    from oracle.rocs_oracle import activation
    acc = np.asarray(X, F64) @ e4m3_decode(Q).T
    y = acc * np.asarray(s, F64)[None, :]
    if b is not None:
        y = y + np.asarray(b, F64)[None, :]
    return activation(y, act)


def w8_glm_linear(X_R, X_C, m, Q_RR, s_RR, Q_CR, s_CR, Q_CC, s_CC, b_R, b_C, act: str = "none"):
    """The two-group GLM linear of the ROCS pages with FP8 weights: Y^R = act(W_RR x^R + b^R) and
    Y^C = act(W_CR x^R_{m_c} + W_CC x^C_c + b^C), each W the effective q * s weight, evaluated per
    candidate on its request's copy of x^R (the early-broadcast form)."""
    X_R = np.asarray(X_R, F64)
    X_C = np.asarray(X_C, F64)
    m = np.asarray(m, np.int64)
    YR = w8_linear(X_R, Q_RR, s_RR, b_R, act) if Q_RR is not None else None
    pre = (X_R[m] @ dequantize_rows(Q_CR, s_CR).T) + (X_C @ dequantize_rows(Q_CC, s_CC).T)
    from oracle.rocs_oracle import activation
    YC = activation(pre + np.asarray(b_C, F64)[None, :], act)
    return YR, YC
