"""ctypes binding of librocs (include/rocs.h).  Argument marshalling only: every step of the
ROCS path runs in the library's CUDA kernels.  Tensors are passed as raw device pointers
(anything with `.data_ptr()`, a plain int, or None for NULL); streams as a cudaStream_t handle
(`torch.cuda.current_stream().cuda_stream`) or None for the default stream.

Importing this module fails loudly if librocs.so has not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librocs.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"librocs.so not built at {LIB_PATH}; run `python -m request_candidate_sharing_b200.build`")
_lib = C.CDLL(LIB_PATH)

# ---- enums ----
ROCS_OK, ROCS_ERR_INVALID_ARG, ROCS_ERR_UNSUPPORTED, ROCS_ERR_CUDA = 0, 1, 2, 3
ROCS_ERR_WORKSPACE, ROCS_ERR_INDEX, ROCS_ERR_DEVICE_TIMEOUT, ROCS_ERR_COUNTS = 4, 5, 6, 7
ROCS_F32, ROCS_BF16 = 0, 1
ACT = {"none": 0, "relu": 1, "gelu": 2, "sigmoid": 3}
MAX_LAYERS = 8

STATUS_NAMES = {0: "ROCS_OK", 1: "ROCS_ERR_INVALID_ARG", 2: "ROCS_ERR_UNSUPPORTED", 3: "ROCS_ERR_CUDA",
                4: "ROCS_ERR_WORKSPACE", 5: "ROCS_ERR_INDEX", 6: "ROCS_ERR_DEVICE_TIMEOUT", 7: "ROCS_ERR_COUNTS"}

P = C.c_void_p
I32 = C.c_int32
I64 = C.c_int64


class RocsError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


# ---- structs (mirror include/rocs.h) ----
class IkboDesc(C.Structure):
    _fields_ = [("B_R", I32), ("B_C", I64), ("d_R_in", I32), ("d_C_in", I32), ("d_R_out", I32),
                ("d_C_out", I32), ("dtype_in", C.c_int), ("dtype_out", C.c_int), ("act", C.c_int)]


class DcaLayerWeights(C.Structure):
    _fields_ = [("Wq", P), ("Wk", P), ("Wv", P), ("Wo", P), ("ln_gamma", P), ("ln_beta", P),
                ("WK_R", P), ("WV_R", P), ("WK_C", P), ("WV_C", P)]


class DcaDesc(C.Structure):
    _fields_ = [("B_R", I32), ("L", I32), ("d", I32), ("H", I32), ("layers", I32)]


class GlmLinearWeights(C.Structure):
    _fields_ = [("W_RR", P), ("W_CR", P), ("W_CC", P), ("b_R", P), ("b_C", P)]


class GlmLayerWeights(C.Structure):
    _fields_ = [("mlp1", GlmLinearWeights), ("mlp2", GlmLinearWeights), ("P_RR", P), ("P_CR", P), ("P_CC", P),
                ("lnR_gamma", P), ("lnR_beta", P), ("lnC_gamma", P), ("lnC_beta", P)]


class QgenWeights(C.Structure):
    _fields_ = [("p_RR", P), ("p_CR", P), ("p_CC", P), ("mlp1", GlmLinearWeights), ("mlp2", GlmLinearWeights)]


class ScoreWeights(C.Structure):
    _fields_ = [("s1", GlmLinearWeights), ("W2", P), ("b2", P), ("w3", P), ("b3", P)]


class ModelWeights(C.Structure):
    _fields_ = [("glm", GlmLayerWeights * MAX_LAYERS), ("dca", DcaLayerWeights * MAX_LAYERS),
                ("qgen", QgenWeights * MAX_LAYERS), ("score", ScoreWeights)]


class ModelDesc(C.Structure):
    _fields_ = [("B_R", I32), ("B_C", I64),
                ("glm_layers", I32), ("n_R", I32), ("n_C", I32), ("D", I32), ("hidden", I32),
                ("fm_out_R", I32), ("fm_out_C", I32), ("lcb_out_R", I32), ("lcb_out_C", I32),
                ("dca_layers", I32), ("L", I32), ("d", I32), ("H", I32), ("q_n_R", I32), ("q_n_C", I32),
                ("q_dim", I32), ("dca_query_source", I32),
                ("score_h1", I32), ("score_h2", I32)]


class Inputs(C.Structure):
    _fields_ = [("counts", P), ("E_R", P), ("E_C", P), ("Hist", P), ("Y_R", P), ("Y_C", P), ("hist_len", P)]


class Outputs(C.Structure):
    _fields_ = [("offsets", P), ("req_idx", P), ("E_R", P), ("E_C", P), ("S", P), ("A_R", P), ("A_C", P),
                ("score", P)]


# ---- prototypes ----
def _proto(name, *args, res=C.c_int):
    f = getattr(_lib, name)
    f.argtypes = list(args)
    f.restype = res
    return f


_lib_create = _proto("rocs_create", C.POINTER(P), C.c_int)
_lib_destroy = _proto("rocs_destroy", P)
_lib_last_error = _proto("rocs_last_error", res=C.c_char_p)
_lib_status = _proto("rocs_get_device_status", P, P, C.POINTER(I32))
_lib_num_sms = _proto("rocs_num_sms", P, res=I32)
_lib_segments = _proto("rocs_segments_from_counts", P, P, I32, P, P, I64, P)
_lib_ikbo_ws = _proto("rocs_linear_ikbo_workspace", P, C.POINTER(IkboDesc), C.POINTER(C.c_size_t))
_lib_ikbo = _proto("rocs_linear_ikbo", P, C.POINTER(IkboDesc), P, P, P, P, P, P, P, P, P, P, P, C.c_size_t, P)
_lib_ln = _proto("rocs_group_layernorm", P, P, I32, P, I32, P, I64, P, P, C.c_float, P, C.c_int, P)
_lib_fm = _proto("rocs_fm_masked", P, P, P, P, I32, I64, I32, I32, I32, P, P, C.c_int, P)
_lib_lcb_ws = _proto("rocs_token_lcb_workspace", P, I32, I32, I32, C.POINTER(C.c_size_t))
_lib_lcb = _proto("rocs_token_lcb", P, P, P, P, I32, I64, I32, I32, I32, P, P, P, I32, I32, P, I64, P, I64, C.c_int,
                  P, C.c_size_t, P)
_lib_attn = _proto("rocs_dca_cross_attn", P, P, P, P, P, I32, I64, I32, I32, I32, C.c_float, P, I64, C.c_int, P, P)
_lib_enc_ws = _proto("rocs_dca_encode_workspace", P, C.POINTER(DcaDesc), C.POINTER(C.c_size_t))
_lib_enc = _proto("rocs_dca_encode", P, C.POINTER(DcaDesc), P, P, C.POINTER(DcaLayerWeights), P, P, P, C.c_size_t, P)
_lib_fwd_ws = _proto("rocs_forward_workspace", P, C.POINTER(ModelDesc), C.POINTER(C.c_size_t))
_lib_fwd = _proto("rocs_forward", P, C.POINTER(ModelDesc), C.POINTER(ModelWeights), C.POINTER(Inputs),
                  C.POINTER(Outputs), P, C.c_size_t, P)

_lib_ikbo_na = _proto("rocs_linear_ikbo_noalloc", P, C.POINTER(IkboDesc), P, P, P, P, P, P, P, P, P, P, P)
_lib_graph = _proto("rocs_set_graph_replay", P, I32)
_lib_fused = _proto("rocs_set_ikbo_fused", P, I32)
_lib_withhold = _proto("rocs_test_withhold_ikbo_flag", P, I32, I64)
_lib_probe = _proto("rocs_probe_exp2_rate", P, I32, C.POINTER(C.c_double), P)
_lib_w8tc = _proto("rocs_set_w8_tensor_cores", P, I32)
_lib_q8 = _proto("rocs_quantize_weights_fp8", P, P, C.c_int, I32, I32, P, P, P)
_lib_w8_ws = _proto("rocs_linear_ikbo_w8_workspace", P, C.POINTER(IkboDesc), C.POINTER(C.c_size_t))
_lib_w8 = _proto("rocs_linear_ikbo_w8", P, C.POINTER(IkboDesc), P, P, P, P, P, P, P, P, P, P, P, P, P, P, C.c_size_t, P)
_lib_sort_ws = _proto("rocs_sort_by_request_workspace", P, I32, I64, C.POINTER(C.c_size_t))
_lib_sort = _proto("rocs_sort_by_request", P, P, I32, I64, P, P, P, C.c_size_t, P)
_lib_xu_ws = _proto("rocs_dca_cross_attn_unsorted_workspace", P, I32, I64, I32, I32, C.c_int, C.POINTER(C.c_size_t))
_lib_xu = _proto("rocs_dca_cross_attn_unsorted", P, P, P, P, P, I32, I64, I32, I32, I32, C.c_float, P, I64, C.c_int, P,
                 P, C.c_size_t, P)
_lib_partition = _proto("rocs_partition_requests", P, I32, I32, C.c_double, C.c_double, P)
_lib_tstart = _proto("rocs_timing_start", P, I32)
_lib_tstop = _proto("rocs_timing_stop", P, C.c_char_p, C.c_size_t)

EXPORTED = ["rocs_linear_ikbo_noalloc", "rocs_timing_start", "rocs_timing_stop", "rocs_create", "rocs_destroy", "rocs_last_error", "rocs_get_device_status", "rocs_num_sms",
            "rocs_segments_from_counts", "rocs_linear_ikbo_workspace", "rocs_linear_ikbo", "rocs_group_layernorm",
            "rocs_fm_masked", "rocs_token_lcb_workspace", "rocs_token_lcb", "rocs_dca_cross_attn",
            "rocs_dca_encode_workspace", "rocs_dca_encode", "rocs_forward_workspace", "rocs_forward",
            "rocs_set_graph_replay", "rocs_set_ikbo_fused", "rocs_test_withhold_ikbo_flag", "rocs_probe_exp2_rate", "rocs_set_w8_tensor_cores", "rocs_sort_by_request_workspace",
            "rocs_sort_by_request", "rocs_dca_cross_attn_unsorted_workspace", "rocs_dca_cross_attn_unsorted",
            "rocs_quantize_weights_fp8", "rocs_linear_ikbo_w8_workspace", "rocs_linear_ikbo_w8",
            "rocs_partition_requests"]


def ptr(x) -> Optional[int]:
    """Device pointer of a tensor-like (data_ptr), an int, or None (NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def partition_requests(counts, n_parts: int, cost_R: float, cost_C: float):
    """rocs_partition_requests on host arrays: the part (0 .. n_parts-1) of each request."""
    import numpy as np
    c = np.ascontiguousarray(counts, dtype=np.int32)
    out = np.empty(len(c), dtype=np.int32)
    _check(_lib_partition(c.ctypes.data, len(c), int(n_parts), float(cost_R), float(cost_C), out.ctypes.data))
    return out


def rocs_last_error() -> str:
    return _lib_last_error().decode("utf-8", "replace")


def _check(st: int):
    if st != ROCS_OK:
        raise RocsError(st, rocs_last_error())


def dtype_code(t) -> int:
    """ROCS_F32 / ROCS_BF16 for a torch dtype or a string."""
    name = str(getattr(t, "dtype", t))
    if "bfloat16" in name or name == "bf16":
        return ROCS_BF16
    if "float32" in name or name == "f32":
        return ROCS_F32
    raise ValueError(f"unsupported dtype {name}")


class Rocs:
    """One librocs handle bound to a CUDA device."""

    def __init__(self, device: int = 0):
        h = P()
        _check(_lib_create(C.byref(h), int(device)))
        self.h = h
        self.device = device

    def close(self):
        if self.h:
            _lib_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- status --
    def rocs_get_device_status(self, stream=None) -> int:
        code = I32(0)
        _check(_lib_status(self.h, stream, C.byref(code)))
        return int(code.value)

    def rocs_num_sms(self) -> int:
        return int(_lib_num_sms(self.h))

    # -- a0 --
    def rocs_segments_from_counts(self, counts, B_R: int, offsets, req_idx, B_C: int, stream=None):
        _check(_lib_segments(self.h, ptr(counts), B_R, ptr(offsets), ptr(req_idx), B_C, stream))

    # -- a1-a3 --
    def rocs_linear_ikbo_workspace(self, desc: IkboDesc) -> int:
        n = C.c_size_t(0)
        _check(_lib_ikbo_ws(self.h, C.byref(desc), C.byref(n)))
        return int(n.value)

    def rocs_linear_ikbo(self, desc: IkboDesc, X_R, X_C, req_idx, W_RR, W_CR, W_CC, b_R, b_C, Y_R, Y_C,
                         workspace, workspace_bytes: int, stream=None):
        _check(_lib_ikbo(self.h, C.byref(desc), ptr(X_R), ptr(X_C), ptr(req_idx), ptr(W_RR), ptr(W_CR), ptr(W_CC),
                         ptr(b_R), ptr(b_C), ptr(Y_R), ptr(Y_C), ptr(workspace), int(workspace_bytes), stream))

    def rocs_linear_ikbo_noalloc(self, desc: IkboDesc, X_R, X_C, req_idx, W_RR, W_CR, W_CC, b_R, b_C, Y_R, Y_C,
                                 stream=None):
        """rocs_linear_ikbo without a workspace: for callers that may not allocate device memory."""
        _check(_lib_ikbo_na(self.h, C.byref(desc), ptr(X_R), ptr(X_C), ptr(req_idx), ptr(W_RR), ptr(W_CR),
                            ptr(W_CC), ptr(b_R), ptr(b_C), ptr(Y_R), ptr(Y_C), stream))

    # -- a6 --
    def rocs_group_layernorm(self, X1, w1, X2, w2, residual, rows, gamma, beta, eps, Y, io, stream=None):
        _check(_lib_ln(self.h, ptr(X1), w1, ptr(X2), w2, ptr(residual), rows, ptr(gamma), ptr(beta), float(eps),
                       ptr(Y), io, stream))

    # -- a4 --
    def rocs_fm_masked(self, E_R, E_C, req_idx, B_R, B_C, n_R, n_C, D, F_R, F_C, out, stream=None):
        _check(_lib_fm(self.h, ptr(E_R), ptr(E_C), ptr(req_idx), B_R, B_C, n_R, n_C, D, ptr(F_R), ptr(F_C), out,
                       stream))

    def rocs_token_lcb_workspace(self, B_R, o_C, D) -> int:
        n = C.c_size_t(0)
        _check(_lib_lcb_ws(self.h, B_R, o_C, D, C.byref(n)))
        return int(n.value)

    def rocs_token_lcb(self, E_R, E_C, req_idx, B_R, B_C, n_R, n_C, D, P_RR, P_CR, P_CC, o_R, o_C, L_R, ld_LR,
                       L_C, ld_LC, out, workspace, workspace_bytes, stream=None):
        _check(_lib_lcb(self.h, ptr(E_R), ptr(E_C), ptr(req_idx), B_R, B_C, n_R, n_C, D, ptr(P_RR), ptr(P_CR),
                        ptr(P_CC), o_R, o_C, ptr(L_R), ld_LR, ptr(L_C), ld_LC, out, ptr(workspace),
                        int(workspace_bytes), stream))

    # -- a9 --
    def rocs_dca_cross_attn(self, Q, K, V, offsets, B_R, rows, L, H, d_h, scale, O, ld_O, out, stream=None,
                            kv_len=None):
        """kv_len: per-request key counts (device int32 [B_R]) for ragged histories, or None."""
        _check(_lib_attn(self.h, ptr(Q), ptr(K), ptr(V), ptr(offsets), B_R, rows, L, H, d_h, float(scale), ptr(O),
                         ld_O, out, ptr(kv_len), stream))

    # -- a7 --
    def rocs_dca_encode_workspace(self, desc: DcaDesc) -> int:
        n = C.c_size_t(0)
        _check(_lib_enc_ws(self.h, C.byref(desc), C.byref(n)))
        return int(n.value)

    def rocs_dca_encode(self, desc: DcaDesc, Hist, layer_weights, S, KV, workspace, workspace_bytes, stream=None,
                        lengths=None):
        """lengths: per-request history lengths (device int32 [B_R]) for ragged histories, or None."""
        arr = (DcaLayerWeights * len(layer_weights))(*layer_weights)
        _check(_lib_enc(self.h, C.byref(desc), ptr(Hist), ptr(lengths), arr, ptr(S), ptr(KV), ptr(workspace),
                        int(workspace_bytes), stream))

    # -- tracing --
    def rocs_timing_start(self, max_launches: int = 4096):
        _check(_lib_tstart(self.h, int(max_launches)))

    def rocs_timing_stop(self) -> Dict[str, tuple]:
        """{"site:kernel": (launches, total_ms)} for the launches since rocs_timing_start."""
        buf = C.create_string_buffer(1 << 20)
        _check(_lib_tstop(self.h, buf, len(buf)))
        out = {}
        for line in buf.value.decode().splitlines():
            name, n, ms = line.rsplit(" ", 2)
            out[name] = (int(n), float(ms))
        return out

    # -- a0-a11 --
    def rocs_forward_workspace(self, model: ModelDesc) -> int:
        n = C.c_size_t(0)
        _check(_lib_fwd_ws(self.h, C.byref(model), C.byref(n)))
        return int(n.value)

    def rocs_forward(self, model: ModelDesc, weights: ModelWeights, inputs: Inputs, outputs: Outputs, workspace,
                     workspace_bytes: int, stream=None):
        _check(_lib_fwd(self.h, C.byref(model), C.byref(weights), C.byref(inputs), C.byref(outputs), ptr(workspace),
                        int(workspace_bytes), stream))

    def rocs_set_graph_replay(self, enable: int):
        _check(_lib_graph(self.h, int(enable)))

    def rocs_set_ikbo_fused(self, enable: int):
        _check(_lib_fused(self.h, int(enable)))

    def rocs_test_withhold_ikbo_flag(self, flag_index: int, wait_budget_cycles: int = 0):
        _check(_lib_withhold(self.h, int(flag_index), int(wait_budget_cycles)))

    def rocs_set_w8_tensor_cores(self, enable: int):
        _check(_lib_w8tc(self.h, int(enable)))

    def rocs_probe_exp2_rate(self, n_poly: int, stream=None) -> float:
        r = C.c_double(0.0)
        _check(_lib_probe(self.h, int(n_poly), C.byref(r), stream))
        return r.value

    # -- FP8-weight (W8A16) IKBO linear --
    def rocs_quantize_weights_fp8(self, W, w_dtype: int, rows: int, cols: int, Q, scale, stream=None):
        _check(_lib_q8(self.h, ptr(W), int(w_dtype), int(rows), int(cols), ptr(Q), ptr(scale), stream))

    def rocs_linear_ikbo_w8_workspace(self, desc: IkboDesc) -> int:
        n = C.c_size_t(0)
        _check(_lib_w8_ws(self.h, C.byref(desc), C.byref(n)))
        return int(n.value)

    def rocs_linear_ikbo_w8(self, desc: IkboDesc, X_R, X_C, req_idx, Q_RR, Q_CR, Q_CC, s_RR, s_CR, s_CC, b_R, b_C,
                            Y_R, Y_C, workspace, workspace_bytes: int, stream=None):
        _check(_lib_w8(self.h, C.byref(desc), ptr(X_R), ptr(X_C), ptr(req_idx), ptr(Q_RR), ptr(Q_CR), ptr(Q_CC),
                       ptr(s_RR), ptr(s_CR), ptr(s_CC), ptr(b_R), ptr(b_C), ptr(Y_R), ptr(Y_C), ptr(workspace),
                       int(workspace_bytes), stream))

    # -- candidates in any order --
    def rocs_sort_by_request_workspace(self, B_R: int, B_C: int) -> int:
        n = C.c_size_t(0)
        _check(_lib_sort_ws(self.h, int(B_R), int(B_C), C.byref(n)))
        return int(n.value)

    def rocs_sort_by_request(self, req_idx, B_R: int, B_C: int, perm, offsets, workspace, workspace_bytes: int,
                             stream=None):
        _check(_lib_sort(self.h, ptr(req_idx), int(B_R), int(B_C), ptr(perm), ptr(offsets), ptr(workspace),
                         int(workspace_bytes), stream))

    def rocs_dca_cross_attn_unsorted_workspace(self, B_R: int, rows: int, H: int, d_h: int, out: int) -> int:
        n = C.c_size_t(0)
        _check(_lib_xu_ws(self.h, int(B_R), int(rows), int(H), int(d_h), int(out), C.byref(n)))
        return int(n.value)

    def rocs_dca_cross_attn_unsorted(self, Q, K, V, req_idx, B_R: int, rows: int, L: int, H: int, d_h: int,
                                     scale: float, O, ld_O: int, out: int, workspace, workspace_bytes: int,
                                     stream=None, kv_len=None):
        _check(_lib_xu(self.h, ptr(Q), ptr(K), ptr(V), ptr(req_idx), int(B_R), int(rows), int(L), int(H), int(d_h),
                       float(scale), ptr(O), int(ld_O), int(out), ptr(kv_len), ptr(workspace), int(workspace_bytes),
                       stream))


# ---- marshalling helpers for the model structs (names follow the synth weight dictionaries) ----
def glm_linear_weights(W: Dict, pre: str) -> GlmLinearWeights:
    g = lambda k: ptr(W.get(pre + k))
    return GlmLinearWeights(g("W_RR"), g("W_CR"), g("W_CC"), g("b_R"), g("b_C"))


def dca_layer_weights(W: Dict, l: int) -> DcaLayerWeights:
    e, k = f"enc{l}.", f"kv{l}."
    return DcaLayerWeights(ptr(W[e + "Wq"]), ptr(W[e + "Wk"]), ptr(W[e + "Wv"]), ptr(W[e + "Wo"]),
                           ptr(W[e + "ln.gamma"]), ptr(W[e + "ln.beta"]), ptr(W[k + "WK_R"]), ptr(W[k + "WV_R"]),
                           ptr(W[k + "WK_C"]), ptr(W[k + "WV_C"]))


def model_weights(W: Dict, glm_layers: int, dca_layers: int, scoring: bool) -> ModelWeights:
    mw = ModelWeights()
    for l in range(glm_layers):
        p = f"glm{l}."
        mw.glm[l] = GlmLayerWeights(glm_linear_weights(W, p + "mlp1."), glm_linear_weights(W, p + "mlp2."),
                                    ptr(W[p + "lcb.P_RR"]), ptr(W[p + "lcb.P_CR"]), ptr(W[p + "lcb.P_CC"]),
                                    ptr(W[p + "lnR.gamma"]), ptr(W[p + "lnR.beta"]), ptr(W[p + "lnC.gamma"]),
                                    ptr(W[p + "lnC.beta"]))
    for l in range(dca_layers):
        mw.dca[l] = dca_layer_weights(W, l)
        q = f"qg{l}."
        mw.qgen[l] = QgenWeights(ptr(W[q + "p_RR"]), ptr(W[q + "p_CR"]), ptr(W[q + "p_CC"]),
                                 glm_linear_weights(W, q + "mlp1."), glm_linear_weights(W, q + "mlp2."))
    if scoring:
        mw.score = ScoreWeights(glm_linear_weights(W, "score1."), ptr(W["score2.W"]), ptr(W["score2.b"]),
                                ptr(W["score3.w"]), ptr(W["score3.b"]))
    return mw


def model_desc(case) -> ModelDesc:
    """Descriptor of a synth.ModelCase."""
    d = ModelDesc()
    d.B_R, d.B_C = case.B_R, case.B_C
    g, a = case.glm, case.dca
    if g is not None:
        d.glm_layers, d.n_R, d.n_C, d.D, d.hidden = g.layers, g.n_R, g.n_C, g.D, g.hidden
        d.fm_out_R, d.fm_out_C, d.lcb_out_R, d.lcb_out_C = g.fm_out_R, g.fm_out_C, g.lcb_out_R, g.lcb_out_C
    if a is not None:
        d.dca_layers, d.L, d.d, d.H = a.layers, a.L, a.d, a.H
        d.q_n_R, d.q_n_C, d.q_dim = a.q_n_R, a.q_n_C, a.q_dim
        d.dca_query_source = 0 if a.source == "own" else 1
    if case.scoring is not None:
        d.score_h1, d.score_h2 = case.scoring
    return d
