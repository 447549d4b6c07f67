"""Host-side checks of the C ABI (no GPU): the library loads, exports every entry point that
include/rocs.h declares, the ctypes structs match the C layout, and argument validation fails
before any CUDA work."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rocs.h")


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:rocs_status|const char\*|int32_t)\s+(rocs_\w+)\s*\(", txt, re.M)))


@pytest.fixture(scope="module")
def rocs():
    from request_candidate_sharing_b200 import build
    build.build()
    from request_candidate_sharing_b200 import rocs as R
    return R


def test_header_declares_the_boundary():
    names = _declared()
    for n in ["rocs_linear_ikbo", "rocs_group_layernorm", "rocs_fm_masked", "rocs_dca_encode",
              "rocs_dca_cross_attn", "rocs_forward", "rocs_segments_from_counts", "rocs_token_lcb"]:
        assert n in names


def test_library_exports_every_declared_symbol(rocs):
    lib = ctypes.CDLL(rocs.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(_declared()) == set(rocs.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", rocs.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (rocs_\w+)$", out, re.M))
    assert exported == set(_declared())


def test_struct_layouts_match_c(rocs):
    structs = {"rocs_ikbo_desc": rocs.IkboDesc, "rocs_dca_layer_weights": rocs.DcaLayerWeights,
               "rocs_dca_desc": rocs.DcaDesc, "rocs_glm_linear_weights": rocs.GlmLinearWeights,
               "rocs_glm_layer_weights": rocs.GlmLayerWeights, "rocs_qgen_weights": rocs.QgenWeights,
               "rocs_score_weights": rocs.ScoreWeights, "rocs_model_weights": rocs.ModelWeights,
               "rocs_model_desc": rocs.ModelDesc, "rocs_inputs": rocs.Inputs, "rocs_outputs": rocs.Outputs}
    fields = {"rocs_model_desc": ["B_C", "glm_layers", "dca_layers", "score_h2"],
              "rocs_ikbo_desc": ["B_C", "act"], "rocs_model_weights": ["dca", "qgen", "score"],
              "rocs_outputs": ["score"]}
    src = ["#include <stdio.h>", "#include <stddef.h>", f'#include "{HEADER}"', "int main(void){"]
    for n in structs:
        src.append(f'printf("{n} %zu\\n", sizeof({n}));')
        for f in fields.get(n, []):
            src.append(f'printf("{n}.{f} %zu\\n", offsetof({n}, {f}));')
    src.append("return 0;}")
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        open(c, "w").write("\n".join(src))
        exe = os.path.join(d, "t")
        subprocess.run(["gcc", "-O0", c, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    got = dict(line.split() for line in out.strip().splitlines())
    for n, cls in structs.items():
        assert int(got[n]) == ctypes.sizeof(cls), n
        for f in fields.get(n, []):
            assert int(got[f"{n}.{f}"]) == getattr(cls, f).offset, (n, f)


def test_validation_errors_without_gpu(rocs):
    lib = ctypes.CDLL(rocs.LIB_PATH)
    # NULL handle -> INVALID_ARG, message set, nothing launched
    d = rocs.IkboDesc(4, 256, 128, 64, 128, 128, 0, 0, 0)
    st = rocs._lib_ikbo(None, ctypes.byref(d), *([None] * 11), 0, None)
    assert st == rocs.ROCS_ERR_INVALID_ARG
    assert "handle" in rocs.rocs_last_error()
    # a dummy handle with invalid descriptors never reaches CUDA
    dummy = ctypes.create_string_buffer(64)
    h = ctypes.cast(dummy, ctypes.c_void_p)
    bad = rocs.IkboDesc(0, 256, 128, 64, 128, 128, 0, 0, 0)
    n = ctypes.c_size_t(0)
    assert rocs._lib_ikbo_ws(h, ctypes.byref(bad), ctypes.byref(n)) == rocs.ROCS_ERR_INVALID_ARG
    f32_to_bf16 = rocs.IkboDesc(4, 256, 128, 64, 128, 128, rocs.ROCS_F32, rocs.ROCS_BF16, 0)
    assert rocs._lib_ikbo_ws(h, ctypes.byref(f32_to_bf16), ctypes.byref(n)) == rocs.ROCS_ERR_INVALID_ARG
    good = rocs.IkboDesc(4, 256, 128, 64, 128, 128, rocs.ROCS_BF16, rocs.ROCS_F32, 0)
    assert rocs._lib_ikbo_ws(h, ctypes.byref(good), ctypes.byref(n)) == rocs.ROCS_OK
    assert n.value >= 4 * 128 * 4
    # misaligned dims add padded operand space (alignment fix)
    odd = rocs.IkboDesc(4, 256, 100, 100, 128, 128, rocs.ROCS_BF16, rocs.ROCS_F32, 0)
    n2 = ctypes.c_size_t(0)
    assert rocs._lib_ikbo_ws(h, ctypes.byref(odd), ctypes.byref(n2)) == rocs.ROCS_OK
    assert n2.value > n.value
    # attention limits (long histories are accepted: they stream through shared memory)
    st = rocs._lib_attn(h, 16, 16, 16, 16, 1 << 20, 1, 4096, 1, 64, 0.125, 16, 64, 1, None, None)
    assert st == rocs.ROCS_ERR_INVALID_ARG and "too large" in rocs.rocs_last_error()
    st = rocs._lib_attn(h, 16, 16, 16, 16, 1, 1, 16, 1, 48, 0.125, 16, 64, 1, None, None)
    assert st == rocs.ROCS_ERR_INVALID_ARG
    # FM limits
    st = rocs._lib_fm(h, 16, 16, 16, 1, 1, 60, 16, 128, 16, 16, 1, None)
    assert st == rocs.ROCS_ERR_INVALID_ARG
    # model descriptor checks
    md = rocs.ModelDesc()
    md.B_R, md.B_C = 2, 3
    assert rocs._lib_fwd_ws(h, ctypes.byref(md), ctypes.byref(n)) == rocs.ROCS_ERR_INVALID_ARG   # nothing to run
    md.glm_layers, md.n_R, md.n_C, md.D, md.hidden = 1, 32, 16, 128, 1024
    md.fm_out_R, md.fm_out_C, md.lcb_out_R, md.lcb_out_C = 16, 8, 16, 8
    assert rocs._lib_fwd_ws(h, ctypes.byref(md), ctypes.byref(n)) == rocs.ROCS_OK
    md.lcb_out_C = 7
    assert rocs._lib_fwd_ws(h, ctypes.byref(md), ctypes.byref(n)) == rocs.ROCS_ERR_INVALID_ARG
    assert "residual" in rocs.rocs_last_error()


def test_create_without_gpu_fails_cleanly(rocs):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(rocs.RocsError):
        rocs.Rocs(0)


def _function_body(src: str, signature: str) -> str:
    """The text of the function whose definition starts with `signature`, through its closing
    brace (brace matching; the sources have no braces inside string literals there)."""
    i = src.index(signature)
    j = src.index("{", i)
    depth = 0
    for k in range(j, len(src)):
        depth += {"{": 1, "}": -1}.get(src[k], 0)
        if depth == 0:
            return src[i:k + 1]
    raise AssertionError(f"unbalanced braces after {signature}")


def test_noalloc_path_calls_no_allocation_routine():
    """rocs_linear_ikbo_noalloc and the launchers it calls name no routine that allocates, frees
    or clears device memory (a memset on the shared scratch would also be a hidden dependency)."""
    import re
    csrc = os.path.join(ROOT, "request_candidate_sharing_b200", "csrc")
    read = lambda f: open(os.path.join(csrc, f)).read()
    code = lambda t: re.sub(r"//[^\n]*", "", t)          # comments may name them
    bodies = [code(read("noalloc.cu")),
              code(_function_body(read("misc.cu"), "rocs_status launch_gemm_f32(")),
              code(_function_body(read("gemm_tc.cu"), "rocs_status launch_gemm_bf16("))]
    banned = re.compile(r"\b(cudaMalloc\w*|cudaFree\w*|cudaMemset\w*|cuMemAlloc\w*|cuMemFree\w*|cuMemCreate|"
                        r"cudaMallocAsync|malloc|free|new|delete)\b")
    for b in bodies:
        assert not banned.search(b), banned.search(b).group(0)
    assert "launch_gemm_f32" in bodies[0] and "launch_gemm_bf16" in bodies[0]
