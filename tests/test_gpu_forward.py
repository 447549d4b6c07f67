"""GPU parity of the whole ROCS forward (rocs_forward) against the float64 dense early-broadcast
oracle: GLM stack (Wukong-style), DCA with own queries, and the end-to-end ranking forward with
the scoring head.  Reduced batch sizes so the oracle finishes in seconds; the model dims are the
configs' own.  Bounds: relative L2 5e-3, max abs 2e-2 + half a bf16 ulp (bf16 outputs)."""
import numpy as np
import pytest
import torch

import synth
from oracle import rocs_oracle as O
from tests.gpu_util import check_bf16, dev, dev_i32, host, stream

pytestmark = pytest.mark.gpu

FP32_KEYS = ("b_R", "b_C", ".b", "gamma", "beta")


@pytest.fixture(scope="module")
def R():
    from request_candidate_sharing_b200 import rocs
    h = rocs.Rocs(0)
    yield h
    h.close()


def run_forward(R, case, x, W):
    from request_candidate_sharing_b200 import rocs
    md = rocs.model_desc(case)
    Wd = {k: dev(v, torch.float32 if k.endswith(FP32_KEYS) else torch.bfloat16) for k, v in W.items()}
    g, a = case.glm, case.dca
    mw = rocs.model_weights(Wd, g.layers if g else 0, a.layers if a else 0, case.scoring is not None)
    keep = dict(W=Wd)
    xin = {k: dev(v) for k, v in x.items() if k != "hist_len"}
    keep["x"] = xin
    counts = dev_i32(case.counts)
    hl = dev_i32(x["hist_len"]) if "hist_len" in x else None
    keep["hist_len"] = hl
    inp = rocs.Inputs(counts.data_ptr(), rocs.ptr(xin.get("E_R")), rocs.ptr(xin.get("E_C")),
                      rocs.ptr(xin.get("H")), rocs.ptr(xin.get("Y_R")), rocs.ptr(xin.get("Y_C")), rocs.ptr(hl))
    B_R, B_C = case.B_R, case.B_C
    out = {"offsets": torch.empty(B_R + 1, dtype=torch.int32, device="cuda"),
           "req_idx": torch.empty(max(B_C, 1), dtype=torch.int32, device="cuda")}
    if g is not None:
        out["E_R"] = torch.empty((B_R, g.n_R, g.D), dtype=torch.float32, device="cuda")
        out["E_C"] = torch.empty((max(B_C, 1), g.n_C, g.D), dtype=torch.float32, device="cuda")
    if a is not None:
        out["S"] = torch.empty((a.layers, B_R, a.L, a.d), dtype=torch.bfloat16, device="cuda")
        out["A_R"] = torch.empty((a.layers, B_R, a.d), dtype=torch.float32, device="cuda")
        out["A_C"] = torch.empty((a.layers, B_C, a.d), dtype=torch.float32, device="cuda")
    if case.scoring is not None:
        out["score"] = torch.empty(max(B_C, 1), dtype=torch.float32, device="cuda")
    o = rocs.Outputs(*[rocs.ptr(out.get(k)) for k in ("offsets", "req_idx", "E_R", "E_C", "S", "A_R", "A_C", "score")])
    nb = R.rocs_forward_workspace(md)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    R.rocs_forward(md, mw, inp, o, ws, nb, stream())
    assert R.rocs_get_device_status(stream()) == 0
    return out


def test_forward_glm_stack(R):
    case = synth.model_cfg3(B_R=3, counts=[5, 0, 37])
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    off, m = O.segments(case.counts)
    assert np.array_equal(out["offsets"].cpu().numpy(), off)
    assert np.array_equal(out["req_idx"][:case.B_C].cpu().numpy(), m)
    ref = O.forward_cfg3(case, x, W, m)
    check_bf16(host(out["E_R"]), ref["E_R"], what="E_R")
    check_bf16(host(out["E_C"][:case.B_C]), ref["E_C"], what="E_C")


def test_forward_glm_stack_narrow_candidates(R):
    """8 candidate and 24 request embeddings: the fused candidate pass then has padding token rows
    (n_C < 16) and four 8-wide Gram column tiles; two GLM layers, fp32 then bf16 stream."""
    g = synth.GLMShape(n_R=24, n_C=8, hidden=256, fm_out_R=12, lcb_out_R=12, fm_out_C=4, lcb_out_C=4, layers=2)
    case = synth.ModelCase("cfg3", np.asarray([5, 0, 37, 120], np.int32), 3, g, None, None)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    _, m = O.segments(case.counts)
    ref = O.forward_cfg3(case, x, W, m)
    check_bf16(host(out["E_R"]), ref["E_R"], what="E_R")
    check_bf16(host(out["E_C"][:case.B_C]), ref["E_C"], what="E_C")


def test_forward_glm_stack_wide_requests(R):
    """48 request and 16 candidate embeddings (n_R + n_C = 64, the widest group pair): the fused
    candidate pass takes layer 0 (bf16 embeddings), and its shared memory would not hold the pair
    tiles next to a ring of fp32 stages, so the later layers take the two-kernel path (masked FM,
    then token LCB).  Three layers: bf16, then two fp32 stream layers."""
    g = synth.GLMShape(n_R=48, n_C=16, hidden=256, fm_out_R=24, lcb_out_R=24, fm_out_C=8, lcb_out_C=8, layers=3)
    case = synth.ModelCase("cfg3", np.asarray([5, 0, 37, 120, 1], np.int32), 11, g, None, None)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    _, m = O.segments(case.counts)
    ref = O.forward_cfg3(case, x, W, m)
    check_bf16(host(out["E_R"]), ref["E_R"], what="E_R")
    check_bf16(host(out["E_C"][:case.B_C]), ref["E_C"], what="E_C")


@pytest.mark.parametrize("cfg", ["cfg3", "cfg4", "cfg5"])
def test_forward_without_candidates(R, cfg):
    """A batch whose requests have no candidates at all (B_C = 0): the request-side results still
    match the oracle, and no candidate pointer is needed."""
    kw = dict(L=256) if cfg == "cfg5" else {}
    case = getattr(synth, "model_" + cfg)(B_R=3, counts=[0, 0, 0], **kw)
    assert case.B_C == 0
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    off, m = O.segments(case.counts)
    assert np.array_equal(out["offsets"].cpu().numpy(), off)
    ref = getattr(O, "forward_" + cfg)(case, x, W, m)
    if case.glm is not None:
        check_bf16(host(out["E_R"]), ref["E_R"], what="E_R")
    if case.dca is not None:
        for l in range(case.dca.layers):
            check_bf16(host(out["S"][l]), ref["S"][l], out_bf16=True, what=f"S_{l}")
            check_bf16(host(out["A_R"][l]), ref["A_R"][l], what=f"A_R_{l}")


def test_forward_glm_invariant_on_gpu(R):
    case = synth.model_cfg3(B_R=2, counts=[9, 4])
    x, W = synth.model_inputs(case), synth.model_weights(case)
    o1 = run_forward(R, case, x, W)
    x2 = dict(x)
    x2["E_C"] = synth.bf16_round(x["E_C"] * 0.5 - 1.0)
    o2 = run_forward(R, case, x2, W)
    assert torch.equal(o1["E_R"], o2["E_R"])
    x3 = dict(x)
    x3["E_C"] = x["E_C"].copy()
    x3["E_C"][2] = synth.bf16_round(x3["E_C"][2] + 1.0)
    o3 = run_forward(R, case, x3, W)
    keep = [i for i in range(case.B_C) if i != 2]
    assert torch.equal(o1["E_C"][keep], o3["E_C"][keep])


def test_forward_dca_own_queries(R):
    case = synth.model_cfg4(B_R=2, counts=[7, 3])
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    _, m = O.segments(case.counts)
    ref = O.forward_cfg4(case, x, W, m)
    for l in range(case.dca.layers):
        check_bf16(host(out["S"][l]), ref["S"][l], out_bf16=True, what=f"S_{l}")
        check_bf16(host(out["A_R"][l]), ref["A_R"][l], what=f"A_R_{l}")
        check_bf16(host(out["A_C"][l]), ref["A_C"][l], what=f"A_C_{l}")


def test_forward_end_to_end_scoring(R):
    case = synth.model_cfg5(B_R=3, counts=[4, 1, 20], L=256)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    _, m = O.segments(case.counts)
    ref = O.forward_cfg5(case, x, W, m)
    check_bf16(host(out["score"][:case.B_C]), ref["score"], what="score")
    check_bf16(host(out["E_R"]), ref["E_R"], what="E_R")
    check_bf16(host(out["E_C"][:case.B_C]), ref["E_C"], what="E_C")
    for l in range(case.dca.layers):
        check_bf16(host(out["A_R"][l]), ref["A_R"][l], what=f"A_R_{l}")
        check_bf16(host(out["A_C"][l]), ref["A_C"][l], what=f"A_C_{l}")


def test_forward_glm_stack_many_candidates(R):
    """More than 16384 candidates: the candidate LayerNorm takes its streaming (bulk-copy ring)
    path, layer 0 with an fp32 input and a bf16 residual, and each CTA of the fused candidate
    pass walks thousands of candidates across request boundaries.  Sampled candidates (first and
    last of every request among them) against the oracle."""
    from tests.gpu_util import sample_candidates
    counts = [6000, 1, 5000, 0, 7000, 2999]
    case = synth.model_cfg3(B_R=len(counts), counts=counts, seed=11)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    _, m = O.segments(case.counts)
    rows = sample_candidates(case.counts, 6)
    xs = dict(x)
    xs["E_C"] = x["E_C"][rows]
    ref = O.forward_cfg3(case, xs, W, m[rows])
    check_bf16(host(out["E_R"]), ref["E_R"], what="E_R")
    check_bf16(host(out["E_C"][torch.from_numpy(rows).cuda()]), ref["E_C"], what="E_C sample")


def test_forward_graph_replay(R):
    """a11: the second identical rocs_forward call captures the launch sequence into a CUDA graph
    and later calls replay it.  On the same buffers every call must equal the eager run bit for
    bit, and new contents of an input buffer must show in the next replay (the graph reads the
    caller's buffers, it does not snapshot them)."""
    from request_candidate_sharing_b200 import rocs
    case = synth.model_cfg5(B_R=3, counts=[4, 1, 20], L=256)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    md = rocs.model_desc(case)
    Wd = {k: dev(v, torch.float32 if k.endswith(FP32_KEYS) else torch.bfloat16) for k, v in W.items()}
    g, a = case.glm, case.dca
    mw = rocs.model_weights(Wd, g.layers, a.layers, True)
    xin = {k: dev(v) for k, v in x.items()}
    counts = dev_i32(case.counts)
    inp = rocs.Inputs(counts.data_ptr(), rocs.ptr(xin.get("E_R")), rocs.ptr(xin.get("E_C")), rocs.ptr(xin.get("H")),
                      rocs.ptr(xin.get("Y_R")), rocs.ptr(xin.get("Y_C")))
    score = torch.empty(case.B_C, dtype=torch.float32, device="cuda")
    EC = torch.empty((case.B_C, g.n_C, g.D), dtype=torch.float32, device="cuda")
    o = rocs.Outputs(None, None, None, EC.data_ptr(), None, None, None, score.data_ptr())
    nb = R.rocs_forward_workspace(md)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")

    def call():
        R.rocs_forward(md, mw, inp, o, ws, nb, stream())
        assert R.rocs_get_device_status(stream()) == 0
        return score.clone(), EC.clone()

    try:
        R.rocs_set_graph_replay(0)
        s_eager, e_eager = call()
        R.rocs_set_graph_replay(1)
        for _ in range(4):   # eager, capture + launch, replay, replay
            s_g, e_g = call()
            assert torch.equal(s_g, s_eager) and torch.equal(e_g, e_eager)
        # new input contents in the same buffer
        xin["E_C"].copy_(dev(synth.bf16_round(x["E_C"] * 0.5 + 0.25)))
        s_new, e_new = call()
        R.rocs_set_graph_replay(0)
        s_ref, e_ref = call()
        assert torch.equal(s_new, s_ref) and torch.equal(e_new, e_ref)
        assert not torch.equal(s_new, s_eager)
    finally:
        R.rocs_set_graph_replay(1)


def test_forward_fused_ikbo_matches_two_launches(R):
    """Every IKBO linear of the forward (GLM MLPs, query generator, scoring layer 1) as one fused
    launch gives the same bits as the request and candidate launches; 160 requests span two
    request row blocks, with empty and one-candidate requests among them."""
    counts = [int(c) for c in np.random.default_rng(5).integers(0, 40, size=160)]
    counts[7], counts[100] = 1, 0
    case = synth.model_cfg5(B_R=len(counts), counts=counts, L=256)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    try:
        R.rocs_set_ikbo_fused(0)
        out0 = run_forward(R, case, x, W)
        R.rocs_set_ikbo_fused(1)
        out1 = run_forward(R, case, x, W)
    finally:
        R.rocs_set_ikbo_fused(1)
    for k in ("score", "E_R", "E_C", "A_R", "A_C"):
        assert torch.equal(out0[k], out1[k]), k


def test_forward_end_to_end_ragged_history(R):
    """Histories of different lengths inside the padded [B_R, L, d] input (hist_len): the encoder,
    the request and candidate cross-attention all stop at each request's length; padding rows
    hold NaN, so a leak would show in the scores."""
    case = synth.model_cfg5(B_R=4, counts=[4, 1, 20, 7], L=512)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    x = dict(x, hist_len=np.asarray([512, 1, 300, 129], np.int32))
    xn = dict(x)
    xn["H"] = x["H"].copy()
    for r, Lr in enumerate(x["hist_len"]):
        xn["H"][r, Lr:] = np.nan
    out = run_forward(R, case, xn, W)
    _, m = O.segments(case.counts)
    ref = O.forward_cfg5(case, x, W, m)
    check_bf16(host(out["score"][:case.B_C]), ref["score"], what="score")
    for l in range(case.dca.layers):
        check_bf16(host(out["A_R"][l]), ref["A_R"][l], what=f"A_R_{l}")
        check_bf16(host(out["A_C"][l]), ref["A_C"][l], what=f"A_C_{l}")


def test_forward_end_to_end_long_history(R):
    """The bench's history length L = 1024: each warp of the request-query attention walks four
    32-row chunks (online softmax across chunks, then the warps' merge), and the tcgen05
    attention runs eight 128-key blocks per tile with the lazy rescale between them."""
    case = synth.model_cfg5(B_R=2, counts=[3, 130], L=1024, seed=5)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    _, m = O.segments(case.counts)
    ref = O.forward_cfg5(case, x, W, m)
    check_bf16(host(out["score"][:case.B_C]), ref["score"], what="score")
    for l in range(case.dca.layers):
        check_bf16(host(out["A_R"][l]), ref["A_R"][l], what=f"A_R_{l}")
        check_bf16(host(out["A_C"][l]), ref["A_C"][l], what=f"A_C_{l}")


def test_forward_end_to_end_full_size_sampled(R):
    """The benchmarked configuration at full size (512 requests, ~242k candidates, L = 1024): the
    GPU runs the whole forward, the oracle only the sampled requests (the first, the one with the
    most candidates and the last) with four of their candidates each.  Requests are independent,
    so the oracle's sub-batch has the same outputs; its inputs are the same rows of the seeded
    full-case generator."""
    case = synth.model_cfg5()
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    off, m = O.segments(case.counts)
    counts = np.asarray(case.counts)
    reqs = sorted({0, int(np.argmax(counts)), case.B_R - 1})
    g = np.random.default_rng(7)
    rows, m_sub = [], []
    for k, r in enumerate(reqs):
        lo, n = int(off[r]), int(counts[r])
        pick = sorted({lo, lo + n - 1} | {lo + int(v) for v in g.integers(0, n, 2)})
        rows += pick
        m_sub += [k] * len(pick)
    rows, reqs_a = np.asarray(rows), np.asarray(reqs)
    xs = synth.model_inputs(case, cand_rows=rows, req_rows=reqs_a)
    ref = O.forward_cfg5(case, xs, W, np.asarray(m_sub, np.int32))
    rt, qt = torch.from_numpy(rows).cuda(), torch.from_numpy(reqs_a).cuda()
    check_bf16(host(out["score"][rt]), ref["score"], what="score (sampled)")
    check_bf16(host(out["E_R"][qt]), ref["E_R"], what="E_R (sampled requests)")
    check_bf16(host(out["E_C"][rt]), ref["E_C"], what="E_C (sampled)")
    for l in range(case.dca.layers):
        check_bf16(host(out["A_R"][l][qt]), ref["A_R"][l], what=f"A_R_{l} (sampled requests)")
        check_bf16(host(out["A_C"][l][rt]), ref["A_C"][l], what=f"A_C_{l} (sampled)")


def test_forward_glm_stack_stated_size(R):
    """The GLM-stack configuration at its stated size: 64 requests with U[100, 1000] candidates
    each (seed 0), three layers of 32 | 16 embeddings of 128.  The GPU runs every candidate; the
    oracle checks every request and four candidates of each request (its first and last among
    them)."""
    from tests.gpu_util import sample_candidates
    case = synth.model_cfg3()
    assert case.B_R == 64 and case.counts.min() >= 100 and case.counts.max() <= 1000
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    off, m = O.segments(case.counts)
    assert np.array_equal(out["offsets"].cpu().numpy(), off)
    rows = sample_candidates(case.counts, 4)
    xs = dict(x, E_C=x["E_C"][rows])
    ref = O.forward_cfg3(case, xs, W, m[rows])
    rt = torch.from_numpy(rows).cuda()
    check_bf16(host(out["E_R"]), ref["E_R"], what="E_R (every request)")
    check_bf16(host(out["E_C"][rt]), ref["E_C"], what="E_C (sampled)")


def test_forward_dca_stated_size(R):
    """The DCA configuration at its stated size: 32 requests x 500 candidates, history L = 200,
    d = 256, 4 heads, 2 encoder layers, 16 + 8 query embeddings of 256 (seed 0).  Every encoder
    output and request attention output is checked, and four candidates of each request."""
    from tests.gpu_util import sample_candidates
    case = synth.model_cfg4()
    assert (case.B_R, case.B_C, case.dca.L, case.dca.H) == (32, 16000, 200, 4)
    x, W = synth.model_inputs(case), synth.model_weights(case)
    out = run_forward(R, case, x, W)
    _, m = O.segments(case.counts)
    rows = sample_candidates(case.counts, 4)
    xs = dict(x, Y_C=x["Y_C"][rows])
    ref = O.forward_cfg4(case, xs, W, m[rows])
    rt = torch.from_numpy(rows).cuda()
    for l in range(case.dca.layers):
        check_bf16(host(out["S"][l]), ref["S"][l], out_bf16=True, what=f"S_{l}")
        check_bf16(host(out["A_R"][l]), ref["A_R"][l], what=f"A_R_{l}")
        check_bf16(host(out["A_C"][l][rt]), ref["A_C"][l], what=f"A_C_{l} (sampled)")
