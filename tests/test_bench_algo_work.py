"""The algorithmic work behind the bench line's roofline fractions, for the end-to-end workload
(512 requests, 242,464 candidates; GLM: 32 | 16 embeddings of width 128, hidden 1024, 16 | 8 FM
tokens and 16 | 8 LCB tokens, 3 layers; DCA: L = 1024, d = 256, 8 heads, 3 depths; scoring
512-256-1), written out by hand from the kernels' definitions."""
import bench

B_R, B_C, L, H, d = 512, 242_464, 1024, 8, 256


def work(label):
    case = bench.make_case("rocs_forward_e2e", 0, 0)
    assert (case.B_R, case.B_C) == (B_R, B_C)
    return bench.algo_work(case, label)


def test_attention_exponentials():
    # one exponential per (query, key) score and head
    assert work("enc.attn:attn_tc") == ("alu", 8 * 512 * 1024 * 1024)           # 4.29e9
    assert work("xattn.cand:attn_tc") == ("alu", 8 * 242_464 * 1024)            # 1.99e9


def test_bandwidth_bound_bytes():
    # candidate LayerNorm: reads the FM-MLP tokens o (8 x 128 fp32), the LCB tokens L (8 x 128
    # fp32) and the residual E (16 x 128 fp32), writes E' (16 x 128 fp32): 24 KiB per candidate
    assert work("glm.lnC:layernorm") == ("hbm", 242_464 * 24_576)
    # fused candidate pass: E^C read once (4 KiB bf16 at layer 0, 8 KiB fp32 at layers 1 and 2:
    # 20 KiB over three layers), F^C written as a hi/lo pair (16 x 48 x 4 bytes), L^C in fp32
    # (8 x 128 x 4) and the query token as a hi/lo pair (128 x 4)
    bound, b = work("glm.fm:glm_cand_fused")
    assert bound == "hbm"
    assert abs(b - 242_464 * (20_480 / 3 + 3_072 + 4_096 + 512)) < 1.0
    # the request query's attention reads the final encoder output once (bf16)
    assert work("xattn.req:attn_req") == ("hbm", 512 * 1024 * 256 * 2)


def test_gemm_flops():
    # GLM-MLP 1: candidates 16 x 48 = 768 FM values -> 1024 hidden; requests 32 x 32 = 1024 FM
    # values -> 1024 hidden, twice (the request output and Z)
    assert work("glm.mlp1.ikbo:gemm_tc") == ("tensor", 2.0 * 242_464 * 1024 * 768 + 2.0 * 512 * 1024 * 1024 * 2)
    # GLM-MLP 2: hidden 1024 -> 8 x 128 candidate tokens; requests -> 16 x 128 + 8 x 128 (Z)
    assert work("glm.mlp2.ikbo:gemm_tc") == ("tensor", 2.0 * 242_464 * 1024 * 1024 + 2.0 * 512 * 3072 * 1024)
    # encoder Q/K/V projections over every history row, d x d each
    assert work("enc.qkv:gemm_tc") == ("tensor", 2.0 * 512 * 1024 * 256 * 256 * 3)
    # candidate-group K/V only (the request group's are absorbed into its query's attention)
    assert work("enc.kv:gemm_tc") == ("tensor", 2.0 * 512 * 1024 * 256 * 256 * 2)
    # scoring layer 1: candidate input 16 x 128 + 3 x 256 = 2816, request input 32 x 128 + 768
    assert work("score.l1.ikbo:gemm_tc") == ("tensor", 2.0 * 242_464 * 512 * 2816 + 2.0 * 512 * 512 * 4864)


def test_unknown_site_has_no_roofline():
    assert work("fwd:iota") is None


def test_roofline_entries_from_launch_times():
    """The per-kernel entries of the bench line: achieved = work per launch / mean launch time,
    against the measured peaks; the split-A GEMMs also report the executed fraction (twice the
    flops).  Launch times as one bench line reported them."""
    case = bench.make_case("rocs_forward_e2e", 0, 0)
    peaks = dict(hbm=6540.0, tensor=1614.0, tensor_sustained=1366.0, sm_mhz=1965.0, source="measured",
                 exp2_gps=5593.6)
    e = bench.roofline_entry(case, "glm.mlp2.ikbo:gemm_tc", 30, 30 * 0.8231, peaks, sustained=True)
    flops = 2.0 * 242_464 * 1024 * 1024 + 2.0 * 512 * 3072 * 1024
    assert e["unit"] == "TFLOP/s" and e["peak"] == 1366.0
    assert abs(e["achieved"] - flops / 0.8231e-3 / 1e12) < 1e-3
    assert abs(e["frac"] - flops / 0.8231e-3 / 1e12 / 1366.0) < 1e-4
    assert abs(e["executed_frac"] - 2 * e["frac"]) < 2e-4
    e = bench.roofline_entry(case, "enc.attn:attn_tc", 30, 30 * 1.7256, peaks, sustained=True)
    assert e["unit"] == "Gexp2/s" and e["peak"] == 5593.6
    assert abs(e["frac"] - 8 * 512 * 1024 * 1024 / 1.7256e-3 / 1e9 / 5593.6) < 1e-4
    e = bench.roofline_entry(case, "glm.lnC:layernorm", 30, 30 * 0.9548, peaks, sustained=True)
    assert e["unit"] == "GB/s" and e["peak"] == 6540.0 and "executed_frac" not in e
    assert abs(e["frac"] - 242_464 * 24_576 / 0.9548e-3 / 1e9 / 6540.0) < 1e-4
    assert bench.roofline_entry(case, "glm.lnC:layernorm", 0, 0.0, peaks, sustained=True) is None


def test_forward_roofline_sums_sites_against_their_roofs():
    """The whole-forward roofline: per step, each site's launches times its work over its roof
    (burst bf16, HBM, the measured exponential rate), summed and divided by the step time.
    Sites with no work entry count as uncovered time."""
    case = bench.make_case("rocs_forward_e2e", 0, 0)
    peaks = dict(hbm=6540.0, tensor=1614.0, tensor_sustained=1366.0, sm_mhz=1965.0, source="measured",
                 exp2_gps=5600.0)
    steps = 2
    report = {"enc.attn:attn_tc": (3 * steps, 5.2 * steps),        # 3 launches per step
              "glm.lnC:layernorm": (3 * steps, 2.9 * steps),
              "glm.mlp2.ikbo:gemm_tc": (3 * steps, 2.5 * steps),
              "qgen.mlp1.cand:gemm_tc": (3 * steps, 0.4 * steps),
              "fwd:iota": (2 * steps, 0.1 * steps),
              "dropped": (0, 0.0)}
    r = bench.forward_roofline(case, report, steps, 20.0, peaks)
    ideal_ms = 1e3 * 3 * (8 * 512 * 1024 * 1024 / 5600e9
                          + 242_464 * 24_576 / 6540e9
                          + (2.0 * 242_464 * 1024 * 1024 + 2.0 * 512 * 3072 * 1024) / 1614e12
                          + 2.0 * 242_464 * 256 * 128 / 1614e12)
    assert abs(r["ideal_ms"] - ideal_ms) < 1e-3
    assert abs(r["frac"] - ideal_ms / 20.0) < 1e-4
    assert abs(r["covered_kernel_ms"] - (5.2 + 2.9 + 2.5 + 0.4)) < 1e-6
    assert abs(r["uncovered_kernel_ms"] - 0.1) < 1e-6
    assert r["measured_ms"] == 20.0
