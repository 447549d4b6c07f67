#!/usr/bin/env python
"""Throughput of the ROCS forward hot path on B200 (librocs), one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl librocs|reference]

A step is one rocs_forward over one batch of synthetic requests (default workload: the
end-to-end ranking forward -- Wukong-style GLM stack, DCA with L=1024 histories, scoring head --
over 512 requests with lognormal candidate counts).  `value` is candidates scored per second
with inputs resident in HBM (device-timed with CUDA events, max over ranks); `e2e` repeats the
measurement through the same C-ABI call with the inputs copied from pinned host memory and the
scores copied back inside the timed region.  With N > 1 (torchrun) every rank runs its own shard
of requests (weak scaling, no collective on the data path).

--impl reference times the float64 oracle (the reference arm of this build) on bounded samples
of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "candidates/sec per B200 for ROCS forward; % of HBM or bf16 tensor roofline"
FP32_KEYS = ("b_R", "b_C", ".b", "gamma", "beta")


# ---------------------------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------------------------
WORKLOADS = {
    "rocs_forward_e2e": "end-to-end ranking forward: GLM stack (3 layers, 32|16 embeddings of 128) + DCA "
                        "(L=1024, d=256, 8 heads, 3 depths) + scoring MLP 512-256-1; 512 requests, "
                        "candidates ~ clipped lognormal (median 300, 16..2000), seed 1",
    "rocs_forward_ragged": "the end-to-end ranking forward with ragged histories: request r's history is its first "
                           "hist_len[r] of the L=1024 rows, hist_len ~ U[256, 1024] (seed 1), padding rows hold zeros",
    "glm_stack": "Wukong-style GLM stack, 3 layers; 64 requests, candidates ~ U[100,1000], seed 0",
    "dca": "DCA path: L=200, d=256, 4 heads, 2 layers; 32 requests x 500 candidates, seed 0",
    "ikbo_sweep": "IKBO linear sweep: B_R=256, N in {64, 256, 1024} candidates per request, d_in = d_out = d in "
                  "{512, 1024, 4096}, bf16 in/out, fp32 accumulate, ReLU; against two materialised-broadcast "
                  "GPU baselines (B1: Z[m] materialised and added; B2: gathered [X^R[m], X^C] with one K=2d GEMM)",
    "w8a16": "FP8-weight (W8A16) IKBO linear against the same linear with bf16 weights, weights read from HBM "
             "(L2 flushed): the UG-Separation review's four configurations (1, N, d_in, d_out) = (1, 16|8, 1280, "
             "2560|640) read as one request with N candidates, plus two larger weight-bound shapes; the default "
             "FP8 path and the opt-in tensor-core path (FP8 operands converted in shared memory)",
    "ex2_rate": "throughput of the attention softmax's exponentials (scale and shift on the packed FMA path, 2^x, "
                "bf16 packing) with n_poly of every eight pairs on the FMA-pipe polynomial and the rest on MUFU ex2, "
                "n_poly = 0..8; every SM filled (2048 threads each)",
    "xattn_unsorted": "candidate cross-attention with candidates in shuffled order (each with its request index): "
                      "512 requests, candidates ~ clipped lognormal (median 300, 16..2000), L=1024, d=256, 8 heads; "
                      "stable sort by request + gather + segment-path attention + scatter, against the grouped call",
}


# Work of one request and of one candidate in the end-to-end forward (microseconds on one B200,
# from the bench's per-site split: the encoder, its projections and the request query scale with
# requests, everything else with candidates); the weights of the LPT request partition.
SHARD_COST_R, SHARD_COST_C = 14.8, 0.0586


def make_case(name: str, rank: int, requests: int = 0, shard: str = "own", world: int = 1):
    """The workload's case; `requests` > 0 keeps only the first requests (smaller profiling runs).
    shard "own": every rank draws its own batch (seed + 1000 rank; weak scaling).  shard "lpt":
    every rank builds the same batch and keeps its part of rocs_partition_requests over `world`
    parts (whole requests, longest processing time first; strong scaling)."""
    if shard == "lpt" and world > 1:
        full = make_case(name, 0, requests)
        from request_candidate_sharing_b200 import rocs
        part = rocs.partition_requests(full.counts, world, SHARD_COST_R, SHARD_COST_C)
        return dataclasses.replace(full, counts=full.counts[part == rank].copy())
    seed_shift = 1000 * rank
    if name == "rocs_forward_e2e":
        case = synth.model_cfg5(seed=1 + seed_shift)
    elif name == "rocs_forward_ragged":
        case = dataclasses.replace(synth.model_cfg5(seed=1 + seed_shift), name="cfg5_ragged")
    elif name == "glm_stack":
        case = synth.model_cfg3(seed=0 + seed_shift)
    elif name == "dca":
        case = synth.model_cfg4(seed=0 + seed_shift)
    else:
        raise SystemExit(f"unknown workload {name}")
    if requests and requests < case.B_R:
        case = dataclasses.replace(case, counts=case.counts[:requests].copy())
    return case


# ---------------------------------------------------------------------------------------------
# algorithmic work per launch (for the roofline of the dominant kernel)
# ---------------------------------------------------------------------------------------------
ATTN_MUFU_SHARE = 5.0 / 8.0   # share of the attention softmax's exponentials evaluated on MUFU


def algo_work(case, label: str):
    """(bound, amount per launch, unit) for a timing-report label "<site>:<kernel>", or None.
    GEMMs: mathematical flops 2*M*N*K (a split hi/lo operand counts once).  Bandwidth-bound
    kernels: compulsory bytes of the tensors they read and write, in their stored precision.
    Attention: exp2 evaluations (one per score), the MUFU-bound quantity."""
    B_R, B_C = case.B_R, case.B_C
    g, a = case.glm, case.dca
    site, _, kern = label.partition(":")
    if g is not None:
        fR, fC = g.n_R * g.n_R, g.n_C * (g.n_R + g.n_C)
        wr, wc = g.n_R * g.D, g.n_C * g.D
        oRw, oCw = g.fm_out_R * g.D, g.fm_out_C * g.D
        lRw, lCw = g.lcb_out_R * g.D, g.lcb_out_C * g.D
        table = {
            "glm.mlp1.cand:gemm_tc": ("tensor", 2.0 * B_C * g.hidden * fC),
            "glm.mlp1.req:gemm_tc": ("tensor", 2.0 * B_R * g.hidden * fR * 2),
            "glm.mlp2.cand:gemm_tc": ("tensor", 2.0 * B_C * oCw * g.hidden),
            "glm.mlp2.req:gemm_tc": ("tensor", 2.0 * B_R * (oRw + oCw) * g.hidden),
            # one fused launch (request and candidate tiles): the sum of the two
            "glm.mlp1.ikbo:gemm_tc": ("tensor", 2.0 * B_C * g.hidden * fC + 2.0 * B_R * g.hidden * fR * 2),
            "glm.mlp2.ikbo:gemm_tc": ("tensor", 2.0 * B_C * oCw * g.hidden + 2.0 * B_R * (oRw + oCw) * g.hidden),
            # fused candidate pass: reads E^C (bf16 at layer 0, fp32 after), writes F^C (hi/lo),
            # L^C (fp32) and, when DCA queries come from the GLM stack, t^C (hi/lo)
            "glm.fm:glm_cand_fused": ("hbm", B_C * (wc * (2 + 4 * (g.layers - 1)) / g.layers + fC * 4 + lCw * 4
                                                   + (4 * a.q_dim if (a is not None and a.source == "glm") else 0))),
            "glm.lnC:layernorm": ("hbm", B_C * (oCw * 4 + lCw * 4 + wc * 4 + wc * 4)),
        }
        if label in table:
            return table[label]
    if a is not None:
        L, d, H = a.L, a.d, a.H
        # history rows that exist (a ragged workload counts each request's own length: the rows
        # the row-wise kernels spend on padding are no algorithmic work)
        hl = hist_len_of(case)
        hl = np.full(B_R, L, np.int64) if hl is None else np.asarray(hl[:B_R], np.int64)
        rows_h = float(hl.sum())                                   # history tokens
        pairs = float((hl * hl).sum())                             # self-attention (query, key) pairs
        cand_keys = float((np.asarray(case.counts, np.int64) * hl).sum())   # candidate (query, key) pairs
        table = {
            "enc.attn:attn": ("alu", H * pairs),
            "enc.attn:attn_tc": ("alu", H * pairs),
            "enc.attn:attn_stream": ("alu", H * pairs),
            "xattn.cand:attn_stream": ("alu", H * cand_keys),
            "xattn.cand:attn_tc": ("alu", H * cand_keys),
            "enc.qkv:gemm_tc": ("tensor", 2.0 * rows_h * d * d * 3),
            # the candidate group's K/V only when the request query's attention absorbs its
            # projections (d = 256, up to 8 heads of a multiple of 16), else all four
            "enc.kv:gemm_tc": ("tensor", 2.0 * rows_h * d * d * (2 if (d == 256 and H <= 8 and (d // H) % 16 == 0) else 4)),
            "enc.wo:gemm_tc": ("tensor", 2.0 * rows_h * d * d),
            "enc.ln:layernorm": ("hbm", rows_h * d * 2 * 3.0),
            # query generator, two IKBO linears q_dim -> d -> d: one fused launch (request and
            # candidate tiles) or a request launch ([Y^R | Z], 2d outputs) and a candidate launch
            "qgen.mlp1.ikbo:gemm_tc": ("tensor", 2.0 * (B_C + 2 * B_R) * d * a.q_dim),
            "qgen.mlp2.ikbo:gemm_tc": ("tensor", 2.0 * (B_C + 2 * B_R) * d * d),
            "qgen.mlp1.req:gemm_tc": ("tensor", 2.0 * 2 * B_R * d * a.q_dim),
            "qgen.mlp1.cand:gemm_tc": ("tensor", 2.0 * B_C * d * a.q_dim),
            "qgen.mlp2.req:gemm_tc": ("tensor", 2.0 * 2 * B_R * d * d),
            "qgen.mlp2.cand:gemm_tc": ("tensor", 2.0 * B_C * d * d),
            # the request query's attention with its projections absorbed reads the final
            # encoder output S once (bf16); weights and queries are L2-resident and negligible
            "xattn.req:attn_req": ("hbm", rows_h * d * 2),
        }
        if label in table:
            return table[label]
    if case.scoring is not None:
        h1, h2 = case.scoring
        xc = g.n_C * g.D + a.layers * a.d
        xr = g.n_R * g.D + a.layers * a.d
        table = {"score.l1.cand:gemm_tc": ("tensor", 2.0 * B_C * h1 * xc),
                 "score.l1.ikbo:gemm_tc": ("tensor", 2.0 * B_C * h1 * xc + 2.0 * B_R * h1 * xr),
                 "score.l2:gemm_tc": ("tensor", 2.0 * B_C * h2 * h1)}
        if label in table:
            return table[label]
    return None


def gpu_local_cpus(dev) -> set:
    """The CPUs of the GPU's own NUMA node (sysfs local_cpulist of its PCI function) that this
    process may run on; empty when unknown."""
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        bdf = f"{p.pci_domain_id:04x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        with open(f"/sys/bus/pci/devices/{bdf}/local_cpulist") as f:
            text = f.read().strip()
        cpus = set()
        for part in text.split(","):
            if "-" in part:
                a, b = part.split("-")
                cpus.update(range(int(a), int(b) + 1))
            elif part:
                cpus.add(int(part))
        return cpus & os.sched_getaffinity(0)
    except (OSError, ValueError, AttributeError, RuntimeError):
        return set()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(hbm=float(j["hbm_gbs"]), tensor=float(j["bf16_tflops"]),
                    tensor_sustained=float(j["bf16_tflops_sustained"]), sm_mhz=float(j.get("sm_max_mhz", 1965.0)),
                    source="measured")
    return dict(hbm=6650.0, tensor=1590.0, tensor_sustained=1400.0, sm_mhz=1965.0, source="fallback")


def forward_roofline(case, report, steps: int, ms_per_step: float, peaks):
    """The whole forward against its roofline: the sum over the per-kernel report's sites of
    (algorithmic work per launch / the site's roof) x launches per step, divided by the measured
    step time.  Roofs: burst bf16 tensor, HBM copy bandwidth, and the exponential rate measured
    in the same run.  Sites with no algorithmic-work entry (small request-side kernels,
    bookkeeping) add nothing to the ideal time; their measured time is reported as uncovered."""
    roof = {"tensor": peaks["tensor"] * 1e12, "hbm": peaks["hbm"] * 1e9,
            "alu": (peaks.get("exp2_gps") or 16 / ATTN_MUFU_SHARE * 148 * peaks["sm_mhz"] * 1e-3) * 1e9}
    ideal = covered = uncovered = 0.0
    for name, (n, t) in report.items():
        w = algo_work(case, name)
        if w is None or n == 0:
            uncovered += t / steps
            continue
        bound, amount = w
        ideal += amount / roof[bound] * 1e3 * n / steps
        covered += t / steps
    return {"ideal_ms": round(ideal, 3), "measured_ms": round(ms_per_step, 4), "frac": round(ideal / ms_per_step, 4),
            "covered_kernel_ms": round(covered, 3), "uncovered_kernel_ms": round(uncovered, 3),
            "roofs": (f"bf16 {peaks['tensor']:.0f} TFLOP/s (burst), HBM {peaks['hbm']:.0f} GB/s, "
                      f"exp2 {roof['alu'] / 1e9:.0f} G/s")}


# GEMM sites whose A operand is a bf16 hi/lo pair (the GLM MLPs and the DCA query generator): the
# tensor cores execute twice the algorithmic flops there
SPLIT_A_SITES = ("glm.mlp1.", "glm.mlp2.", "qgen.mlp1.", "qgen.mlp2.")


def roofline_entry(case, label, launches, total_ms, peaks, sustained: bool):
    w = algo_work(case, label)
    if w is None or launches == 0:
        return None
    bound, amount = w
    per_launch_s = total_ms / launches / 1e3
    if bound == "tensor":
        achieved = amount / per_launch_s / 1e12
        peak = peaks["tensor_sustained"] if sustained else peaks["tensor"]
        unit = "TFLOP/s"
    elif bound == "hbm":
        achieved = amount / per_launch_s / 1e9
        peak = peaks["hbm"]
        unit = "GB/s"
    else:
        achieved = amount / per_launch_s / 1e9
        unit = "Gexp2/s"
        if peaks.get("exp2_gps"):
            # measured in this run by rocs_probe_exp2_rate: the softmax's per-score steps with the
            # attention kernels' split (3 of 8 exponential pairs on the FMA-pipe polynomial)
            peak = peaks["exp2_gps"]
            return {"kernel": label, "bound": bound, "achieved": round(achieved, 3), "peak": round(peak, 1),
                    "unit": unit, "frac": round(achieved / peak, 4), "per_launch_ms": round(total_ms / launches, 4),
                    "launches": launches, "peak_source": "measured in this run (rocs_probe_exp2_rate, 3-in-8 split)"}
        # without the probe: MUFU does 16 per clock per SM at the max SM clock and takes 5/8 of
        # the softmax's exponentials, so it caps the rate at 16 / (5/8) = 25.6 per clock per SM
        peak = 16 / ATTN_MUFU_SHARE * 148 * peaks["sm_mhz"] * 1e6 / 1e9
    e = {"kernel": label, "bound": bound, "achieved": round(achieved, 3), "peak": round(peak, 1), "unit": unit,
         "frac": round(achieved / peak, 4), "per_launch_ms": round(total_ms / launches, 4), "launches": launches,
         "peak_source": (f"{peaks['source']}{' sustained' if sustained and bound == 'tensor' else ''}"
                         if bound != "alu" else "derived: 16 ex2/clk/SM / (5/8) x 148 SMs x max SM clock")}
    if bound == "tensor" and label.startswith(SPLIT_A_SITES):
        e["executed_frac"] = round(2.0 * achieved / peak, 4)   # hi and lo halves of A both multiplied
    return e


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        text = open(self.f.name).read()
        os.unlink(self.f.name)
        return summarize_clocks(text)


def summarize_clocks(text: str):
    """The clock record of a timed region from nvidia-smi's CSV rows (ClockSampler.FIELDS, no
    header, no units): the median SM clock of the busier half of the samples (the GPU under
    load), the maximum SM clock, and the throttle reasons that were active in any sample."""
    rows = [r.split(",") for r in text.strip().splitlines() if r.strip()]
    if not rows:
        return None
    sm = [float(r[1]) for r in rows if len(r) > 1 and r[1].strip().replace(".", "").isdigit()]
    mx = float(rows[0][2]) if len(rows[0]) > 2 and rows[0][2].strip().replace(".", "").isdigit() else None
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 5 + i and "Active" in r[5 + i]
                      and "Not" not in r[5 + i]})
    under = sorted(sm)[len(sm) // 2:] if sm else []
    return {"sm_mhz": statistics.median(under) if under else None, "sm_max_mhz": mx, "reasons": reasons,
            "samples": len(rows)}


# ---------------------------------------------------------------------------------------------
# oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def hist_len_of(case):
    """Per-request history lengths of a ragged workload (None otherwise)."""
    if not case.name.endswith("_ragged"):
        return None
    return synth.hist_lengths(case.seed, case.B_R, case.dca.L, case.dca.L // 4)


def ragged_inputs(case, x, req_ids=None):
    """Adds the ragged workload's lengths to the inputs and zeroes the padding rows of H."""
    hl = hist_len_of(case)
    if hl is None:
        return x
    if req_ids is not None:
        hl = hl[np.asarray(req_ids, np.int64)]
    x = dict(x, hist_len=hl)
    H = x["H"].copy()
    for r, Lr in enumerate(hl):
        H[r, Lr:] = 0.0
    x["H"] = H
    return x


def oracle_requests(case, req_ids):
    """Runs the oracle on whole requests `req_ids` of the workload; returns candidates processed."""
    from oracle import rocs_oracle as O
    counts = np.asarray(case.counts)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    req_ids = np.asarray(req_ids, np.int64)
    cand_rows = np.concatenate([np.arange(offsets[r], offsets[r + 1]) for r in req_ids]) if len(req_ids) else \
        np.zeros(0, np.int64)
    sub = dataclasses.replace(case, counts=counts[req_ids])
    x = ragged_inputs(case, synth.model_inputs(case, cand_rows=cand_rows, req_rows=req_ids), req_ids)
    W = synth.model_weights(case)
    _, m = O.segments(sub.counts)
    if case.scoring is not None:
        O.forward_cfg5(sub, x, W, m)
    elif case.dca is not None:
        O.forward_cfg4(sub, x, W, m)
    else:
        O.forward_cfg3(sub, x, W, m)
    return int(counts[req_ids].sum())


def oracle_rate(case, seconds: float, start_req: int = 0):
    """Oracle candidates/s over whole requests taken in order until `seconds` of CPU time."""
    t0 = time.perf_counter()
    n = 0
    r = start_req
    reqs = 0
    while time.perf_counter() - t0 < seconds and reqs < case.B_R:
        n += oracle_requests(case, [r % case.B_R])
        r += 1
        reqs += 1
    dt = time.perf_counter() - t0
    return n / dt, n, reqs, dt


# ---------------------------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------------------------
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    return rank, world, local


def allreduce(x: float, op: str, world: int) -> float:
    """Max or sum of a scalar over ranks (the measurement's only collective)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def shard_totals(workload: str, rank: int, world: int, requests: int, local_ms: float, shard: str = "own"):
    """Multi-rank bookkeeping of one rank: its request shard, the job-wide candidate total and the
    max-over-ranks time that the throughput divides by."""
    case = make_case(workload, rank, requests, shard, world)
    total = allreduce(float(case.B_C), "sum", world)
    ms_max = allreduce(local_ms, "max", world)
    return case.B_C, total, ms_max


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------------------------
# librocs arm
# ---------------------------------------------------------------------------------------------
def run_librocs(args, rank, world, local):
    import torch

    from request_candidate_sharing_b200 import rocs
    torch.cuda.set_device(local)
    case = make_case(args.workload, rank, args.requests, args.shard, world)
    dev = torch.device("cuda", local)
    t_gen = time.perf_counter()
    W = synth.model_weights(case)
    x = ragged_inputs(case, synth.model_inputs(case))
    hist_len = x.pop("hist_len", None)
    gen_s = time.perf_counter() - t_gen

    def to_dev(v, dt):
        return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(dev).to(dt)

    Wd = {k: to_dev(v, torch.float32 if k.endswith(FP32_KEYS) else torch.bfloat16) for k, v in W.items()}
    xd = {k: to_dev(v, torch.bfloat16) for k, v in x.items()}
    counts_d = torch.from_numpy(case.counts).to(dev)
    hl_d = torch.from_numpy(np.ascontiguousarray(hist_len, np.int32)).to(dev) if hist_len is not None else None
    g, a = case.glm, case.dca
    R = rocs.Rocs(local)
    R.rocs_set_ikbo_fused(args.ikbo_fused)
    md = rocs.model_desc(case)
    mw = rocs.model_weights(Wd, g.layers if g else 0, a.layers if a else 0, case.scoring is not None)
    B_C = case.B_C
    score = torch.empty(max(B_C, 1), dtype=torch.float32, device=dev)
    outE = None
    if case.scoring is None:   # without a scoring head the final activations are the result
        if g is not None:
            outE = (torch.empty((case.B_R, g.n_R, g.D), dtype=torch.float32, device=dev),
                    torch.empty((max(B_C, 1), g.n_C, g.D), dtype=torch.float32, device=dev))
        else:
            outE = (torch.empty((a.layers, case.B_R, a.d), dtype=torch.float32, device=dev),
                    torch.empty((a.layers, max(B_C, 1), a.d), dtype=torch.float32, device=dev))
    nb = R.rocs_forward_workspace(md)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)

    def outputs():
        if case.scoring is not None:
            return rocs.Outputs(None, None, None, None, None, None, None, score.data_ptr())
        if g is not None:
            return rocs.Outputs(None, None, outE[0].data_ptr(), outE[1].data_ptr(), None, None, None, None)
        return rocs.Outputs(None, None, None, None, None, outE[0].data_ptr(), outE[1].data_ptr(), None)

    inp = rocs.Inputs(counts_d.data_ptr(), rocs.ptr(xd.get("E_R")), rocs.ptr(xd.get("E_C")), rocs.ptr(xd.get("H")),
                      rocs.ptr(xd.get("Y_R")), rocs.ptr(xd.get("Y_C")), rocs.ptr(hl_d))
    out = outputs()
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    def step():
        R.rocs_forward(md, mw, inp, out, ws, nb, sh)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = R.rocs_get_device_status(sh)
    if st != 0:
        raise RuntimeError(f"device status {rocs.STATUS_NAMES.get(st, st)} after warm-up")

    # ---- device-timed region: inputs resident in HBM ----
    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
    clocks = ClockSampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else (uuid or str(local)))
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    # inputs smaller than twice the L2: each step is timed alone after an L2 flush (outside its
    # event pair); larger inputs: the steps run back to back
    in_bytes = sum(v.numel() * v.element_size() for v in xd.values())
    small = in_bytes < (256 << 20)
    if small:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        step_ms = []
        for _ in range(args.steps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            step_ms.append(e0.elapsed_time(e1))
        ms = sum(step_ms)
        barrier(world)
    else:
        # an event after every step: the region is first to last, each step the gap between two
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        evs[0].record(stream)
        for i in range(args.steps):
            step()
            evs[i + 1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        ms = evs[0].elapsed_time(evs[-1])
        step_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    # per-kernel report: the same steps again with per-launch CUDA events (direct launches; the
    # timed region above replays the forward's CUDA graph)
    R.rocs_timing_start(200 * args.steps + 64)
    for _ in range(args.steps):
        if small:
            flush.fill_(1)
        step()
    torch.cuda.synchronize(dev)
    report = R.rocs_timing_stop()
    clk = clocks.stop()
    st = R.rocs_get_device_status(sh)
    if st != 0:
        raise RuntimeError(f"device status {rocs.STATUS_NAMES.get(st, st)} in the timed region")
    # the exponential ceiling of the attention kernels, measured on this GPU now (rocs_probe_exp2_rate)
    exp2_probe = {f"n_poly={n}": round(R.rocs_probe_exp2_rate(n, sh) / 1e9, 1) for n in (0, 3, 8)}
    _, total_c, ms_max = shard_totals(args.workload, rank, world, args.requests, ms, args.shard)
    cands = total_c * args.steps
    value = cands / (ms_max / 1e3)

    # ---- end-to-end through the same call with host buffers ----
    # the pinned buffers are allocated (and their pages first touched) by a thread bound to the
    # GPU's local CPUs, so the copy engine reads memory of the GPU's own NUMA node
    old_aff = os.sched_getaffinity(0)
    local = gpu_local_cpus(dev)
    if local:
        os.sched_setaffinity(0, local)
    host = {k: v.cpu().pin_memory() for k, v in xd.items()}
    counts_h = counts_d.cpu().pin_memory()
    hl_h = hl_d.cpu().pin_memory() if hl_d is not None else None
    score_h = torch.empty_like(score, device="cpu").pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values()) + counts_h.numel() * 4 + \
        (hl_h.numel() * 4 if hl_h is not None else 0)
    res = score if case.scoring is not None else outE[1]
    res_h = torch.empty_like(res, device="cpu").pin_memory()
    if local:
        os.sched_setaffinity(0, old_aff)
    d2h = res.numel() * res.element_size()

    # two device input sets: step k+1's inputs are copied (copy stream) while step k computes;
    # every step's inputs still cross PCIe inside the timed region, and each set has its own
    # captured forward graph
    sets = [(xd, counts_d, inp, hl_d)]
    xd2 = {k: torch.empty_like(v) for k, v in xd.items()}
    counts_d2 = torch.empty_like(counts_d)
    hl_d2 = torch.empty_like(hl_d) if hl_d is not None else None
    inp2 = rocs.Inputs(counts_d2.data_ptr(), rocs.ptr(xd2.get("E_R")), rocs.ptr(xd2.get("E_C")),
                       rocs.ptr(xd2.get("H")), rocs.ptr(xd2.get("Y_R")), rocs.ptr(xd2.get("Y_C")), rocs.ptr(hl_d2))
    sets.append((xd2, counts_d2, inp2, hl_d2))
    copy_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    done = [torch.cuda.Event(), torch.cuda.Event()]

    def h2d_into(k):
        xs, cs, _, hs = sets[k % 2]
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(done[k % 2])     # the forward that last read this set is finished
            for name, v in host.items():
                xs[name].copy_(v, non_blocking=True)
            cs.copy_(counts_h, non_blocking=True)
            if hs is not None:
                hs.copy_(hl_h, non_blocking=True)
            copied[k % 2].record(copy_stream)

    def forward_on(k):
        stream.wait_event(copied[k % 2])
        R.rocs_forward(md, mw, sets[k % 2][2], out, ws, nb, sh)
        done[k % 2].record(stream)
        res_h.copy_(res, non_blocking=True)

    def e2e_run(nsteps):
        h2d_into(0)
        for k in range(nsteps):
            if k + 1 < nsteps:
                h2d_into(k + 1)
            forward_on(k)

    e2e_run(4)   # each set's forward: a direct run, then its graph capture, before the timed region
    torch.cuda.synchronize(dev)
    barrier(world)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    copy_stream.wait_event(f0)   # the first copy starts inside the timed region
    e2e_run(args.steps)
    f1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = allreduce(f0.elapsed_time(f1), "max", world)
    e2e_value = cands / (e2e_ms / 1e3)

    # ---- per-kernel breakdown and the dominant kernel's roofline ----
    peaks = load_peaks()
    peaks["exp2_gps"] = exp2_probe["n_poly=3"]
    kernels = sorted(report.items(), key=lambda kv: -kv[1][1])
    launches = sum(n for name, (n, _) in report.items() if name != "dropped")
    total_k = sum(t for _, (_, t) in report.items())
    rooflines = []
    for name, (n, t) in kernels:
        e = roofline_entry(case, name, n, t, peaks, sustained=True)
        if e is not None:
            e["share"] = round(t / total_k, 4) if total_k else None
            rooflines.append(e)
    top = rooflines[0] if rooflines else None
    if top is not None:
        traffic = None
        tp = os.path.join(ROOT, "profiles", "traffic.json")
        if os.path.exists(tp):
            tj = json.load(open(tp)).get(args.workload, {}).get(top["kernel"])
            if tj is not None:
                traffic = tj
        top = {"bound": top["bound"], "achieved": top["achieved"], "peak": top["peak"], "unit": top["unit"],
               "frac": top["frac"], "traffic": traffic, "kernel": top["kernel"],
               "per_launch_ms": top["per_launch_ms"], "peak_source": top["peak_source"] + " (of measured)"
               if top["peak_source"].startswith("measured") else top["peak_source"]}

    line = {"metric": METRIC, "value": round(value, 1), "unit": "candidates/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4),
            "higher_is_better": True, "scaling": "strong" if args.shard == "lpt" and world > 1 else "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) inputs, N(0,1/fan_in) bf16 weights)",
            "config": {"workload": args.workload + (f"[first {case.B_R} requests]" if args.requests else ""),
                       "description": WORKLOADS[args.workload], "B_R": case.B_R,
                       "B_C_per_rank": B_C,
                       "l2": (f"inputs {in_bytes / 1e9:.3f} GB < 2 x L2: each step timed alone after a 256 MB "
                              "L2 flush" if small else f"inputs larger than L2 ({in_bytes / 1e9:.2f} GB), "
                              "steps back to back"),
                       "parallelism": f"replicas x{world}",
                       "ikbo_launch": "fused (request + candidate tiles, completion flags)" if args.ikbo_fused
                                      else "two launches (request GEMM, then candidate GEMM)",
                       "launch": "value and e2e: the forward's captured CUDA graph replayed; per-kernel report "
                                 "(roofline): the same steps again with direct launches and per-launch CUDA events",
                       "e2e_pipelining": "two device input sets: step k+1's host-to-device copy (pinned, copy "
                                         "stream) overlaps step k's forward; every step's inputs are copied and "
                                         "its scores read back inside the timed region",
                       "e2e_host_buffers": (f"pinned, allocated from the GPU's NUMA node ({len(local)} local CPUs)"
                                            if local else "pinned (the GPU's NUMA node is unknown)")},
            "roofline": top,
            "forward_roofline": forward_roofline(case, report, args.steps, ms_max / args.steps, peaks),
            "step_ms": {"median": round(statistics.median(step_ms), 4),
                        "p90": round(sorted(step_ms)[min(len(step_ms) - 1, int(math.ceil(0.9 * len(step_ms))) - 1)], 4),
                        "n": len(step_ms), "rank": 0},
            "e2e": {"value": round(e2e_value, 1), "unit": "candidates/s", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h)},
            "gpu_launches": int(launches),
            "clocks": clk,
            "kernels": [{k: v for k, v in e.items() if k in ("kernel", "bound", "achieved", "unit", "frac", "share",
                                                             "per_launch_ms", "launches", "executed_frac")}
                        for e in rooflines[:8]],
            "kernel_ms": {name: round(t / args.steps, 4) for name, (n, t) in kernels[:16]},
            "input_generation_s": round(gen_s, 1),
            "exp2_probe_Gexp2_per_s": exp2_probe}
    if a is not None and g is not None and not args.no_baselines:
        del ws, sets, xd2
        torch.cuda.empty_cache()
        line["baselines"] = gpu_baselines(R, dev, sh, case, peaks, rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, reqs, dt = oracle_rate(case, args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(rate, 2), "unit": "candidates/s", "cores": blas_threads(),
                                "kind": "oracle",
                                "sample": f"{reqs} whole requests ({n} candidates) of the same workload, "
                                          f"{dt:.1f} s of float64 numpy on the host"}
    R.close()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# GPU materialised-broadcast baselines (torch / cuBLAS / SDPA), beside the headline
# ---------------------------------------------------------------------------------------------
def _timed_median(fn, reps, warmup, flush, dev):
    import torch
    for _ in range(warmup):
        fn()
    ts = []
    for _ in range(reps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize(dev)
        ts.append(e0.elapsed_time(e1))
    ts.sort()
    return ts[len(ts) // 2]


def gpu_baselines(R, dev, sh, case, peaks, rank):
    """B1 and B2 against rocs_linear_ikbo at the IKBO sweep point N = 1024, d = 1024 (256 requests,
    262,144 candidates, bf16, ReLU), and B3 against rocs_dca_cross_attn on the forward's depth-0
    candidate cross-attention shapes (its counts, L, heads).  Each repetition is timed alone after
    an L2 flush (256 MB write); medians.  Inputs: seeded torch normal draws on the device.
      B1  Z = X^R W_CR^T + b^C written out as Z[m] [B_C, d] and added to X^C W_CC^T ("Fig. 3(a)")
      B2  [X^R[m], X^C] gathered and one K = 2d GEMM (the early broadcast)
      B3  K/V copied per candidate ([c, L, d], chunks of 2048 candidates), then SDPA (the pages'
          "explicit K/V broadcast" attention arms)"""
    import torch
    import torch.nn.functional as F
    from request_candidate_sharing_b200 import rocs
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    bf = torch.bfloat16
    out = {}
    # ---- B1 / B2: the IKBO linear ----
    B_R, N, d = 256, 1024, 1024
    B_C = B_R * N
    gen = torch.Generator(device=dev).manual_seed(20 + rank)
    XR = torch.randn(B_R, d, device=dev, generator=gen).to(bf)
    XC = torch.randn(B_C, d, device=dev, generator=gen).to(bf)
    W_RR, W_CR, W_CC = (torch.randn(d, d, device=dev, generator=gen).mul_(d ** -0.5).to(bf) for _ in range(3))
    bR = torch.rand(d, device=dev, generator=gen) * 0.2 - 0.1
    bC = torch.rand(d, device=dev, generator=gen) * 0.2 - 0.1
    m = torch.arange(B_R, device=dev, dtype=torch.int32).repeat_interleave(N)
    mi = m.long()
    YR = torch.empty(B_R, d, dtype=bf, device=dev)
    YC = torch.empty(B_C, d, dtype=bf, device=dev)
    desc = rocs.IkboDesc(B_R, B_C, d, d, d, d, rocs.ROCS_BF16, rocs.ROCS_BF16, rocs.ACT["relu"])
    nb = R.rocs_linear_ikbo_workspace(desc)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
    W2 = torch.cat([W_CR, W_CC], 1)
    res = {}

    def ikbo():
        R.rocs_linear_ikbo(desc, XR, XC, m, W_RR, W_CR, W_CC, bR, bC, YR, YC, ws, nb, sh)

    def b1():
        z = torch.addmm(bC, XR.float(), W_CR.float().t()).to(bf)
        res["b1"] = torch.relu_(torch.addmm(z.index_select(0, mi), XC, W_CC.t()))
        torch.relu_(torch.addmm(bR.to(bf), XR, W_RR.t()))

    def b2():
        xg = torch.cat([XR.index_select(0, mi), XC], 1)
        res["b2"] = torch.relu_(torch.addmm(bC.to(bf), xg, W2.t()))
        torch.relu_(torch.addmm(bR.to(bf), XR, W_RR.t()))

    t_i, t_1, t_2 = (_timed_median(f, 5, 3, flush, dev) for f in (ikbo, b1, b2))
    flops = 2.0 * B_C * d * d + 2.0 * B_R * d * d * 2
    out["linear_N1024_d1024"] = {
        "rocs_linear_ikbo_ms": round(t_i, 4), "B1_materialised_Zm_ms": round(t_1, 4),
        "B2_gathered_2d_gemm_ms": round(t_2, 4), "speedup_vs_B1": round(t_1 / t_i, 3),
        "speedup_vs_B2": round(t_2 / t_i, 3),
        "ikbo_tflops": round(flops / (t_i / 1e3) / 1e12, 1),
        "max_abs_diff_vs_B2": round(float((YC.float() - res["b2"].float()).abs().max()), 4)}
    del XR, XC, W_RR, W_CR, W_CC, YR, YC, ws, W2, res, m, mi
    torch.cuda.empty_cache()
    # ---- B3: candidate cross-attention with K/V copied per candidate ----
    a = case.dca
    L, H, dh = a.L, a.H, a.d // a.H
    counts = torch.from_numpy(np.asarray(case.counts, np.int64)).to(dev)
    Bc = int(counts.sum())
    Q = torch.randn(Bc, a.d, device=dev, generator=gen).to(bf)
    K = torch.randn(case.B_R, L, a.d, device=dev, generator=gen).to(bf)
    V = torch.randn(case.B_R, L, a.d, device=dev, generator=gen).to(bf)
    off = torch.zeros(case.B_R + 1, dtype=torch.int32, device=dev)
    off[1:] = counts.cumsum(0).to(torch.int32)
    mq = torch.repeat_interleave(torch.arange(case.B_R, device=dev), counts)
    O = torch.empty(Bc, a.d, device=dev)
    O3 = torch.empty(Bc, a.d, device=dev, dtype=bf)
    scale = 1.0 / math.sqrt(dh)
    chunk = 2048

    def rocs_x():
        R.rocs_dca_cross_attn(Q, K, V, off, case.B_R, Bc, L, H, dh, scale, O, a.d, rocs.ROCS_F32, sh)

    def b3():
        for c0 in range(0, Bc, chunk):
            idx = mq[c0:c0 + chunk]
            kc = K.index_select(0, idx).view(-1, L, H, dh).transpose(1, 2)     # [c, H, L, dh] copy per candidate
            vc = V.index_select(0, idx).view(-1, L, H, dh).transpose(1, 2)
            q = Q[c0:c0 + chunk].view(-1, H, 1, dh)
            O3[c0:c0 + chunk] = F.scaled_dot_product_attention(q, kc, vc).reshape(-1, a.d)

    t_x = _timed_median(rocs_x, 5, 3, flush, dev)
    t_3 = _timed_median(b3, 2, 1, flush, dev)
    out["dca_cross_attn_depth0"] = {
        "candidates": Bc, "L": L, "heads": H, "rocs_dca_cross_attn_ms": round(t_x, 4),
        "B3_kv_copied_per_candidate_sdpa_ms": round(t_3, 3), "speedup_vs_B3": round(t_3 / t_x, 1),
        "B3_chunk": chunk, "max_abs_diff_vs_B3": round(float((O - O3.float()).abs().max()), 4)}
    if R.rocs_get_device_status(sh) != 0:
        raise RuntimeError("device status set in the baselines")
    del Q, K, V, O, O3
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------------------------
# reference arm: the float64 oracle on the host
# ---------------------------------------------------------------------------------------------
def run_reference(args, rank, world):
    if rank != 0:
        return
    case = make_case(args.workload, 0, args.requests)
    per_step = max(1.0, args.ref_step_seconds)
    for i in range(args.warmup):
        oracle_rate(case, per_step, start_req=i)
    t = 0.0
    n = 0
    for i in range(args.steps):
        rate, c, reqs, dt = oracle_rate(case, per_step, start_req=args.warmup + i)
        t += dt
        n += c
    value = n / t
    line = {"metric": METRIC, "value": round(value, 2), "unit": "candidates/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * t / args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "description": WORKLOADS[args.workload]},
            "cpu_baseline": {"value": round(value, 2), "unit": "candidates/s", "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": f"each step: whole requests of the workload for ~{per_step:.0f} s"},
            "e2e": {"value": round(value, 2), "unit": "candidates/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# IKBO linear sweep with materialised-broadcast baselines
# ---------------------------------------------------------------------------------------------
def run_ikbo_sweep(args, rank, world, local):
    """Each (N, d) point: rocs_linear_ikbo (bf16 in/out, ReLU), B1 = Z = X^R W_CR^T, Z[m] written
    out and added to X^C W_CC^T (torch/cuBLAS), B2 = [X^R[m], X^C] gathered and one K=2d GEMM
    (torch/cuBLAS).  Each repetition is timed alone with CUDA events after an L2 flush (a 256 MB
    write); the median is reported.  Inputs: the seeded synth draws of each point (X ~ N(0,1),
    W ~ N(0, 1/fan_in), b ~ U(-0.1, 0.1), bf16), the same values tests/test_gpu_ops.py checks
    against the oracle at every point (rank r > 0 shifts the seed by 1000 r)."""
    import torch
    from request_candidate_sharing_b200 import rocs
    dev = torch.device("cuda", local)
    R = rocs.Rocs(local)
    R.rocs_set_ikbo_fused(args.ikbo_fused)
    peaks = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    B_R = 256
    reps = max(args.steps, 3)
    points = []

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        ts.sort()
        return ts[len(ts) // 2]

    only = tuple(int(v) for v in args.sweep_point.split(",")) if args.sweep_point else None
    for N in (64, 256, 1024):
        for d in (512, 1024, 4096):
            if only is not None and (N, d) != only:
                continue
            # the seeded inputs the parity test checks against the oracle at this point
            case = dataclasses.replace(synth.linear_cfg2(N, d, B_R), seed=synth.linear_cfg2(N, d, B_R).seed + 1000 * rank)
            x = synth.linear_inputs(case, cand_rows=np.zeros(0, np.int64))
            B_C = B_R * N
            bf = torch.bfloat16
            up = lambda v, dt=bf: torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(dev).to(dt)
            XR, W_RR, W_CR, W_CC = (up(x[k]) for k in ("X_R", "W_RR", "W_CR", "W_CC"))
            bR, bC = up(x["b_R"], torch.float32), up(x["b_C"], torch.float32)
            XC = torch.empty(B_C, d, dtype=bf, device=dev)
            for r0, blk in synth.normal_blocks(case.seed, "X_C", (B_C, d)):
                XC[r0:r0 + len(blk)].copy_(torch.from_numpy(synth.bf16_round(blk)).to(bf))
            m = torch.arange(B_R, device=dev, dtype=torch.int32).repeat_interleave(N)
            YR = torch.empty(B_R, d, dtype=bf, device=dev)
            YC = torch.empty(B_C, d, dtype=bf, device=dev)
            desc = rocs.IkboDesc(B_R, B_C, d, d, d, d, rocs.ROCS_BF16, rocs.ROCS_BF16, rocs.ACT["relu"])
            nb = R.rocs_linear_ikbo_workspace(desc)
            ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
            sh = torch.cuda.current_stream(dev).cuda_stream

            def ikbo():
                R.rocs_linear_ikbo(desc, XR, XC, m, W_RR, W_CR, W_CC, bR, bC, YR, YC, ws, nb, sh)

            mi = m.long()

            def b1():
                z = torch.addmm(bC, XR.float(), W_CR.float().t()).to(bf)   # request partial (bias folded)
                zm = z.index_select(0, mi)                                  # materialised broadcast [B_C, d]
                torch.relu_(torch.addmm(zm, XC, W_CC.t()))
                torch.relu_(torch.addmm(bR.to(bf), XR, W_RR.t()))

            W2 = torch.cat([W_CR, W_CC], 1)                                 # [d, 2d]

            def b2():
                xg = torch.cat([XR.index_select(0, mi), XC], 1)            # gathered rows [B_C, 2d]
                torch.relu_(torch.addmm(bC.to(bf), xg, W2.t()))
                torch.relu_(torch.addmm(bR.to(bf), XR, W_RR.t()))

            ms_i, ms_1, ms_2 = timed(ikbo), timed(b1), timed(b2)
            st = R.rocs_get_device_status(sh)
            if st != 0:
                raise RuntimeError(f"device status {st} at N={N} d={d}")
            # the timed outputs against an fp32 evaluation of B2 (the gathered operands), in row
            # blocks: the largest absolute difference, beside the largest output (a bf16 output
            # is within half an ulp of its value, 2^-9 relative, plus accumulation order)
            diff, ymax = 0.0, 0.0
            for r0 in range(0, B_C, 8192):
                r1 = min(B_C, r0 + 8192)
                xg = torch.cat([XR.index_select(0, mi[r0:r1]), XC[r0:r1]], 1)
                ref = torch.relu(torch.addmm(bC, xg.float(), W2.float().t()))
                diff = max(diff, float((YC[r0:r1].float() - ref).abs().max()))
                ymax = max(ymax, float(ref.abs().max()))
            ref = torch.relu(torch.addmm(bR, XR.float(), W_RR.float().t()))
            diff = max(diff, float((YR.float() - ref).abs().max()))
            ymax = max(ymax, float(ref.abs().max()))
            flops = 2.0 * B_C * d * d + 2.0 * B_R * d * d * 2
            tf = flops / (ms_i / 1e3) / 1e12
            points.append({"N": N, "d": d, "B_C": B_C, "ikbo_ms": round(ms_i, 4),
                           "ikbo_cands_per_s": round(B_C / (ms_i / 1e3), 1),
                           "ikbo_tflops": round(tf, 2), "ikbo_frac_of_bf16_peak": round(tf / peaks["tensor"], 4),
                           "b1_materialised_Zm_ms": round(ms_1, 4), "b2_gathered_2d_gemm_ms": round(ms_2, 4),
                           "speedup_vs_b1": round(ms_1 / ms_i, 3), "speedup_vs_b2": round(ms_2 / ms_i, 3),
                           "max_abs_diff_vs_fp32_b2": round(diff, 5), "max_abs_output": round(ymax, 3)})
            del XR, XC, W_RR, W_CR, W_CC, YR, YC, ws, W2
            torch.cuda.empty_cache()
    head = next((p for p in points if p["N"] == 1024 and p["d"] == 1024), points[-1])
    if rank == 0:
        line = {"metric": METRIC, "value": head["ikbo_cands_per_s"], "unit": "candidates/s", "n_gpus": world,
                "steps": reps, "warmup": args.warmup, "ms_per_step": head["ikbo_ms"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded synth draws, the inputs of the per-point parity test)",
                "config": {"workload": "ikbo_sweep", "description": WORKLOADS["ikbo_sweep"],
                           "headline_point": f"N={head['N']}, d={head['d']}",
                           "l2": "flushed (256 MB write) before every repetition",
                           "peak_source": peaks["source"] + " (of measured, burst: each GEMM timed alone)"},
                "points": points}
        print(json.dumps(line), flush=True)
    R.close()


def run_w8a16(args, rank, world, local):
    """Per configuration (B_R, N, d_in, d_out): rocs_linear_ikbo with bf16 weights and
    rocs_linear_ikbo_w8 with per-channel E4M3 weights (quantised by rocs_quantize_weights_fp8),
    bf16 activations and outputs, GELU.  Each repetition is timed alone with CUDA events after an L2
    flush (a 256 MB write), so the weights come from HBM as in a model whose other layers evict
    them; medians.  Inputs: torch normal draws on the device."""
    import torch
    from request_candidate_sharing_b200 import rocs
    dev = torch.device("cuda", local)
    R = rocs.Rocs(local)
    peaks = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    reps = max(args.steps, 3)
    sh = torch.cuda.current_stream(dev).cuda_stream

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        ts.sort()
        return ts[len(ts) // 2]

    points = []
    only = tuple(int(v) for v in args.sweep_point.split(",")) if args.sweep_point else None
    for (B_R, N, di, do) in ((1, 16, 1280, 2560), (1, 16, 1280, 640), (1, 8, 1280, 2560), (1, 8, 1280, 640),
                             (1, 16, 8192, 8192), (4, 16, 4096, 16384)):
        if only is not None and (B_R, N, di, do) != only:
            continue
        B_C = B_R * N
        g = torch.Generator(device=dev).manual_seed(di + do + N)
        bf = torch.bfloat16
        XR = torch.randn(B_R, di, device=dev, generator=g).to(bf)
        XC = torch.randn(B_C, di, device=dev, generator=g).to(bf)
        Ws = [torch.randn(do, di, device=dev, generator=g).mul_(di ** -0.5).to(bf) for _ in range(3)]
        bR = torch.rand(do, device=dev, generator=g) * 0.2 - 0.1
        bC = torch.rand(do, device=dev, generator=g) * 0.2 - 0.1
        m = torch.arange(B_R, device=dev, dtype=torch.int32).repeat_interleave(N)
        Q = [torch.empty(do, di, dtype=torch.uint8, device=dev) for _ in range(3)]
        S = [torch.empty(do, dtype=torch.float32, device=dev) for _ in range(3)]
        for i in range(3):
            R.rocs_quantize_weights_fp8(Ws[i], rocs.ROCS_BF16, do, di, Q[i], S[i], sh)
        desc = rocs.IkboDesc(B_R, B_C, di, di, do, do, rocs.ROCS_BF16, rocs.ROCS_BF16, rocs.ACT["gelu"])
        nb = R.rocs_linear_ikbo_workspace(desc)
        nb8 = R.rocs_linear_ikbo_w8_workspace(desc)
        ws = torch.empty(max(nb, nb8, 16), dtype=torch.uint8, device=dev)
        YR = torch.empty(B_R, do, dtype=bf, device=dev)
        YC = torch.empty(B_C, do, dtype=bf, device=dev)
        ms_b = timed(lambda: R.rocs_linear_ikbo(desc, XR, XC, m, Ws[0], Ws[1], Ws[2], bR, bC, YR, YC, ws, nb, sh))
        YC_b = YC.float().clone()
        ms_8 = timed(lambda: R.rocs_linear_ikbo_w8(desc, XR, XC, m, Q[0], Q[1], Q[2], S[0], S[1], S[2], bR, bC, YR, YC,
                                                    ws, nb8, sh))
        # the opt-in path: FP8 operands converted in shared memory for the tcgen05 MMAs
        R.rocs_set_w8_tensor_cores(1)
        nbt = R.rocs_linear_ikbo_w8_workspace(desc)
        wst = torch.empty(max(nbt, 16), dtype=torch.uint8, device=dev)
        YC_t = torch.empty_like(YC)
        ms_t = timed(lambda: R.rocs_linear_ikbo_w8(desc, XR, XC, m, Q[0], Q[1], Q[2], S[0], S[1], S[2], bR, bC, YR, YC_t,
                                                    wst, nbt, sh))
        R.rocs_set_w8_tensor_cores(0)
        if R.rocs_get_device_status(sh) != 0:
            raise RuntimeError("device status set")
        # per-kernel times of both calls (direct launches, per-launch CUDA events, L2 flushed)
        kern = {}
        for name, fn in (("bf16", lambda: R.rocs_linear_ikbo(desc, XR, XC, m, Ws[0], Ws[1], Ws[2], bR, bC, YR, YC, ws, nb,
                                                            sh)),
                         ("fp8", lambda: R.rocs_linear_ikbo_w8(desc, XR, XC, m, Q[0], Q[1], Q[2], S[0], S[1], S[2], bR,
                                                               bC, YR, YC, ws, nb8, sh))):
            R.rocs_timing_start(256)
            for _ in range(reps):
                flush.fill_(1)
                fn()
            kern[name] = {k: round(t / reps, 4) for k, (n_, t) in R.rocs_timing_stop().items()}
        rel = float((YC.float() - YC_b).norm() / YC_b.norm())
        wbytes8 = 3.0 * do * di + 3 * do * 4
        act_bytes = (B_R + B_C) * di * 2.0 + (B_R + B_C) * do * 2.0
        gbs = (wbytes8 + act_bytes) / (ms_8 / 1e3) / 1e9
        points.append({"B_R": B_R, "N": N, "d_in": di, "d_out": do, "bf16_weights_ms": round(ms_b, 4),
                       "fp8_weights_ms": round(ms_8, 4), "latency_change": round(ms_8 / ms_b - 1.0, 4),
                       "fp8_tensor_core_path_ms": round(ms_t, 4),
                       "tensor_core_path_max_abs_diff": round(float((YC_t.float() - YC.float()).abs().max()), 5),
                       "fp8_GBps": round(gbs, 1), "fp8_frac_of_hbm": round(gbs / peaks["hbm"], 4),
                       "rel_l2_vs_bf16_weights": round(rel, 5), "kernel_ms": kern})
        del XR, XC, Ws, Q, S, ws, YR, YC, wst, YC_t
        torch.cuda.empty_cache()
    if rank == 0:
        head = points[0]
        line = {"metric": METRIC, "value": round(head["N"] * head["B_R"] / (head["fp8_weights_ms"] / 1e3), 1),
                "unit": "candidates/s", "n_gpus": world, "steps": reps, "warmup": args.warmup,
                "ms_per_step": head["fp8_weights_ms"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16 activations, e4m3 weights",
                "data": "synthetic (torch normal draws on the device)",
                "config": {"workload": "w8a16", "description": WORKLOADS["w8a16"],
                           "l2": "flushed (256 MB write) before every repetition",
                           "peak_source": peaks["source"] + " (of measured)"},
                "points": points}
        print(json.dumps(line), flush=True)
    R.close()


def run_xattn_unsorted(args, rank, world, local):
    """The grouped cross-attention (rocs_dca_cross_attn) and the same rows shuffled, each with its
    request index (rocs_dca_cross_attn_unsorted: sort, gather, attention, scatter), plus the sort
    alone (rocs_sort_by_request).  Each repetition is timed alone with CUDA events after an L2
    flush; medians.  Inputs: the forward workload's counts (seed 1 + 1000 x rank), bf16 normal Q,
    K, V drawn on the device, fp32 output."""
    import torch
    from request_candidate_sharing_b200 import rocs
    import synth
    dev = torch.device("cuda", local)
    R = rocs.Rocs(local)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    reps = max(args.steps, 3)
    counts = synth.counts_lognormal(1 + 1000 * rank, 512, 300.0, 1.0, 16, 2000)
    B_R, L, H, dh = len(counts), 1024, 8, 32
    d = H * dh
    B_C = int(counts.sum())
    g = torch.Generator(device=dev).manual_seed(7 + rank)
    bf = torch.bfloat16
    Q = torch.randn(B_C, d, device=dev, generator=g).to(bf)
    K = torch.randn(B_R * L, d, device=dev, generator=g).to(bf)
    V = torch.randn(B_R * L, d, device=dev, generator=g).to(bf)
    off = torch.zeros(B_R + 1, dtype=torch.int32, device=dev)
    off[1:] = torch.from_numpy(counts).to(dev).cumsum(0)
    m = torch.repeat_interleave(torch.arange(B_R, device=dev, dtype=torch.int32), torch.from_numpy(counts).to(dev).long())
    order = torch.randperm(B_C, device=dev, generator=g)
    Qs, ms = Q[order].contiguous(), m[order].contiguous()
    O = torch.empty(B_C, d, device=dev)
    Ou = torch.empty(B_C, d, device=dev)
    scale = 1.0 / math.sqrt(dh)
    sh = torch.cuda.current_stream(dev).cuda_stream
    nb = R.rocs_dca_cross_attn_unsorted_workspace(B_R, B_C, H, dh, rocs.ROCS_F32)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)
    nbs = R.rocs_sort_by_request_workspace(B_R, B_C)
    wss = torch.empty(max(nbs, 16), dtype=torch.uint8, device=dev)
    perm = torch.empty(B_C, dtype=torch.int32, device=dev)
    offs = torch.empty(B_R + 1, dtype=torch.int32, device=dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        ts.sort()
        return ts[len(ts) // 2]

    ms_g = timed(lambda: R.rocs_dca_cross_attn(Q, K, V, off, B_R, B_C, L, H, dh, scale, O, d, rocs.ROCS_F32, sh))
    ms_u = timed(lambda: R.rocs_dca_cross_attn_unsorted(Qs, K, V, ms, B_R, B_C, L, H, dh, scale, Ou, d, rocs.ROCS_F32,
                                                        ws, nb, sh))
    ms_s = timed(lambda: R.rocs_sort_by_request(ms, B_R, B_C, perm, offs, wss, nbs, sh))
    if R.rocs_get_device_status(sh) != 0:
        raise RuntimeError("device status set")
    same = bool(torch.equal(Ou, O[order]))
    # per-kernel times of the unsorted call (direct launches, per-launch CUDA events)
    R.rocs_timing_start(64)
    for _ in range(reps):
        flush.fill_(1)
        R.rocs_dca_cross_attn_unsorted(Qs, K, V, ms, B_R, B_C, L, H, dh, scale, Ou, d, rocs.ROCS_F32, ws, nb, sh)
    kern = {k: round(t / reps, 4) for k, (n, t) in R.rocs_timing_stop().items()}
    if rank == 0:
        line = {"metric": METRIC, "value": round(B_C / (ms_u / 1e3), 1), "unit": "candidates/s", "n_gpus": world,
                "steps": reps, "warmup": args.warmup, "ms_per_step": round(ms_u, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded counts; torch normal Q/K/V drawn on the device)",
                "config": {"workload": "xattn_unsorted", "description": WORKLOADS["xattn_unsorted"], "B_R": B_R,
                           "B_C": B_C, "l2": "flushed (256 MB write) before every repetition"},
                "grouped_ms": round(ms_g, 4), "unsorted_ms": round(ms_u, 4), "sort_ms": round(ms_s, 4),
                "unsorted_overhead": round(ms_u / ms_g - 1.0, 4),
                "sort_cands_per_s": round(B_C / (ms_s / 1e3), 1),
                "unsorted_equals_grouped": same, "unsorted_kernel_ms": kern}
        print(json.dumps(line), flush=True)
    R.close()


def run_ex2_rate(args, rank, world, local):
    """The attention softmax's exponential throughput on this GPU (rocs_probe_exp2_rate) for every
    split of the exponentials between MUFU ex2 and the FMA-pipe polynomial (n_poly of every eight
    pairs on the polynomial), with the SM clock sampled during the measurement."""
    import torch
    from request_candidate_sharing_b200 import rocs
    torch.cuda.set_device(local)
    R = rocs.Rocs(local)
    sh = torch.cuda.current_stream(local).cuda_stream
    uuid = str(getattr(torch.cuda.get_device_properties(local), "uuid", "") or "")
    clocks = ClockSampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else (uuid or str(local)))
    for n in range(9):       # warm-up: clocks up
        R.rocs_probe_exp2_rate(n, sh)
    clocks.start()
    time.sleep(0.3)
    rates = {}
    for _ in range(max(1, args.steps // 3)):
        for n in range(9):
            rates[n] = max(rates.get(n, 0.0), R.rocs_probe_exp2_rate(n, sh))
    clk = clocks.stop()
    R.close()
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    mhz = (clk or {}).get("sm_mhz") or 1965.0
    per_clk = {f"n_poly={n}": round(r / (sms * mhz * 1e6), 2) for n, r in rates.items()}
    best = max(rates, key=rates.get)
    if rank == 0:
        print(json.dumps({"metric": "exponentials/s of the attention softmax's per-score steps", "value": round(rates[3], 1),
                          "unit": "exp2/s", "n_gpus": 1, "steps": args.steps, "warmup": 9, "higher_is_better": True,
                          "dtype": "f32", "data": "synthetic", "impl": "librocs",
                          "config": {"workload": "ex2_rate", "description": WORKLOADS["ex2_rate"],
                                     "headline": "n_poly=3, the attention kernels' split"},
                          "rates_exp2_per_s": {f"n_poly={n}": round(r, 1) for n, r in rates.items()},
                          "per_clock_per_sm": per_clk, "best_split": f"n_poly={best}", "sms": sms,
                          "clocks": clk}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="rocs_forward_e2e", choices=sorted(WORKLOADS))
    ap.add_argument("--shard", default="own", choices=["own", "lpt"],
                    help="N > 1: each rank its own batch (weak scaling, the default) or the LPT "
                         "partition of one batch (strong scaling)")
    ap.add_argument("--impl", default="librocs", choices=["librocs", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-baselines", action="store_true", help="skip the GPU materialised-broadcast baselines")
    ap.add_argument("--requests", type=int, default=0, help="keep only the first N requests (profiling runs)")
    ap.add_argument("--sweep-point", default="", help="ikbo_sweep: run only the point 'N,d'; w8a16: only "
                                                      "'B_R,N,d_in,d_out' (profiling runs)")
    ap.add_argument("--ikbo-fused", type=int, default=1, choices=[0, 1],
                    help="IKBO linears as one fused launch (1, the library default) or two launches (0)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "librocs":
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, rank, world)
        return
    rank, world, local = dist_setup(args.gpus)
    if args.workload == "ikbo_sweep":
        run_ikbo_sweep(args, rank, world, local)
    elif args.workload == "xattn_unsorted":
        run_xattn_unsorted(args, rank, world, local)
    elif args.workload == "w8a16":
        run_w8a16(args, rank, world, local)
    elif args.workload == "ex2_rate":
        run_ex2_rate(args, rank, world, local)
    else:
        run_librocs(args, rank, world, local)


if __name__ == "__main__":
    main()
