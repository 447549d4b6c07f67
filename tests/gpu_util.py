"""Helpers shared by the GPU parity tests: device upload of the seeded host inputs, read-back,
the tolerance checks and the seeded candidate sampling."""
from __future__ import annotations

import numpy as np
import torch

from oracle import rocs_oracle as O

# Tolerances.  fp32 path: max relative error 1e-4, per element relative to max(|ref|, 0.1 rms).
# bf16-in / fp32-accumulate path: relative L2 <= 5e-3 and max abs <= 2e-2 on unit-scale outputs;
# a bf16-rounded output may add its half-ulp (2^-8 |ref|) on top of the max-abs bound.
FP32_REL = 1e-4
BF16_REL_L2 = 5e-3
BF16_MAX_ABS = 2e-2


def dev(x: np.ndarray, dtype=torch.bfloat16) -> torch.Tensor:
    """Upload host values (already representable in `dtype`) to cuda:0."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(dtype).contiguous()


def dev_i32(x) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to("cuda")


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def stream():
    return torch.cuda.current_stream().cuda_stream


def check_fp32(got, ref, rel=FP32_REL, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    denom = np.maximum(np.abs(ref), 0.1 * rms + 1e-30)
    err = float(np.max(np.abs(got - ref) / denom)) if ref.size else 0.0
    assert err <= rel, f"{what}: max relative error {err:.3e} > {rel:.1e}"
    return err


def check_bf16(got, ref, out_bf16=False, what="", rel_l2=BF16_REL_L2, max_abs=BF16_MAX_ABS):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    if ref.size == 0:
        return 0.0, 0.0
    l2 = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    bound = max_abs + (2.0 ** -8) * np.abs(ref) if out_bf16 else max_abs
    excess = np.abs(got - ref) - bound
    worst = float(np.max(np.abs(got - ref)))
    assert l2 <= rel_l2, f"{what}: relative L2 {l2:.3e} > {rel_l2:.1e}"
    assert float(np.max(excess)) <= 0.0, f"{what}: max abs error {worst:.3e} beyond bound"
    return l2, worst


def sample_candidates(counts, per_request: int, seed: int = 123) -> np.ndarray:
    """Sorted candidate positions: up to `per_request` per request, always each non-empty
    request's first and last candidate."""
    offsets, _ = O.segments(counts)
    g = np.random.default_rng(seed)
    picks = []
    for r, n in enumerate(np.asarray(counts).tolist()):
        if n == 0:
            continue
        base = int(offsets[r])
        idx = {0, n - 1}
        extra = max(0, min(per_request, n) - len(idx))
        if extra:
            idx.update(g.choice(n, size=min(n, extra + 2), replace=False).tolist())
        picks.extend(base + i for i in sorted(idx)[:max(per_request, 2)])
    return np.asarray(sorted(set(picks)), dtype=np.int64)


def dev_normal_bf16(seed: int, name: str, shape, std: float = 1.0, keep_rows=None):
    """The seeded N(0, std^2) tensor `synth.normal(seed, name, shape, std)` rounded to bf16, built
    on cuda:0 one row block at a time (the full-size candidate batches are several GB).  With
    `keep_rows` (sorted row indices) it also returns those rows' host values, taken from the same
    blocks as they pass."""
    import synth
    out = torch.empty(tuple(shape), dtype=torch.bfloat16, device="cuda")
    keep = None if keep_rows is None else np.asarray(keep_rows, np.int64)
    kept = None if keep is None else np.empty((len(keep),) + tuple(shape[1:]), np.float32)
    for r0, blk in synth.normal_blocks(seed, name, shape, std):
        blk = synth.bf16_round(blk)
        out[r0:r0 + len(blk)].copy_(torch.from_numpy(blk).to(torch.bfloat16))
        if keep is not None:
            sel = np.flatnonzero((keep >= r0) & (keep < r0 + len(blk)))
            kept[sel] = blk[keep[sel] - r0]
    return out if keep is None else (out, kept)
