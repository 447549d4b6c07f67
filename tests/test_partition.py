"""rocs_partition_requests (host, no GPU): whole requests over parts by longest processing time
first.  Checked against an exhaustive search on small batches (the 4/3 bound of the method),
against the lower bound max(total / parts, largest request) on large ones, and for coverage,
determinism, tie order and argument checks."""
import itertools

import numpy as np
import pytest

from request_candidate_sharing_b200 import rocs


def _loads(counts, part, n, cr, cc):
    w = cr + cc * np.asarray(counts, np.float64)
    return np.array([w[part == p].sum() for p in range(n)])


@pytest.mark.parametrize("seed", range(40))
def test_within_four_thirds_of_the_best_split(seed):
    rng = np.random.default_rng(seed)
    B_R, n = int(rng.integers(2, 9)), int(rng.integers(2, 4))
    counts = rng.integers(0, 50, B_R).astype(np.int32)
    cr, cc = float(rng.choice([0.0, 1.0, 7.5])), float(rng.choice([0.5, 1.0]))
    part = rocs.partition_requests(counts, n, cr, cc)
    got = _loads(counts, part, n, cr, cc).max()
    w = cr + cc * counts.astype(np.float64)
    best = min(max(sum(w[i] for i in range(B_R) if a[i] == p) for p in range(n))
               for a in itertools.product(range(n), repeat=B_R))
    assert got <= best * (4 / 3 - 1 / (3 * n)) + 1e-9


@pytest.mark.parametrize("B_R,n", [(512, 2), (512, 8), (3000, 7), (5, 8)])
def test_large_batches_cover_every_request_and_balance(B_R, n):
    import synth
    counts = synth.counts_lognormal(1, B_R, 300.0, 1.0, 16, 2000)
    part = rocs.partition_requests(counts, n, 14.8, 0.0586)
    assert part.shape == (B_R,) and part.min() >= 0 and part.max() < n
    loads = _loads(counts, part, n, 14.8, 0.0586)
    w = 14.8 + 0.0586 * counts.astype(np.float64)
    lower = max(w.sum() / n, w.max())
    assert loads.max() <= lower * (4 / 3) + 1e-9
    assert np.array_equal(part, rocs.partition_requests(counts, n, 14.8, 0.0586))   # deterministic


def test_ties_go_in_index_order_to_the_lower_part():
    assert rocs.partition_requests([5, 5, 5, 5], 2, 0.0, 1.0).tolist() == [0, 1, 0, 1]
    # the heaviest request first, then the next heaviest to the emptier part
    assert rocs.partition_requests([1, 9, 4, 4], 2, 0.0, 1.0).tolist() == [1, 0, 1, 1]
    # with request work only, requests are dealt round robin
    assert rocs.partition_requests([0, 0, 0, 0, 0], 3, 2.0, 0.0).tolist() == [0, 1, 2, 0, 1]


@pytest.mark.parametrize("args", [([1, -1], 2, 1.0, 1.0), ([1, 2], 0, 1.0, 1.0), ([1, 2], 2, 0.0, 0.0),
                                  ([1, 2], 2, float("nan"), 1.0), ([1, 2], 2, -1.0, 1.0), ([], 2, 1.0, 1.0)])
def test_bad_arguments_are_refused(args):
    with pytest.raises(rocs.RocsError):
        rocs.partition_requests(*args)
