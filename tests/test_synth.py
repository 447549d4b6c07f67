"""The seeded input generators that the oracle and the CUDA path share (synth/): a sampled subset
of rows regenerates exactly the rows of the whole draw, block-wise filling gives the same
tensor, bf16 rounding is round-to-nearest-even (checked against torch's conversion), and the
workloads' candidate counts stay what the measurements quote."""
import numpy as np
import pytest
import torch

import synth


def test_sampled_rows_equal_the_whole_draw():
    shape = (2 * synth.ROW_BLOCK + 452, 3, 5)
    full = synth.normal(7, "X_C", shape, std=0.5)
    rows = [0, 1, synth.ROW_BLOCK - 1, synth.ROW_BLOCK, 2 * synth.ROW_BLOCK - 1, 2 * synth.ROW_BLOCK, shape[0] - 1, 5]
    assert np.array_equal(synth.normal(7, "X_C", shape, std=0.5, rows=rows), full[rows])
    u = synth.uniform(7, "b", shape, -0.1, 0.1)
    assert np.array_equal(synth.uniform(7, "b", shape, -0.1, 0.1, rows=rows), u[rows])
    assert u.min() >= -0.1 and u.max() < 0.1


def test_block_filling_equals_the_whole_draw():
    shape = (synth.ROW_BLOCK + 17, 4)
    full = synth.normal(3, "E_C", shape)
    parts = list(synth.normal_blocks(3, "E_C", shape))
    assert [r0 for r0, _ in parts] == [0, synth.ROW_BLOCK]
    assert np.array_equal(np.concatenate([b for _, b in parts]), full)


def test_streams_are_independent_of_name_seed_and_block():
    a = synth.normal(0, "W_RR", (4, 8))
    assert not np.array_equal(a, synth.normal(0, "W_CR", (4, 8)))
    assert not np.array_equal(a, synth.normal(1, "W_RR", (4, 8)))
    two = synth.normal(0, "X", (2 * synth.ROW_BLOCK, 1))
    assert not np.array_equal(two[:8], two[synth.ROW_BLOCK:synth.ROW_BLOCK + 8])


def test_bf16_rounding_is_nearest_even():
    one = 1.0
    ulp = 2.0 ** -7
    x = np.array([one + ulp / 2,            # tie, to the even neighbour 1.0
                  one + ulp + ulp / 2,      # tie, to the even neighbour 1 + 2 ulp
                  one + ulp / 2 + 2 ** -20,  # just above the tie: up
                  -3.1415926, 65504.0, 1e-40, 3.0e38, -0.0], np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.bf16_bits(x), ref)
    assert synth.bf16_round(x)[0] == 1.0 and synth.bf16_round(x)[1] == one + 2 * ulp
    assert synth.bf16_bits(np.array([np.nan], np.float32))[0] == 0x7FC0
    r = synth.normal(11, "R", (1000,))
    assert np.array_equal(synth.bf16_round(r), torch.from_numpy(r).to(torch.bfloat16).float().numpy())


def test_workload_counts():
    # the end-to-end workload: 512 requests, clipped lognormal, seed 1 -> 242,464 candidates
    c5 = synth.counts_lognormal(1, 512, 300.0, 1.0, 16, 2000)
    assert c5.sum() == 242_464 and c5.min() >= 16 and c5.max() <= 2000
    c3 = synth.counts_uniform(0, 64, 100, 1000)
    assert c3.min() >= 100 and c3.max() <= 1000
    assert np.array_equal(c3, synth.counts_uniform(0, 64, 100, 1000))


@pytest.mark.parametrize("B_R", [1, 2, 9])
def test_history_lengths_cover_both_ends(B_R):
    h = synth.hist_lengths(5, B_R, 200, lo=3)
    assert h.min() >= 3 and h.max() <= 200
    if B_R >= 2:
        assert h[0] == 200 and h[1] == 3
