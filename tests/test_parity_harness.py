"""The parity harness's bounds, on hand-made values (no GPU).

The harness compares bf16 outputs with the oracle's exact values: these
cases pin that a correctly rounded bf16 output passes everywhere (also for
elements so large that the bf16 spacing alone exceeds 2e-2 x RMS), that an
error of one spacing more fails, that an ordinary element off by more than
2e-2 x RMS fails, and that order-swapped combine weights are compared after
pairing by expert id.
"""
import numpy as np
import pytest
import torch

from parity import GRID_SLACK, MAX_ABS_RMS, bf16_errors, bf16_half_spacing, paired_weight_error


def _bf16(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).double().numpy()


def _pow2_above(v: float) -> float:
    return float(2.0 ** np.ceil(np.log2(v)))


def _case(seed=0, n=20000):
    rng = np.random.default_rng(seed)
    exact = rng.standard_normal(n)
    return exact


def test_correct_rounding_passes_and_is_not_grid_limited_below_five_rms():
    exact = _case()
    exact = exact / np.sqrt((exact ** 2).mean())          # RMS 1
    exact = np.clip(exact, -4.5, 4.5)
    got = _bf16(exact)
    rel, mx, over, grid, _ = bf16_errors(got, exact, got)
    assert over <= 1.0 and grid == 0
    assert mx <= MAX_ABS_RMS
    assert rel < 3e-3                                      # bf16 rounding alone


def test_large_element_rounded_correctly_passes_through_the_grid_allowance():
    exact = _case(1)
    rms = np.sqrt((exact ** 2).mean())
    # an element just above a power of two beyond 5.2 x RMS, 0.49 of a
    # spacing above it: its half spacing exceeds 2e-2 x RMS
    big = _pow2_above(5.2 * rms) * (1 + 0.49 * 2.0 ** -7)
    exact[7] = big
    rms = np.sqrt((exact ** 2).mean())
    assert bf16_half_spacing(np.array([big]))[0] > MAX_ABS_RMS * rms
    got = _bf16(exact)
    rel, mx, over, grid, _ = bf16_errors(got, exact, got)
    assert mx > MAX_ABS_RMS                                # the raw bound cannot hold here
    assert over <= 1.0 and grid >= 1


def test_one_spacing_too_far_on_a_large_element_fails():
    exact = _case(2)
    rms = np.sqrt((exact ** 2).mean())
    big = _pow2_above(5.2 * rms) * (1 + 0.25 * 2.0 ** -7)   # a quarter spacing above
    exact[3] = big
    got = _bf16(exact)
    got[3] += 2 * bf16_half_spacing(np.array([big]))[0]    # the far neighbour
    *_, over, grid, _ = bf16_errors(got, exact, _bf16(exact))
    assert over > 1.0


def test_ordinary_element_beyond_the_bound_fails():
    exact = _case(3)
    rms = np.sqrt((exact ** 2).mean())
    got = _bf16(exact)
    i = int(np.argmin(np.abs(exact - rms)))
    got[i] = exact[i] + 0.03 * rms
    rel, mx, over, grid, _ = bf16_errors(got, exact, _bf16(exact))
    assert over > 1.0 and mx >= 0.03 - 1e-12


def test_grid_allowance_is_the_half_spacing_plus_slack():
    exact = _case(4)
    rms = np.sqrt((exact ** 2).mean())
    big = _pow2_above(5.2 * rms) * (1 + 0.1 * 2.0 ** -7)
    exact[0] = big
    rms = np.sqrt((exact ** 2).mean())
    half = bf16_half_spacing(np.array([big]))[0]
    got = _bf16(exact)
    got[0] = big + half + 0.5 * GRID_SLACK * rms
    assert bf16_errors(got, exact, _bf16(exact))[2] <= 1.0
    got[0] = big + half + 2.0 * GRID_SLACK * rms
    assert bf16_errors(got, exact, _bf16(exact))[2] > 1.0


def test_swapped_slots_are_paired_by_expert():
    ig = np.array([[5, 3, 9], [1, 2, 0]])
    wg = np.array([[0.5, 0.3, 0.2], [0.6, 0.3, 0.1]])
    io = np.array([[3, 5, 9], [1, 2, 0]])
    wo = np.array([[0.3, 0.5, 0.2], [0.6, 0.3, 0.1]])
    assert paired_weight_error(ig, wg, io, wo) == 0.0
    wo_bad = wo.copy()
    wo_bad[0, 0] = 0.31
    assert paired_weight_error(ig, wg, io, wo_bad) == pytest.approx(0.01)
    with pytest.raises(AssertionError):
        paired_weight_error(ig, wg, np.array([[3, 5, 8], [1, 2, 0]]), wo)
