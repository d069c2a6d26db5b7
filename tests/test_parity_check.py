"""The GPU parity tests' output comparison (tests/parity_check.py) on
constructed arrays: it accepts exact agreement, a one-ulp rounding flip next to
a rounding midpoint and a P~-code move within the oracle's own bound, and
rejects everything else beyond 2e-3.  CPU only."""
import numpy as np
import pytest
import torch

from parity_check import compare_out


def _f16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).half().float().numpy()


def test_identical_passes_and_offset_fails():
    rng = np.random.default_rng(0)
    ref32 = rng.standard_normal((2, 40, 64)).astype(np.float32)
    got = _f16(ref32)
    st = compare_out(got, ref32, np.zeros_like(ref32), "fp16")
    assert st["over_2e3"] == 0
    bad = got.copy()
    bad[1, 3, 7] += 5e-3
    with pytest.raises(AssertionError):
        compare_out(bad, ref32, np.zeros_like(ref32), "fp16")


def test_p_code_move_within_bound_passes_and_counts_rows():
    ref32 = np.full((1, 200, 16), 0.25, np.float32)
    flip = np.zeros_like(ref32)
    got = _f16(ref32)
    got[0, 5, :] += 4e-3          # one row moved by a P~ code
    flip[0, 5, :] = 3e-3           # the oracle says one code moves it by up to 3e-3
    st = compare_out(got, ref32, flip, "fp16")
    assert st["p_code_rows"] == 1 and st["p_code"] == 16
    # beyond the bound: rejected
    got2 = got.copy()
    got2[0, 6, 0] += 6e-3
    flip2 = flip.copy()
    flip2[0, 6, 0] = 3e-3
    with pytest.raises(AssertionError):
        compare_out(got2, ref32, flip2, "fp16")
    # within the bound but in too many rows (more than 2 % of 200 = 4 rows): rejected
    got3 = _f16(ref32)
    flip3 = np.zeros_like(ref32)
    got3[0, :5, 0] += 4e-3
    flip3[0, :5, 0] = 3e-3
    with pytest.raises(AssertionError):
        compare_out(got3, ref32, flip3, "fp16")


def test_rounding_flip_only_next_to_a_midpoint():
    # bf16 spacing in [1, 2) is 2^-7: 1.5 and 1.5078125 are adjacent values
    lo, hi = 1.5, 1.5078125
    mid = 0.5 * (lo + hi)
    ref32 = np.full((1, 50, 64), lo, np.float32)
    got = ref32.copy()
    ref32[0, 0, 0] = mid - 1e-4                           # rounds to lo
    got[0, 0, 0] = hi                                     # the GPU's value rounded up
    st = compare_out(got, ref32, np.zeros_like(ref32), "bf16")
    assert st["boundary"] == 1
    ref32[0, 0, 0] = lo + 1e-3                            # far from the midpoint: rounds to lo
    with pytest.raises(AssertionError):
        compare_out(got, ref32, np.zeros_like(ref32), "bf16")
