"""The output comparison of the GPU parity tests (CUDA path vs the CPU oracle).

Spec bounds: max-abs 2e-3 and relative L1 5e-4 against the oracle.  The
two sides evaluate the softmax exponential differently (the GPU on its
special-function unit, the oracle with the library exp2) and round the logits
in a different order, so a P~ code can land on the neighbouring code where
p * Pr sits within a few fp32 ulps of a rounding midpoint, and an output can
round to the neighbouring 16-bit value where it sits next to a rounding
boundary.  Elements beyond 2e-3 are accepted only for these two derived
reasons, and counted:

  boundary  the GPU value and the oracle's rounded value are adjacent 16-bit
            values, and the oracle's unrounded fp32 value lies within 2e-3 of
            the midpoint between them (an fp32 difference inside the bound
            moved the rounding);
  p_code    |gpu - oracle fp32| <= 2e-3 + F + half an output ulp, where F is the
            oracle's own figure for the element: the largest change that one
            P~ code (NVFP4: one P~ block) moved by one step would cause,
            step(P~_j) * |v_jc| * scale_v / (Pr * l) over the row's keys.
            A moved code shifts its whole output row, so the count is of
            rows: at most 2 % of the compared rows (at least 2) may hold such
            elements.

The relative L1 bound covers every element.
"""
import numpy as np
import torch

MAX_ABS, REL_L1 = 2e-3, 5e-4
P_CODE_ROW_SHARE = 0.02

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


def to_dtype_np(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(DTYPES[dtype]).float().numpy()


def _bits(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(DTYPES[dtype]).view(torch.int16).numpy().astype(
        np.int32)


def _half_ulp(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(np.abs(x), np.float32)).to(DTYPES[dtype])
    up = torch.nextafter(t, torch.full_like(t, float("inf")))
    return 0.5 * (up.float() - t.float()).numpy()


def compare_out(o_gpu, ref32, flip, dtype, label=""):
    """o_gpu: GPU output as float32 (values of `dtype`); ref32: the oracle's
    unrounded fp32 output; flip: the oracle's per-element P~ sensitivity F.
    Returns a dict of the counts; raises AssertionError on a violation."""
    a = np.asarray(o_gpu, np.float64)
    ref = to_dtype_np(ref32, dtype).astype(np.float64)
    y = np.asarray(ref32, np.float64)
    diff = np.abs(a - ref)
    over = diff > MAX_ABS
    adjacent = (np.abs(_bits(o_gpu, dtype) - _bits(ref, dtype)) == 1) & (np.sign(a) == np.sign(ref))
    boundary = over & adjacent & (np.abs(y - 0.5 * (a + ref)) <= MAX_ABS)
    rest = over & ~boundary
    p_bound = MAX_ABS + np.asarray(flip, np.float64) + _half_ulp(o_gpu, dtype)
    p_code = rest & (np.abs(a - y) <= p_bound)
    bad = rest & ~p_code
    rows = p_code.reshape(-1, p_code.shape[-1]).any(axis=1) if p_code.ndim else p_code
    n_rows = max(1, rows.size)
    n_p_allowed = max(2, int(np.ceil(P_CODE_ROW_SHARE * n_rows)))
    rel = float(diff.sum() / max(np.abs(ref).sum(), 1e-30))
    stats = dict(label=str(label), elements=int(diff.size), rows=int(n_rows),
                 max_abs=float(diff.max()) if diff.size else 0.0,
                 rel_l1=rel, over_2e3=int(over.sum()), boundary=int(boundary.sum()), p_code=int(p_code.sum()),
                 p_code_rows=int(rows.sum()),
                 p_code_max_abs=float(diff[p_code].max()) if p_code.any() else 0.0,
                 max_abs_plain=float(np.where(over, 0.0, diff).max()) if diff.size else 0.0)
    print("parity", stats)
    assert int(bad.sum()) == 0 and int(rows.sum()) <= n_p_allowed and rel <= REL_L1, (
        stats, "unexplained" if bad.any() else "", np.argwhere(bad)[:5].tolist(),
        float(diff[bad].max()) if bad.any() else 0.0)
    return stats
