"""Parity checks of a GPU result against the oracle, used by every GPU parity test.

One global relative L2 error (the per-block bound of 2e-2) hides localized bugs: at the
8352-token joint sequence one completely wrong token row adds only sqrt(1/8352) = 1.1%
to it.  So besides the global figure every result is checked per row and per element:

* global:  ||got - ref|| / ||ref|| <= tol.
* per row (a row = one token, the last axis):  ||got_i - ref_i|| / max(||ref_i||,
  0.1 median_j ||ref_j||) <= row_tol (tol unless given).  The floor keeps a row whose
  reference is near zero from turning rounding noise into a large ratio.
* per element:  |got_ij - ref_ij| <= rtol (8 rms_i + |ref_ij|), rms_i the row's RMS
  (floored like the row norm).  Each bf16 rounding on the path (operand or stored
  value; unit roundoff u = 2^-8, bf16 keeping 8 significant bits) perturbs an output
  element by a relative error of at most u of the terms it sums, whose scale is the
  row's RMS, not the element's own value (an element near zero by cancellation still
  carries errors of the row's scale); with n roundings the error's standard deviation
  is about u sqrt(n / 3) rms_i, so rtol = u sqrt(n) puts the bound at 8 sqrt(3) = 13.9
  standard deviations, beyond the largest of 10^9 Gaussian draws (~6.1), while a wrong
  element (error of the row's scale) exceeds it whenever 8 u sqrt(n) < 1.

With `base` (the input of a residual update x_out = base + update) the global check is
applied to the output and to the update, and the row and element checks to the update:
the output is dominated by the unchanged input and would hide errors in the update.

Plain NumPy: the tests of this file's checks run without a GPU.
"""
from __future__ import annotations

import numpy as np

U_BF16 = 2.0 ** -8


class ParityError(AssertionError):
    pass


def parity_metrics(got, ref, n_round: int = 10, rtol: float | None = None):
    """Error figures of got vs ref: global rel-L2, mean / median / max |diff|, the worst
    row ratio and the worst element ratio (|diff| over the element bound; <= 1 passes)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if got.shape != ref.shape:
        raise ParityError(f"shape {got.shape} != {ref.shape}")
    if not np.all(np.isfinite(got)):
        raise ParityError("non-finite values in the result")
    n = ref.shape[-1] if ref.ndim else 1
    g2 = got.reshape(-1, n)
    r2 = ref.reshape(-1, n)
    diff = g2 - r2
    ad = np.abs(diff)
    row_norm = np.linalg.norm(r2, axis=1)
    floor = 0.1 * float(np.median(row_norm))
    row_den = np.maximum(row_norm, max(floor, 1e-300))
    row_rel = np.linalg.norm(diff, axis=1) / row_den
    rms = row_den / np.sqrt(n)
    rt = U_BF16 * np.sqrt(n_round) if rtol is None else rtol
    bound = rt * (8.0 * rms[:, None] + np.abs(r2))
    elem_ratio = ad / np.maximum(bound, 1e-300)
    worst = np.unravel_index(int(np.argmax(elem_ratio)), elem_ratio.shape)
    return {
        "rel_l2": float(np.linalg.norm(diff) / max(np.linalg.norm(r2), 1e-300)),
        "mean_abs": float(ad.mean()), "median_abs": float(np.median(ad)), "max_abs": float(ad.max()),
        "worst_row": int(np.argmax(row_rel)), "worst_row_rel": float(row_rel.max()),
        "worst_elem": (int(worst[0]), int(worst[1])), "worst_elem_ratio": float(elem_ratio[worst]),
        "rows": int(r2.shape[0]),
    }


def assert_parity(got, ref, tol: float, base=None, n_round: int = 10, rtol: float | None = None,
                  row_tol: float | None = None, label: str = ""):
    """Raises ParityError unless got matches ref globally, per row and per element (see the
    module docstring).  Returns the metrics of the checked quantity (the update if `base`)."""
    row_tol = tol if row_tol is None else row_tol
    out = None
    if base is not None:
        base = np.asarray(base, np.float64)
        out = parity_metrics(got, ref, n_round, rtol)
        got = np.asarray(got, np.float64) - base
        ref = np.asarray(ref, np.float64) - base
    m = parity_metrics(got, ref, n_round, rtol)
    what = "update" if base is not None else "output"
    print(f"\n{label} {what}: rel-L2 {m['rel_l2']:.3e}, mean |d| {m['mean_abs']:.3e}, median |d| "
          f"{m['median_abs']:.3e}, max |d| {m['max_abs']:.3e}, worst row {m['worst_row']} "
          f"rel {m['worst_row_rel']:.3e}, worst element {m['worst_elem']} at {m['worst_elem_ratio']:.3f} "
          f"of its bound ({m['rows']} rows)" + (f"; output rel-L2 {out['rel_l2']:.3e}" if out else ""))
    if out is not None and out["rel_l2"] > tol:
        raise ParityError(f"{label}: output rel-L2 {out['rel_l2']:.3e} > {tol}")
    if m["rel_l2"] > tol:
        raise ParityError(f"{label}: {what} rel-L2 {m['rel_l2']:.3e} > {tol}")
    if m["worst_row_rel"] > row_tol:
        raise ParityError(f"{label}: {what} row {m['worst_row']} rel-L2 {m['worst_row_rel']:.3e} > {row_tol}")
    if m["worst_elem_ratio"] > 1.0:
        raise ParityError(f"{label}: {what} element {m['worst_elem']} is {m['worst_elem_ratio']:.2f}x its bound")
    return m
