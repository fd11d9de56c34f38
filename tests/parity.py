"""Parity checks shared by the GPU tests: three bounds on one comparison.

For a GPU result ``got`` and the oracle's ``ref`` of the same shape, where the
last axis is one output row (the d channels of one query, or of one key for dk
and dv):

* pooled relative L2, ||got - ref||_F / ||ref||_F <= tol (the tolerance the
  method's accuracy contract states: 1e-4 on the fp32 path, 2e-2 on the bf16
  path);
* per row, max_t ||got_t - ref_t|| / ||ref_t|| <= row_tol, so that one wrong
  row cannot hide in the pooled figure (a single row whose error equals its own
  norm moves the pooled figure by only sqrt(1/rows)).  Gradients (GRAD_BOUNDS)
  take the row norm floored at the rms row norm: a gradient row can cancel to
  nearly nothing, and its relative error then measures rounding of the
  cancelling terms, not a wrong row;
* per element, |got - ref| <= atol + rtol |ref| with rtol = elem_tol and
  atol = elem_tol * rms(ref), the rms taken over the whole compared output, so
  that an element that is off by more than a few rounding steps of its own row
  fails even when its row's norm is dominated by other channels.

Rows whose reference norm is below 1e-6 of the rms row norm are left to the
element-wise bound (their relative error is not meaningful).

With the environment variable PISA_PARITY_LOG set to a file path, every
comparison appends one JSON line with the measured figures (test id, rel-L2,
worst row, worst element ratio) to it.
"""
from __future__ import annotations

import json
import os

import oracle

# Bounds per dtype: pooled rel-L2 (the contract), worst row, element ratio.  Measured on the
# B200 over every forward comparison of the GPU suite: worst row 6.2e-3 and worst element
# 1.4e-2 in bf16, 2.9e-6 and 1.2e-5 in fp32.
BOUNDS = {
    "f32": {"tol": 1e-4, "row_tol": 1e-4, "elem_tol": 1e-4, "row_floor": 0.0},
    "bf16": {"tol": 2e-2, "row_tol": 2e-2, "elem_tol": 2e-2, "row_floor": 0.0},
}
# Gradients: rows floored at the rms row norm, elements at 5x the tolerance (bf16 dq: the
# rounding of dS and P to bf16 before the products, with cancellation in the sums; measured
# worst element 0.074 of the 0.1 bound).
GRAD_BOUNDS = {
    "f32": {"tol": 1e-4, "row_tol": 1e-4, "elem_tol": 5e-4, "row_floor": 1.0},
    "bf16": {"tol": 2e-2, "row_tol": 2e-2, "elem_tol": 1e-1, "row_floor": 1.0},
}


def metrics(got, ref, row_floor=0.0) -> dict:
    """rel-L2, the worst row's relative error and the worst element's ratio to its bound
    (oracle.parity_metrics)."""
    return oracle.parity_metrics(got, ref, row_floor)


def _log(rec: dict):
    path = os.environ.get("PISA_PARITY_LOG")
    if not path:
        return
    rec = dict(rec)
    rec["test"] = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def check(got, ref, dt: str, what: str = "", tol=None, row_tol=None, elem_tol=None, grad=False) -> dict:
    """Assert the three bounds for dtype ``dt`` ("f32" or "bf16"), of GRAD_BOUNDS when ``grad``;
    returns the measured figures."""
    b = (GRAD_BOUNDS if grad else BOUNDS)[dt]
    tol = b["tol"] if tol is None else tol
    row_tol = b["row_tol"] if row_tol is None else row_tol
    elem_tol = b["elem_tol"] if elem_tol is None else elem_tol
    m = metrics(got, ref, b["row_floor"])
    _log({"what": what, "dt": dt, **m})
    assert m["rel_l2"] <= tol, (what, "rel-L2", m)
    assert m["row_max"] <= row_tol, (what, "worst row", m)
    assert m["elem_max"] <= elem_tol, (what, "worst element", m)
    return m
