"""Shared test helpers: golden-file parsing and the parity error measure."""
from __future__ import annotations

import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name: str) -> dict:
    """Parse a `key v1 v2 ...` text fixture (lines starting with # are comments)."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = np.array([float(x) for x in vals], dtype=np.float64)
    return out


# Every parity error the tests compute, with the test and the line that
# asked for it; conftest.py prints the worst per test at the end of the run
# and, when RETNET_PARITY_LOG names a file, writes them all there as JSON.
MEASURED = []


def record(value: float, what: str = "") -> float:
    """Keeps an achieved error (and what it measures) for the run's report."""
    import inspect
    caller = inspect.stack()[1]
    frame = caller
    for f in inspect.stack()[1:]:            # the test function's own line
        if os.path.basename(f.filename).startswith("test_"):
            frame = f
            break
    MEASURED.append({"test": os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0],
                     "where": f"{os.path.basename(frame.filename)}:{frame.lineno}",
                     "what": what, "err": float(value)})
    return value


def slice_rel_err(got, ref, head_axis: int = 2, keep: bool = True) -> float:
    """Norm-wise relative error, worst over (batch, head) slices.

    For each (batch, head) slice: max|got - ref| / max|ref|.  This is the
    reading of "max relative error" used for parity: an elementwise ratio is
    meaningless at the many near-zero entries of a retention output.
    Arrays are [B, n, H, d] (head_axis=2) or [B, H, ...] (head_axis=1).
    keep=False leaves the value out of the run's report of achieved errors.
    """
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if got.size == 0:
        return 0.0
    g = np.moveaxis(got, head_axis, 1).reshape(got.shape[0], got.shape[head_axis], -1)
    r = np.moveaxis(ref, head_axis, 1).reshape(ref.shape[0], ref.shape[head_axis], -1)
    num = np.abs(g - r).max(axis=-1)
    den = np.abs(r).max(axis=-1)
    den = np.where(den == 0, 1.0, den)
    err = float("inf") if not np.all(np.isfinite(g)) else float((num / den).max())
    return record(err, "slice") if keep else err
