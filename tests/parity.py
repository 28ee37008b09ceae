"""Shared helpers of the GPU parity tests: run a case through the C ABI and
through the CPU oracle on the same seeded inputs, and compare.

Tolerance.  Logits are compared to the oracle's fp64 LUT result, softcapped
in fp64.  The gate is the normwise maximum error per token,
    max_v |y_gpu[b,v] - y_ref[b,v]| <= 1e-5 * max_v |y_ref[b,v]|,
the 1e-5 relative fp32 bar stated for this path.  (Elementwise relative
error is ill-conditioned for logits near zero.)  The fp32 GPU path carries
about sqrt(P) * 2^-24 of the partial-sum magnitude (P = M*L table terms per
row) plus tanhf's few ulp, i.e. ~1e-6 relative at the Gemma-2 shape.
The lookup tables themselves are compared elementwise at 2e-6 relative to
the largest table entry (6-term fp32 dot products with FMA).

Argmax: both sides decide in fp32 (the GPU's own precision): the oracle's
fp64 logits are rounded to fp32 and the lowest index of the maximum is
taken.  When the oracle's top-two gap exceeds twice the error bound the two
must agree exactly; otherwise the GPU's choice must lie in the set of rows
within that bound of the maximum (ties are then reported, not hidden).
"""
from __future__ import annotations

import numpy as np

import oracle

RTOL = 1e-5


def normwise_err(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per-token max |got - ref| / max |ref| (rows = tokens)."""
    got = np.atleast_2d(got).astype(np.float64)
    ref = np.atleast_2d(ref).astype(np.float64)
    den = np.maximum(np.max(np.abs(ref), axis=1), 1e-30)
    return np.max(np.abs(got - ref), axis=1) / den


def assert_logits_close(got, ref, rtol=RTOL, what="logits"):
    err = normwise_err(got, ref)
    assert np.all(err <= rtol), f"{what}: normwise error {err.max():.3g} > {rtol}"
    return float(err.max())


def check_argmax(gpu_idx, y_ref64, rtol=RTOL):
    """gpu_idx [B]; y_ref64 [B, V] full oracle logits (fp64).  Returns the
    number of tokens whose top-two gap was within the bound (ties)."""
    ties = 0
    y32 = y_ref64.astype(np.float32)
    want = oracle.argmax(y32)
    for b in range(y_ref64.shape[0]):
        row = y_ref64[b]
        bound = 2 * rtol * np.max(np.abs(row))
        order = np.argsort(row)[::-1]
        gap = row[order[0]] - row[order[1]] if row.size > 1 else np.inf
        if gap > bound:
            assert int(gpu_idx[b]) == int(want[b]), (b, int(gpu_idx[b]), int(want[b]), gap)
        else:
            ties += 1
            near = set(np.nonzero(row >= row[order[0]] - bound)[0].tolist())
            assert int(gpu_idx[b]) in near, (b, int(gpu_idx[b]), sorted(near)[:8])
    return ties
