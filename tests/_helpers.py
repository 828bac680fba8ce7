"""Shared test plumbing: build the same workload on the GPU (through the C ABI)
and in the oracle, and compare under the stated tolerances."""
from __future__ import annotations

import numpy as np

from compressed_paged_kv_tq4_b200 import inputs as I
from oracle import tq4_oracle as O

BF16_ABS_TOL = 2e-3       # attention outputs in bf16
F32_ABS_TOL = 1e-4        # attention outputs kept in fp32
RECON_REL_TOL = 1e-3      # reconstructed K/V, per vector ||d|| / ||x||
BOUNDARY_EXEMPT = 1e-6    # quantiser decisions this close to a boundary may differ


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def bf16_tolerance(expect):
    """|gpu - oracle| allowed per element for bf16 outputs: 2e-3, or one bf16 ulp
    of the oracle value where the bf16 grid itself is coarser than 2e-3."""
    return np.maximum(BF16_ABS_TOL, bf16_ulp(expect))


def assert_bf16_close(got, expect, what=""):
    got = np.asarray(got, np.float64)
    expect = np.asarray(expect, np.float64)
    err = np.abs(got - expect)
    tol = bf16_tolerance(expect)
    bad = ~(err <= tol)   # a NaN or Inf anywhere fails too
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(np.isfinite(err), err - tol, np.inf)), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst at {i}: "
                             f"got {got[i]} expect {expect[i]} (tol {tol[i]})")
    return float(err.max())


def oracle_codebook():
    c, _ = O.codebook()
    return c


def check_words_against_oracle(gpu_words, ora_words, ora_y, boundaries, what=""):
    """Packed words must match bit for bit, except nibbles whose oracle coordinate
    lies within BOUNDARY_EXEMPT of a decision boundary, where the GPU may pick the
    neighbouring cell. Returns the number of exempt nibbles that differ."""
    gi = O.unpack_indices(np.asarray(gpu_words, np.uint32)).astype(np.int64)
    oi = O.unpack_indices(np.asarray(ora_words, np.uint32)).astype(np.int64)
    diff = gi != oi
    if not diff.any():
        return 0
    y = np.asarray(ora_y)[diff]
    dist = np.min(np.abs(y[:, None] - np.asarray(boundaries)[None, :]), axis=1)
    near = dist < BOUNDARY_EXEMPT
    adjacent = np.abs(gi[diff] - oi[diff]) == 1
    ok = near & adjacent
    if not ok.all():
        k = int(np.flatnonzero(~ok)[0])
        raise AssertionError(f"{what}: {int((~ok).sum())} nibbles differ away from a boundary; "
                             f"first: y={y[k]!r} dist={dist[k]:.3g} gpu={gi[diff][k]} oracle={oi[diff][k]}")
    return int(diff.sum())


def check_norms_against_oracle(gpu_norm16, ora_norm16, x, what=""):
    """fp16 norms must match except where ||x|| is within 1e-6 (relative) of an fp16 rounding midpoint."""
    g = np.asarray(gpu_norm16, np.float16)
    o = np.asarray(ora_norm16, np.float16)
    diff = g.view(np.uint16) != o.view(np.uint16)
    if not diff.any():
        return 0
    n = np.linalg.norm(np.asarray(x, np.float64).reshape(-1, 256), axis=1).reshape(o.shape)[diff]
    lo = np.minimum(g[diff], o[diff]).astype(np.float64)
    hi = np.maximum(g[diff], o[diff]).astype(np.float64)
    mid = 0.5 * (lo + hi)
    ok = (np.abs(n - mid) <= 1e-6 * n) & (np.nextafter(lo.astype(np.float16), np.float16(np.inf)).astype(np.float64) == hi)
    if not ok.all():
        raise AssertionError(f"{what}: {int((~ok).sum())} fp16 norms differ away from a rounding midpoint")
    return int(diff.sum())
