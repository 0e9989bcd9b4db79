"""Comparison of bf16 kernel outputs with fp64 oracle values, and row sampling.

Tolerance (stated for the path): relative Frobenius error <= 1e-2 and max abs
error <= 3e-2 on the bf16 outputs. Where |oracle| >= 8 the bf16 grid itself is
coarser than 3e-2 (half an ulp is 2^-5 = 0.03125 on [8, 16)), so such
elements are reported on their own and pass when their error is within half
an ulp of the bf16 grid at that magnitude plus HAZARD_SLACK = 1e-3, the
representation-limited bound; the Frobenius bound is never relaxed.

With MLA_PARITY_LOG set to a file path, every check appends its label and
metrics to that file as one JSON line (the record of n_hazard,
hazard_worst_excess and hazard_max_err_ulps behind a run).
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

REL_FROB = 1e-2
MAX_ABS = 3e-2
HAZARD = 8.0
HAZARD_SLACK = 1e-3


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 1e-30)))
    return 0.5 * np.exp2(e - 7)


def metrics(got: np.ndarray, ref: np.ndarray) -> dict:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    err = np.abs(got - ref)
    nref = np.linalg.norm(ref)
    rel = float(np.linalg.norm(got - ref) / nref) if nref > 0 else float(np.linalg.norm(got - ref))
    haz = np.abs(ref) >= HAZARD
    out = {
        "rel_frob": rel,
        "max_abs": float(err[~haz].max()) if (~haz).any() else 0.0,
        "max_abs_all": float(err.max()) if err.size else 0.0,
        "max_ref": float(np.abs(ref).max()) if ref.size else 0.0,
        "n_hazard": int(haz.sum()),
        "finite": bool(np.isfinite(got).all()),
    }
    if haz.any():
        excess = err[haz] - (bf16_half_ulp(ref[haz]) + HAZARD_SLACK)
        out["hazard_worst_excess"] = float(excess.max())
        out["hazard_max_err_ulps"] = float((err[haz] / (2 * bf16_half_ulp(ref[haz]))).max())
    return out


def log_metrics(label: str, m: dict) -> None:
    path = os.environ.get("MLA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"label": label, **m}) + "\n")


def assert_parity(got, ref, label: str = "") -> dict:
    m = metrics(got, ref)
    log_metrics(label, m)
    msg = f"{label}: {m}"
    assert m["finite"], msg
    assert m["rel_frob"] <= REL_FROB, msg
    assert m["max_abs"] <= MAX_ABS, msg
    if m["n_hazard"]:
        assert m["hazard_worst_excess"] <= 0.0, msg
    return m


def assert_peaked(got, ref, rows, label: str = "") -> None:
    """Rows whose answer is essentially one value row (the causal rows of
    inputs.make_peaked_inputs): every element within half a bf16 ulp of the
    oracle, plus 1e-4 for the vanishing weight of the other keys."""
    g = np.asarray(got, dtype=np.float64)[rows]
    r = np.asarray(ref, dtype=np.float64)[rows]
    err = np.abs(g - r)
    bad = np.argwhere(err > bf16_half_ulp(r) + 1e-4)
    assert bad.size == 0, (f"{label}: {len(bad)} elements off, first at (row, col) "
                           f"{bad[0].tolist()}: got {g[tuple(bad[0])]} want {r[tuple(bad[0])]}")


def sample_rows(B: int, T: int, n_random: int, seed: int = 0, valid_len=None, tile: int = 128):
    """Rows (b, t) to check at full size: t = 0 and T-1, every tile boundary
    +-1, every row of the last query tile, rows around each valid length, and
    random rows; all batches."""
    g = np.random.default_rng(seed)
    rows = set()
    for b in range(B):
        picks = {0, T - 1}
        for t0 in range(tile, T, tile):
            picks.update({t0 - 1, t0, t0 + 1})
        last0 = ((T - 1) // tile) * tile
        picks.update(range(last0, T))
        if valid_len is not None:
            L = int(valid_len[b])
            picks.update({L - 2, L - 1, L, L + 1})
        for t in picks:
            if 0 <= t < T:
                rows.add((b, t))
    n_b = max(1, n_random // B)
    for b in range(B):
        for t in g.integers(0, T, size=n_b):
            rows.add((b, int(t)))
    return sorted(rows)
