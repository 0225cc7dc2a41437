"""Shared helpers of the test suite: error metric and oracle/GPU glue."""
from __future__ import annotations

import numpy as np

# Tolerances on the max relative error (see rel_err): fp32 mode, bf16-in/fp32-accumulate mode.
TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def rel_err(o, ref) -> float:
    """Max over tokens of |o_t - ref_t|_inf / max(|ref_t|_inf, rms(ref)).

    Per-token relative error in the infinity norm, with the floor at the RMS
    of the whole reference output: for a token whose read-out nearly cancels,
    the achievable absolute error is set by the size of the terms, not by the
    (tiny) result, so it is measured against the typical output size.
    """
    o = np.asarray(o, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    d = np.abs(o - ref).reshape(-1, ref.shape[-1]).max(-1)
    rms = np.sqrt(np.mean(ref ** 2))
    den = np.maximum(np.abs(ref).reshape(-1, ref.shape[-1]).max(-1), rms)
    den = np.where(den > 0, den, 1.0)
    return float((d / den).max())


def err_report(o, ref) -> dict:
    """Diagnostics: the asserted metric plus two other normalisations."""
    o = np.asarray(o, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(o - ref).reshape(-1, ref.shape[-1]).max(-1)
    rms = np.sqrt(np.mean(ref ** 2))
    tok = np.abs(ref).reshape(-1, ref.shape[-1]).max(-1)
    return dict(rel=rel_err(o, ref),
                rel_floor_1e3rms=float((d / np.maximum(tok, 1e-3 * rms)).max()),
                global_rel=float(np.abs(o - ref).max() / max(np.abs(ref).max(), 1e-300)))


def count_agreement(iters, iters_ref) -> tuple[int, float]:
    """(max |iters - iters_ref|, fraction of tokens whose count differs)."""
    diff = np.abs(np.asarray(iters, np.int64) - np.asarray(iters_ref, np.int64))
    if diff.size == 0:
        return 0, 0.0
    return int(diff.max()), float((diff > 0).mean())


def log_parity(case: str, o, ref, **extra) -> dict:
    """err_report of one parity comparison; when MESA_PARITY_LOG names a file,
    the report is also appended to it as one JSON line (with the case name),
    so a run keeps both error floors of every case it checked."""
    import json
    import os
    rep = dict(case=case, **err_report(o, ref), **extra)
    path = os.environ.get("MESA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rep) + "\n")
    return rep
