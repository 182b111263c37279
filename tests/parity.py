"""Parity checks of library results against the oracle (tolerances written here, used by the GPU tests).

Index sets: identical to the oracle's, except positions whose oracle score lies within
1e-4 relative of the oracle's M-th score (floor 1e-3 * rms of the scores), where fp32
rounding on the device may legitimately swap tied-in-practice neighbours.

Outputs: per (b, query head) row, max_i |o_i - o*_i| / max_i |o*_i| <= 1e-2 for bf16 outputs
with fp32 accumulation; o* is the oracle's output.  Outputs are only compared for (b, KV head)
pairs whose index sets are identical (a legitimate swap inside the tie band changes the set the
output is computed over); the other pairs are checked for a valid set.
"""

from __future__ import annotations

import numpy as np

INDEX_REL_BAND = 1e-4
OUT_REL_TOL = 1e-2


def index_band(scores: np.ndarray, m: int) -> tuple:
    s_sorted = np.sort(scores)[::-1]
    s_m = s_sorted[m - 1]
    rms = float(np.sqrt(np.mean(scores**2)))
    return s_m, INDEX_REL_BAND * max(abs(s_m), 1e-3 * rms)


def check_index_sets(gpu_idx: np.ndarray, gpu_count: np.ndarray, oracle: dict, seq_lens, M: int, pairs) -> list:
    """Assert validity of every set; return the pairs whose sets equal the oracle's exactly."""
    identical = []
    for b, h in pairs:
        n = int(seq_lens[b])
        m = min(M, n)
        assert int(gpu_count[b, h]) == m, (b, h, int(gpu_count[b, h]), m)
        sel = gpu_idx[b, h, :m].astype(np.int64)
        assert np.all((sel >= 0) & (sel < n)), (b, h)
        assert np.all(np.diff(sel) > 0), ("not strictly ascending", b, h)
        assert np.all(gpu_idx[b, h, m:] == -1), (b, h)
        ref = oracle["idx"][b][h]
        if np.array_equal(sel, ref):
            identical.append((b, h))
            continue
        s = oracle["scores"][b][h]
        s_m, tol = index_band(s, m)
        diff = np.setxor1d(sel, ref)
        far = [int(t) for t in diff if abs(s[t] - s_m) > tol]
        assert not far, f"(b={b}, h={h}): positions {far[:8]} differ outside the tie band (s_M={s_m}, tol={tol})"
    return identical


def check_outputs(gpu_out: np.ndarray, ref_out: np.ndarray, pairs, G: int, tol: float = OUT_REL_TOL) -> float:
    worst = 0.0
    for b, h in pairs:
        for j in range(h * G, (h + 1) * G):
            ref = ref_out[b, j]
            err = np.max(np.abs(gpu_out[b, j] - ref)) / max(np.max(np.abs(ref)), 1e-30)
            worst = max(worst, float(err))
            assert err <= tol, (b, j, err)
    return worst
