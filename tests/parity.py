"""Comparison rules between the CUDA library and the fp64 oracle.

Selection (HySparse2 summary, onedev.kr/papers/146, 'What differs': the
recent window first, then the highest-scoring tokens outside it):
  * the window part of every row must be identical;
  * the global parts must have the same size;
  * every index in the symmetric difference must have an oracle score within
    `rel` (relative) of the oracle's k-th global score sigma_k: such a swap is
    a tie up to rounding, any other difference is an error.
Structure (checked on every row, any size): window inside the selection,
|Sel| = min(t+1, W+k), every index in [0, t], no duplicates, -1 only as tail
padding.
"""
from __future__ import annotations

import numpy as np


def window_of(t: int, W: int) -> np.ndarray:
    return np.arange(max(0, t - W + 1), t + 1, dtype=np.int64)


def check_structure(idx: np.ndarray, t: np.ndarray, W: int, k: int) -> None:
    """idx [R, W+k] int32 in the library's format; t [R] query positions."""
    idx = np.asarray(idx)
    t = np.asarray(t)
    R, S = idx.shape
    assert S == W + k
    n_valid = (idx >= 0).sum(axis=1)
    expect = np.minimum(t + 1, W + k)
    bad = np.nonzero(n_valid != expect)[0]
    assert bad.size == 0, f"row {bad[0]}: {n_valid[bad[0]]} valid entries, expected {expect[bad[0]]}"
    # -1 only as tail padding
    pos = np.arange(S)[None, :]
    assert np.all((idx >= 0) == (pos < n_valid[:, None])), "padding not at the tail"
    assert np.all(idx <= t[:, None]), "index beyond the query position"
    assert np.all(idx >= -1)
    # window slots first, ascending
    wlen = np.minimum(t + 1, W)
    for r in range(R):
        w = window_of(int(t[r]), W)
        assert np.array_equal(idx[r, : wlen[r]], w), f"row {r}: window slots differ"
        sel = idx[r, : n_valid[r]]
        assert np.unique(sel).size == sel.size, f"row {r}: duplicate indices"


def check_selection(gpu_idx: np.ndarray, ora: dict, t: np.ndarray, W: int, k: int,
                    rel: float = 1e-5):
    """Compare selections row by row.  `ora` holds idx, sel_score, sigma_k and
    probe_score (oracle scores of the GPU's entries, probed with gpu_idx).

    Returns (n_swapped, overlap) where overlap is the mean |G_gpu & G_ora| / |G|.
    """
    gpu_idx = np.asarray(gpu_idx)
    t = np.asarray(t)
    R = gpu_idx.shape[0]
    n_swap = 0
    overlaps = []
    for r in range(R):
        wl = min(int(t[r]) + 1, W)
        g_w, o_w = gpu_idx[r, :wl], ora["idx"][r, :wl]
        assert np.array_equal(g_w, o_w), f"row {r} (t={t[r]}): window differs"
        g_glob = gpu_idx[r, wl:]
        g_glob = g_glob[g_glob >= 0]
        o_glob = ora["idx"][r, wl:]
        o_glob = o_glob[o_glob >= 0]
        assert g_glob.size == o_glob.size, \
            f"row {r} (t={t[r]}): {g_glob.size} globals vs oracle {o_glob.size}"
        if o_glob.size == 0:
            continue
        gs, os_ = set(g_glob.tolist()), set(o_glob.tolist())
        overlaps.append(len(gs & os_) / len(os_))
        only_g = gs - os_
        only_o = os_ - gs
        if not only_g and not only_o:
            continue
        sig = ora["sigma_k"][r]
        assert sig >= 0, f"row {r}: sets differ although every candidate is taken"
        tol = rel * sig
        # oracle scores of GPU-only picks (probe scores follow gpu_idx order)
        probe = ora["probe_score"][r]
        pmap = {int(p): probe[j] for j, p in enumerate(gpu_idx[r]) if p >= 0}
        for s in only_g:
            assert abs(pmap[s] - sig) <= tol, \
                f"row {r} (t={t[r]}): GPU picked {s} (score {pmap[s]!r}) vs sigma_k {sig!r}"
        omap = {int(p): ora["sel_score"][r, j] for j, p in enumerate(ora["idx"][r]) if p >= 0}
        for s in only_o:
            assert abs(omap[s] - sig) <= tol, \
                f"row {r} (t={t[r]}): GPU missed {s} (score {omap[s]!r}) vs sigma_k {sig!r}"
        n_swap += len(only_g)
    return n_swap, (float(np.mean(overlaps)) if overlaps else 1.0)


def max_abs(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - b)))
