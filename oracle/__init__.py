"""fp64 CPU oracle of HySparse2's token-level KV Reuse -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
import this package.  It loads oracle/_hs2_oracle.so (built from
hs2_oracle.c by oracle/build.py) and marshals numpy / torch CPU tensors.  It
shares nothing with the CUDA library.

Every function returns float64 results computed from the exact values of the
stored bf16 / e4m3 inputs; see hs2_oracle.c for the definitions and the
passages of the HySparse2 summary (onedev.kr/papers/146) they follow.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import build as _build

_lib = None
_c_i64p = ctypes.POINTER(ctypes.c_int64)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        L.hs2o_bf16_value.argtypes = [ctypes.c_uint16]
        L.hs2o_bf16_value.restype = dbl
        L.hs2o_e4m3_value.argtypes = [ctypes.c_uint8]
        L.hs2o_e4m3_value.restype = dbl
        L.hs2o_full_select.argtypes = [i32, i32, i32, i32, i32, i32, dbl, vp, vp, vp, i64, vp, vp,
                                       vp, vp, vp, vp, i32, vp, vp, vp]
        L.hs2o_full_select.restype = i32
        L.hs2o_sparse.argtypes = [i32, i32, i32, i32, dbl, vp, i32, vp, vp, vp, vp, i32, vp, i64,
                                  vp, vp]
        L.hs2o_sparse.restype = i32
        L.hs2o_decode_select.argtypes = [i32, i32, i32, i32, i32, i32, dbl, vp, i32, vp, vp, vp, vp,
                                         vp, vp, vp, vp, vp, vp, i32, vp, vp]
        L.hs2o_decode_select.restype = i32
        L.hs2o_decode_sparse.argtypes = [i32, i32, i32, i32, dbl, vp, i32, vp, vp, vp, vp, i32, vp,
                                         vp]
        L.hs2o_decode_sparse.restype = i32
        L.hs2o_num_threads.argtypes = []
        L.hs2o_num_threads.restype = i32
        _lib = L
    return _lib


def _np(x, dtype=None):
    """Contiguous numpy view of a CPU tensor / array (bf16 -> its uint16 bits)."""
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu()
        if x.dtype == torch.bfloat16:
            x = x.view(torch.int16)
        elif x.dtype == torch.float8_e4m3fn:
            x = x.view(torch.uint8)
        x = x.contiguous().numpy()
    x = np.ascontiguousarray(x)
    if dtype is not None:
        x = np.ascontiguousarray(x.astype(dtype, copy=False))
    return x


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().hs2o_num_threads()


def bf16_value(bits: int) -> float:
    return lib().hs2o_bf16_value(bits)


def e4m3_value(code: int) -> float:
    return lib().hs2o_e4m3_value(code)


def full_select(q, k, v, W: int, k_top: int, rows=None, scale=None, probe=None,
                want_score_row: bool = False):
    """Full-attention layer with token selection on query rows `rows`
    (flattened b*L+t; default all).  q [B,L,Hq,d], k/v [B,L,d] bf16.

    Returns dict: o [R,Hq,d], lse [R,Hq], idx [R,W+k] (window ascending, then
    globals best-first, -1 padding), sel_score [R,W+k], sigma_k [R] (-1 when
    every candidate is taken), probe_score [R,P] if probe [R,P] given,
    score_row [R,L] if asked.
    """
    B, L, Hq, d = q.shape
    scale = (1.0 / np.sqrt(d)) if scale is None else scale
    qn, kn, vn = _np(q), _np(k), _np(v)
    rows = np.arange(B * L, dtype=np.int64) if rows is None else _np(rows, np.int64)
    R, S = rows.shape[0], W + k_top
    o = np.zeros((R, Hq, d)); lse = np.zeros((R, Hq))
    idx = np.zeros((R, S), dtype=np.int32); sel = np.zeros((R, S)); sig = np.zeros(R)
    n_probe, pr, ps = 0, None, None
    if probe is not None:
        pr = _np(probe, np.int32)
        n_probe = pr.shape[1]
        ps = np.zeros((R, n_probe))
    srow = np.zeros((R, L)) if want_score_row else None
    rc = lib().hs2o_full_select(B, L, Hq, d, W, k_top, scale, _p(qn), _p(kn), _p(vn), R,
                                _p(rows), _p(o), _p(lse), _p(idx), _p(sel), _p(sig), n_probe,
                                _p(pr), _p(ps), _p(srow))
    if rc != 0:
        raise RuntimeError(f"hs2o_full_select failed ({rc})")
    out = dict(o=o, lse=lse, idx=idx, sel_score=sel, sigma_k=sig, rows=rows)
    if ps is not None:
        out["probe_score"] = ps
    if srow is not None:
        out["score_row"] = srow
    return out


def _kv_args(kv, k, v, k_scale, v_scale):
    kvd = {"bf16": 0, "e4m3": 1}[kv]
    kn, vn = _np(k), _np(v)
    ks = None if k_scale is None else _np(k_scale, np.float32)
    vs = None if v_scale is None else _np(v_scale, np.float32)
    if kvd == 1 and (ks is None or vs is None):
        raise ValueError("e4m3 K/V need per-token scales")
    return kvd, kn, vn, ks, vs


def sparse(q, k, v, idx, rows=None, scale=None, kv="bf16", k_scale=None, v_scale=None):
    """Sparse layer: each query row attends to the K/V rows named by idx [B*L, S]
    (entries < 0 ignored).  Returns o [R,Hq,d]."""
    B, L, Hq, d = q.shape
    scale = (1.0 / np.sqrt(d)) if scale is None else scale
    kvd, kn, vn, ks, vs = _kv_args(kv, k, v, k_scale, v_scale)
    qn = _np(q)
    idn = _np(idx, np.int32).reshape(B * L, -1)
    S = idn.shape[1]
    rows = np.arange(B * L, dtype=np.int64) if rows is None else _np(rows, np.int64)
    o = np.zeros((rows.shape[0], Hq, d))
    rc = lib().hs2o_sparse(B, L, Hq, d, scale, _p(qn), kvd, _p(kn), _p(vn), _p(ks), _p(vs), S,
                           _p(idn), rows.shape[0], _p(rows), _p(o))
    if rc != 0:
        raise RuntimeError(f"hs2o_sparse failed ({rc})")
    return o


def decode_select(q, k_cache, v_cache, lengths, W: int, k_top: int, kv="e4m3", k_scale=None,
                  v_scale=None, scale=None, probe=None):
    """Decode full layer: query of sequence b at position lengths[b]-1.
    Returns dict o [B,Hq,d], lse [B,Hq], idx/sel_score [B,W+k], sigma_k [B],
    probe_score [B,P] if probe [B,P] given."""
    B, Hq, d = q.shape
    Tmax = k_cache.shape[1]
    scale = (1.0 / np.sqrt(d)) if scale is None else scale
    kvd, kn, vn, ks, vs = _kv_args(kv, k_cache, v_cache, k_scale, v_scale)
    qn = _np(q)
    ln = _np(lengths, np.int32)
    S = W + k_top
    o = np.zeros((B, Hq, d)); lse = np.zeros((B, Hq)); idx = np.zeros((B, S), dtype=np.int32)
    sel = np.zeros((B, S)); sig = np.zeros(B)
    n_probe, pr, ps = 0, None, None
    if probe is not None:
        pr = _np(probe, np.int32)
        n_probe = pr.shape[1]
        ps = np.zeros((B, n_probe))
    rc = lib().hs2o_decode_select(B, Tmax, Hq, d, W, k_top, scale, _p(qn), kvd, _p(kn), _p(vn),
                                  _p(ks), _p(vs), _p(ln), _p(o), _p(lse), _p(idx), _p(sel),
                                  _p(sig), n_probe, _p(pr), _p(ps))
    if rc != 0:
        raise RuntimeError(f"hs2o_decode_select failed ({rc})")
    out = dict(o=o, lse=lse, idx=idx, sel_score=sel, sigma_k=sig)
    if ps is not None:
        out["probe_score"] = ps
    return out


def decode_sparse(q, k_cache, v_cache, idx, kv="e4m3", k_scale=None, v_scale=None, scale=None):
    """Decode sparse layer over idx [B,S] (entries < 0 ignored).  Returns o [B,Hq,d]."""
    B, Hq, d = q.shape
    Tmax = k_cache.shape[1]
    scale = (1.0 / np.sqrt(d)) if scale is None else scale
    kvd, kn, vn, ks, vs = _kv_args(kv, k_cache, v_cache, k_scale, v_scale)
    qn = _np(q)
    idn = _np(idx, np.int32)
    S = idn.shape[1]
    o = np.zeros((B, Hq, d))
    rc = lib().hs2o_decode_sparse(B, Tmax, Hq, d, scale, _p(qn), kvd, _p(kn), _p(vn), _p(ks),
                                  _p(vs), S, _p(idn), _p(o))
    if rc != 0:
        raise RuntimeError(f"hs2o_decode_sparse failed ({rc})")
    return o


def global_picks(row, t: int, W: int) -> set:
    """The global picks of one idx row of query position t: its entries s with
    0 <= s <= t - W (window entries and -1 padding excluded)."""
    return {int(s) for s in row if 0 <= int(s) <= t - W}


def selection_overlap(idx_a, idx_b, W: int, k_top: int):
    """Cross-layer overlap of two selections [B, L, S] (the IndexCache page,
    Appendix A, "Cross-Layer Top-(k) Index Overlap": |T(i) ∩ T(j)| / k).

    Per query row t: inter = |G_a(t) ∩ G_b(t)| with G the global picks, and
    ratio = inter / min(k, t - W + 1); rows without global candidates
    (t < W or k = 0) get ratio 1.  Returns (inter int64 [B, L], ratio float64
    [B, L]); plain Python sets, one row at a time."""
    a = _np(idx_a, np.int32)
    b = _np(idx_b, np.int32)
    B, L, _ = a.shape
    inter = np.zeros((B, L), dtype=np.int64)
    ratio = np.ones((B, L), dtype=np.float64)
    for bb in range(B):
        for t in range(L):
            n = len(global_picks(a[bb, t], t, W) & global_picks(b[bb, t], t, W))
            inter[bb, t] = n
            denom = min(k_top, t - W + 1) if (t >= W and k_top > 0) else 0
            if denom > 0:
                ratio[bb, t] = n / denom
    return inter, ratio


def block_select(q, k, v, W: int, k_top: int, block: int = 64, rows=None, scale=None):
    """Block-level selector of HySparse (64-token blocks, the same forced
    window), from the oracle's fp64 score rows.

    Candidate blocks of row t: the aligned `block`-position ranges that hold a
    position <= t - W; mass(t, j) = sum of score(t, s) over the block's
    positions s <= t - W.  The k_top/block blocks of largest mass are chosen
    (ties to the lower block; all when there are fewer).  Returns dict:
    idx [R, W+k] (window ascending, then the chosen blocks' candidate positions
    in ascending block order, -1 padding), mass [R, nblk] (0 beyond the
    candidates), sigma [R] (the smallest chosen mass, -1 when every block is
    taken), rows."""
    B, L = q.shape[:2]
    out = full_select(q, k, v, W, k_top, rows=rows, scale=scale, want_score_row=True)
    sr, rows = out["score_row"], out["rows"]
    R, S = rows.shape[0], W + k_top
    nsel = k_top // block
    nblk = (L + block - 1) // block
    idx = -np.ones((R, S), dtype=np.int32)
    mass = np.zeros((R, nblk))
    sigma = -np.ones(R)
    for r in range(R):
        t = int(rows[r] % L)
        w0 = max(0, t - W + 1)
        win = list(range(w0, t + 1))
        last = t - W
        nb = last // block + 1 if last >= 0 else 0
        for j in range(nb):
            mass[r, j] = float(np.sum(sr[r, block * j: min(block * j + block, last + 1)]))
        order = sorted(range(nb), key=lambda j: (-mass[r, j], j))
        chosen = sorted(order[:nsel])
        if nb > nsel:
            sigma[r] = mass[r, order[nsel - 1]]
        glob = [s for j in chosen for s in range(block * j, min(block * j + block, last + 1))]
        row = win + glob
        idx[r, :len(row)] = row
    return dict(idx=idx, mass=mass, sigma=sigma, rows=rows)
