"""hs2_decode_select_noalloc: the decode select variant for callers that
cannot allocate device memory (for example a server whose KV-cache pool
already holds nearly all HBM, or a plugin whose host exposes no allocator).

It must give the same results as hs2_decode_select with a caller workspace
and as the fp64 oracle, on consecutive calls (its fixed scratch keeps the
previous call's contents), and refuse shapes whose workspace would not fit
the scratch.  This file is collected last on purpose, so a failure here
comes after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import token_level_top_hs2_b200 as hs2
from tests.parity import check_selection, check_structure, max_abs
from token_level_top_hs2_b200 import build as hs2_build
from token_level_top_hs2_b200 import inputs

TOL_O = 2e-2       # output tolerances of the other parity tests: e4m3 KV
TOL_O_BF16 = 1e-2  # bf16 KV
TOL_LSE = 2e-3


def _noalloc(lib, x, dev):
    shape = hs2.decode_shape(x.B, x.Tmax, x.q.shape[1], x.d, x.W, x.k, x.kv)
    q, kc, vc = x.q.to(dev), x.k_cache.to(dev), x.v_cache.to(dev)
    ks = None if x.k_scale is None else x.k_scale.to(dev)
    vs = None if x.v_scale is None else x.v_scale.to(dev)
    lens = x.lengths.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(x.B, q.shape[1], dtype=torch.float32, device=dev)
    idx = torch.empty(x.B, x.W + x.k, dtype=torch.int32, device=dev)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = lib.hs2_decode_select_noalloc(ctypes.byref(shape), p(q), p(kc), p(vc), p(ks), p(vs),
                                       p(lens), p(o), p(lse), p(idx),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == hs2.HS2_OK, hs2.status_string(st)
    return o, lse, idx


def _same_selection(a, b, W, lengths):
    for r in range(a.shape[0]):
        wl = min(int(lengths[r]), W)
        assert np.array_equal(a[r, :wl], b[r, :wl])
        assert set(a[r][a[r] >= 0].tolist()) == set(b[r][b[r] >= 0].tolist())


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["e4m3_sketch", "e4m3_ragged", "e4m3_register_path", "bf16_d64"])
def test_noalloc_matches_workspace_version_on_consecutive_calls(cuda_lib, case):
    """Two calls in a row on the shared scratch, each against hs2_decode_select
    with a caller workspace and against the fp64 oracle.  The cases reach
    every workspace layout the scratch has to hold: the e4m3 sketch path
    (TMA-fed, d = 128), ragged lengths, the register path (Tmax % 4 != 0 with
    more than one sequence, where TMA cannot describe the scale rows) and a
    bf16 cache with d = 64."""
    lib = hs2.load()
    dev = torch.device("cuda:0")
    if case == "e4m3_sketch":
        x = inputs.make_decode(4, 65536, 16, 128, 128, 1024, kv="e4m3", seed=101, n_sparse=0)
    elif case == "e4m3_ragged":
        x = inputs.make_decode(4, 65536, 16, 128, 128, 1024, kv="e4m3", seed=202, n_sparse=0,
                               lengths=[65536, 30000, 7, 1200])
    elif case == "e4m3_register_path":
        x = inputs.make_decode(2, 5001, 16, 128, 128, 256, kv="e4m3", seed=303, n_sparse=0,
                               lengths=[5001, 3000])
    else:
        x = inputs.make_decode(2, 5000, 8, 64, 32, 128, kv="bf16", seed=404, n_sparse=0,
                               lengths=[5000, 77])
    tol_o = TOL_O if x.kv == "e4m3" else TOL_O_BF16
    o_ref, lse_ref, idx_ref = hs2.hs2_decode_select(
        x.q.to(dev), x.k_cache.to(dev), x.v_cache.to(dev), x.lengths.to(dev), x.W, x.k,
        kv=x.kv, k_scale=None if x.k_scale is None else x.k_scale.to(dev),
        v_scale=None if x.v_scale is None else x.v_scale.to(dev))
    outs = [_noalloc(lib, x, dev) for _ in range(2)]
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    for o, lse, idx in outs:
        assert (o.float() - o_ref.float()).abs().max().item() <= tol_o
        assert (lse - lse_ref).abs().max().item() <= TOL_LSE
        _same_selection(idx.cpu().numpy(), idx_ref.cpu().numpy(), x.W, x.lengths)
    # and against the oracle
    o, lse, idx = (t.cpu() for t in outs[1])
    idx = idx.numpy()
    ora = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, x.W, x.k, kv=x.kv,
                               k_scale=x.k_scale, v_scale=x.v_scale, probe=idx)
    assert max_abs(o.float().numpy(), ora["o"]) <= tol_o
    assert max_abs(lse.numpy(), ora["lse"]) <= TOL_LSE
    t = x.lengths.numpy().astype(np.int64) - 1
    check_structure(idx, t, x.W, x.k)
    check_selection(idx, ora, t, x.W, x.k)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    hs2_build.build()
    lib = hs2.load()
    fake = 1 << 20  # aligned stand-in pointers; the call must return before using them
    big = hs2.decode_shape(64, 1 << 20, 16, 128, 128, 1024, "e4m3")
    assert hs2.hs2_decode_select_workspace(big) > (96 << 20)
    st = lib.hs2_decode_select_noalloc(ctypes.byref(big), fake, fake, fake, fake, fake, fake,
                                       fake, None, fake, None)
    assert st == hs2.HS2_ERR_WORKSPACE
    fits = hs2.decode_shape(16, 262144, 16, 128, 128, 1024, "e4m3")
    assert hs2.hs2_decode_select_workspace(fits) <= (96 << 20)
