"""hs2_decode_select_noalloc: the decode select variant for callers that
cannot allocate device memory (for example a server whose KV-cache pool
already holds nearly all HBM, or a plugin whose host exposes no allocator).

It must give the same results as hs2_decode_select with a caller workspace,
on consecutive calls (its fixed scratch keeps the previous call's contents),
and refuse shapes whose workspace would not fit the scratch.  This file is
collected last on purpose, so a failure here comes after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import token_level_top_hs2_b200 as hs2
from token_level_top_hs2_b200 import build as hs2_build
from token_level_top_hs2_b200 import inputs

TOL_O = 2e-2    # e4m3 KV output tolerance used by the other parity tests
TOL_LSE = 2e-3


def _noalloc(lib, x, dev):
    shape = hs2.decode_shape(x.B, x.Tmax, x.q.shape[1], x.d, x.W, x.k, x.kv)
    q, kc, vc = x.q.to(dev), x.k_cache.to(dev), x.v_cache.to(dev)
    ks, vs, lens = x.k_scale.to(dev), x.v_scale.to(dev), x.lengths.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(x.B, q.shape[1], dtype=torch.float32, device=dev)
    idx = torch.empty(x.B, x.W + x.k, dtype=torch.int32, device=dev)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
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
def test_noalloc_matches_workspace_version_on_consecutive_calls(cuda_lib):
    lib = hs2.load()
    dev = torch.device("cuda:0")
    cases = [
        inputs.make_decode(4, 65536, 16, 128, 128, 1024, kv="e4m3", seed=101, n_sparse=0),
        inputs.make_decode(4, 65536, 16, 128, 128, 1024, kv="e4m3", seed=202, n_sparse=0,
                           lengths=[65536, 30000, 7, 1200]),
    ]
    for x in cases:  # two calls in a row on the shared scratch
        o_ref, lse_ref, idx_ref = hs2.hs2_decode_select(
            x.q.to(dev), x.k_cache.to(dev), x.v_cache.to(dev), x.lengths.to(dev), x.W, x.k,
            kv="e4m3", k_scale=x.k_scale.to(dev), v_scale=x.v_scale.to(dev))
        o, lse, idx = _noalloc(lib, x, dev)
        torch.cuda.synchronize()
        assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
        assert (o.float() - o_ref.float()).abs().max().item() <= TOL_O
        assert (lse - lse_ref).abs().max().item() <= TOL_LSE
        _same_selection(idx.cpu().numpy(), idx_ref.cpu().numpy(), x.W, x.lengths)


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
