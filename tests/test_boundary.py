"""Host-side boundary tests of the C ABI (no GPU needed): the library loads,
exports every entry point include/hs2.h declares, sizes workspaces, and
rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest
import torch

import token_level_top_hs2_b200 as hs2
from token_level_top_hs2_b200 import build as hs2_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    hs2_build.build()
    return hs2.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hs2.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hs2_\w+)\s*\(", src)))


def test_header_declares_the_four_entry_points():
    names = declared_functions()
    for n in ["hs2_full_attn_select", "hs2_sparse_attn", "hs2_decode_select",
              "hs2_decode_sparse"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
    assert sorted(hs2.EXPORTED) == names


def test_status_strings(lib):
    for code in range(7):
        assert hs2.status_string(code) != "unknown status"
    assert hs2.status_string(99) == "unknown status"
    assert lib.hs2_version() >= 100


def test_workspace_sizes(lib):
    s = hs2.prefill_shape(1, 131072, 16, 128, 128, 1024)
    ws = hs2.hs2_full_attn_select_workspace(s)
    # lse area, the query-block flags, and four candidate streams of
    # round_up(2k + 128, 32) 8-byte keys per query row
    cap = (2 * 1024 + 128 + 31) // 32 * 32
    assert ws >= 131072 * 4 * cap * 8 + 131072 * 16 * 4
    assert ws < 131072 * 4 * cap * 8 + 131072 * 16 * 4 + 4096 + 1024 * 4
    assert hs2.hs2_full_attn_select_workspace(hs2.prefill_shape(1, 10, 3, 128, 8, 8)) == 0
    d = hs2.decode_shape(16, 262144, 16, 128, 128, 1024)
    assert hs2.hs2_decode_select_workspace(d) > 16 * 1024 * 8
    assert hs2.hs2_decode_select_workspace(hs2.decode_shape(1, 100, 16, 96, 8, 8)) == 0


FAKE = 1 << 20  # 16-byte aligned non-null stand-ins: never dereferenced on failure


def call_full(lib, shape, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, idx=FAKE, ws=FAKE,
              ws_bytes=1 << 40):
    return lib.hs2_full_attn_select(ctypes.byref(shape), q, k, v, o, lse, idx, ws, ws_bytes, None)


@pytest.mark.parametrize("fields,code", [
    (dict(d=96), hs2.HS2_ERR_UNSUPPORTED),
    (dict(Hq=3), hs2.HS2_ERR_UNSUPPORTED),
    (dict(W=1024, k=1025), hs2.HS2_ERR_UNSUPPORTED),
    (dict(W=0), hs2.HS2_ERR_INVALID_ARG),
    (dict(k=-1), hs2.HS2_ERR_INVALID_ARG),
    (dict(L=0), hs2.HS2_ERR_INVALID_ARG),
    (dict(B=0), hs2.HS2_ERR_INVALID_ARG),
    (dict(scale=0.0), hs2.HS2_ERR_INVALID_ARG),
    (dict(scale=float("nan")), hs2.HS2_ERR_INVALID_ARG),
])
def test_full_select_rejects_bad_shapes(lib, fields, code):
    base = dict(B=1, L=64, Hq=16, d=128, W=8, k=8, scale=0.1)
    base.update(fields)
    s = hs2.PrefillShape(**base)
    assert call_full(lib, s) == code


def test_full_select_rejects_bad_pointers_and_workspace(lib):
    s = hs2.prefill_shape(1, 64, 16, 128, 8, 8)
    assert call_full(lib, s, q=None) == hs2.HS2_ERR_INVALID_ARG
    assert call_full(lib, s, idx=None) == hs2.HS2_ERR_INVALID_ARG
    assert call_full(lib, s, k=FAKE + 8) == hs2.HS2_ERR_INVALID_ARG
    assert call_full(lib, s, lse=FAKE + 4) == hs2.HS2_ERR_INVALID_ARG
    need = hs2.hs2_full_attn_select_workspace(s)
    assert call_full(lib, s, ws_bytes=need - 1) == hs2.HS2_ERR_WORKSPACE
    assert lib.hs2_full_attn_select(None, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 40,
                                    None) == hs2.HS2_ERR_INVALID_ARG


def test_sparse_rejects_bad_arguments(lib):
    s = hs2.prefill_shape(1, 64, 16, 128, 8, 8)
    f = lib.hs2_sparse_attn
    assert f(ctypes.byref(s), FAKE, FAKE, FAKE, hs2.HS2_KV_E4M3, None, FAKE, FAKE, FAKE,
             None) == hs2.HS2_ERR_INVALID_ARG
    assert f(ctypes.byref(s), FAKE, FAKE, FAKE, 7, None, None, FAKE, FAKE,
             None) == hs2.HS2_ERR_INVALID_ARG
    assert f(ctypes.byref(s), FAKE, FAKE, FAKE, hs2.HS2_KV_BF16, None, None, None, FAKE,
             None) == hs2.HS2_ERR_INVALID_ARG
    s64 = hs2.prefill_shape(1, 64, 16, 64, 8, 8)
    assert f(ctypes.byref(s64), FAKE, FAKE, FAKE, hs2.HS2_KV_E4M3, FAKE, FAKE, FAKE, FAKE,
             None) == hs2.HS2_ERR_UNSUPPORTED


def test_decode_rejects_bad_arguments(lib):
    s = hs2.decode_shape(2, 1000, 16, 128, 8, 8, "e4m3")
    f = lib.hs2_decode_select
    need = hs2.hs2_decode_select_workspace(s)
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE]
    assert f(ctypes.byref(s), *args, need - 1, None) == hs2.HS2_ERR_WORKSPACE
    bad = list(args)
    bad[3] = None  # k_scale missing for e4m3
    assert f(ctypes.byref(s), *bad, need, None) == hs2.HS2_ERR_INVALID_ARG
    bad = list(args)
    bad[5] = None  # lengths
    assert f(ctypes.byref(s), *bad, need, None) == hs2.HS2_ERR_INVALID_ARG
    s_bad = hs2.DecodeShape(2, 0, 16, 128, 8, 8, 0.1, 1)
    assert f(ctypes.byref(s_bad), *args, need, None) == hs2.HS2_ERR_INVALID_ARG
    s_kv = hs2.DecodeShape(2, 100, 16, 128, 8, 8, 0.1, 5)
    assert f(ctypes.byref(s_kv), *args, need, None) == hs2.HS2_ERR_INVALID_ARG
    g = lib.hs2_decode_sparse
    assert g(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
             None) == hs2.HS2_ERR_INVALID_ARG


def test_split_prefill_calls_reject_bad_arguments(lib):
    s = hs2.prefill_shape(1, 64, 16, 128, 8, 8)
    # hs2_full_attn needs lse (the selection reads it)
    assert lib.hs2_full_attn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None,
                             None) == hs2.HS2_ERR_INVALID_ARG
    need = hs2.hs2_full_attn_select_workspace(s)
    f = lib.hs2_select
    assert f(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, None) == hs2.HS2_ERR_WORKSPACE
    assert f(ctypes.byref(s), FAKE, FAKE, None, FAKE, FAKE, need, None) == hs2.HS2_ERR_INVALID_ARG
    bad = hs2.prefill_shape(1, 64, 12, 128, 8, 8)  # 12 query heads: unsupported
    assert f(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, need, None) == hs2.HS2_ERR_UNSUPPORTED


def test_overlap_rejects_bad_arguments(lib):
    s = hs2.prefill_shape(1, 64, 16, 128, 8, 8)
    f = lib.hs2_selection_overlap
    # both outputs missing, an input missing, a misaligned output
    assert f(ctypes.byref(s), FAKE, FAKE, None, None, None) == hs2.HS2_ERR_INVALID_ARG
    assert f(ctypes.byref(s), None, FAKE, FAKE, FAKE, None) == hs2.HS2_ERR_INVALID_ARG
    assert f(ctypes.byref(s), FAKE, FAKE, FAKE + 4, None, None) == hs2.HS2_ERR_INVALID_ARG
    # positions must fit the 21-bit hash-set entries
    big = hs2.prefill_shape(1, (1 << 21) - 1, 16, 128, 8, 8)
    assert f(ctypes.byref(big), FAKE, FAKE, FAKE, FAKE, None) == hs2.HS2_ERR_UNSUPPORTED
    s_bad = hs2.prefill_shape(1, 64, 16, 128, 1024, 1025)  # W + k > 2048
    assert f(ctypes.byref(s_bad), FAKE, FAKE, FAKE, FAKE, None) == hs2.HS2_ERR_UNSUPPORTED


def test_binding_fails_loudly_without_library(tmp_path):
    saved = hs2._lib
    hs2._lib = None
    try:
        with pytest.raises(RuntimeError, match="not built"):
            hs2.load(str(tmp_path / "missing.so"))
    finally:
        hs2._lib = saved


def test_binding_refuses_host_strided_mistyped_and_missized_tensors(lib):
    """The binding hands the library raw pointers; anything the kernels would
    misread (a host tensor, a strided view, another dtype, a wrong extent) is
    refused on the host before the call."""
    B, L, Hq, d, W, k = 1, 64, 16, 128, 8, 8
    q = torch.zeros(B, L, Hq, d, dtype=torch.bfloat16)
    kv = torch.zeros(B, L, d, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="q: must be a CUDA tensor"):
        hs2.hs2_full_attn_select(q, kv, kv, W, k)
    with pytest.raises(ValueError, match="q: must be contiguous"):
        hs2.hs2_full_attn_select(q.transpose(1, 2).contiguous().transpose(1, 2), kv, kv, W, k)
    with pytest.raises(ValueError, match="idx_a: must be a CUDA tensor"):
        idx = torch.zeros(B, L, W + k, dtype=torch.int32)
        hs2.hs2_selection_overlap(idx, idx, W, k)
    with pytest.raises(TypeError, match="idx_a: dtype torch.int64"):
        idx = torch.zeros(B, L, W + k, dtype=torch.int64)
        hs2.hs2_selection_overlap(idx, idx, W, k)
    with pytest.raises(ValueError, match="idx_a: 1088 elements, expected 1024"):
        idx = torch.zeros(B, L, W + k + 1, dtype=torch.int32)
        hs2.hs2_selection_overlap(idx, idx, W, k)
    with pytest.raises(TypeError, match="k_cache: dtype torch.bfloat16"):
        hs2._ptr(kv, "k_cache", hs2._kv_dtypes("e4m3"))
    assert hs2._kv_dtypes("bf16") == (torch.bfloat16,)
    with pytest.raises(TypeError, match="expected a torch.Tensor"):
        hs2._ptr([0], "k")
    assert hs2._ptr(None, "lse") is None


def test_binding_refuses_tensors_off_the_current_device(monkeypatch):
    """The library launches on the current device; a tensor on another GPU is
    refused on the host (checked here with the current device faked as 0)."""
    monkeypatch.setattr(hs2, "_current_device", lambda: 0)
    hs2._check_device("q", torch.device("cuda", 0))
    hs2._check_device("q", torch.device("cuda"))
    with pytest.raises(ValueError, match="q: on cuda:1 but the current device is cuda:0"):
        hs2._check_device("q", torch.device("cuda", 1))
    with pytest.raises(ValueError, match="k: must be a CUDA tensor"):
        hs2._check_device("k", torch.device("cpu"))


def test_bounded_wait_check_rejects_bad_limits(lib):
    # refused before anything is launched (no GPU is touched)
    assert lib.hs2_check_bounded_wait(0, None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_check_bounded_wait(1000001, None) == hs2.HS2_ERR_INVALID_ARG


def test_row_range_calls_reject_bad_ranges(lib):
    s = hs2.prefill_shape(1, 1000, 16, 128, 8, 8)
    for r0, r1 in [(-128, 128), (0, 0), (256, 128), (1, 128), (0, 100), (0, 1001), (128, 999)]:
        assert lib.hs2_full_attn_rows(ctypes.byref(s), r0, r1, FAKE, FAKE, FAKE, FAKE, FAKE,
                                      None) == hs2.HS2_ERR_INVALID_ARG, (r0, r1)
        assert lib.hs2_select_rows(ctypes.byref(s), r0, r1, FAKE, FAKE, FAKE, FAKE, FAKE,
                                   1 << 40, None) == hs2.HS2_ERR_INVALID_ARG, (r0, r1)
    # a range ending at L need not end on a 128-row boundary
    assert lib.hs2_select_rows(ctypes.byref(s), 896, 1000, FAKE, FAKE, FAKE, FAKE, FAKE, 16,
                               None) == hs2.HS2_ERR_WORKSPACE
