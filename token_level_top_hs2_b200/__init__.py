"""B200 (sm_100a) library for HySparse2's token-level KV Reuse hot path.

Python binding of the C ABI in include/hs2.h, argument marshalling only: every
step of the computation runs in the CUDA kernels of libhs2.so.  PyTorch is used
for device memory and streams.  Loading fails loudly when the library is
missing; there is no CPU fallback.

Entry points (same names as the C ABI):
  hs2_full_attn_select  full-attention layer + window/top-k selection (prefill)
  hs2_sparse_attn       sparse layer over the inherited selection (prefill)
  hs2_decode_select     decode full layer + selection, split over the cache
  hs2_decode_sparse     decode sparse layer over the inherited selection
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhs2.so")

HS2_OK = 0
HS2_ERR_INVALID_ARG = 1
HS2_ERR_UNSUPPORTED = 2
HS2_ERR_WORKSPACE = 3
HS2_ERR_CUDA = 4
HS2_ERR_DEVICE_DATA = 5
HS2_ERR_TIMEOUT = 6
HS2_KV_BF16 = 0
HS2_KV_E4M3 = 1

EXPORTED = [
    "hs2_status_string", "hs2_version", "hs2_full_attn_select_workspace",
    "hs2_full_attn_select", "hs2_sparse_attn", "hs2_decode_select_workspace",
    "hs2_decode_select", "hs2_decode_sparse", "hs2_get_last_device_error",
    "hs2_decode_select_noalloc", "hs2_selection_overlap",
    "hs2_full_attn_select_blocks_workspace", "hs2_full_attn_select_blocks",
    "hs2_decode_stage_workspace", "hs2_decode_stage", "hs2_decode_sparse_staged",
    "hs2_full_attn", "hs2_select", "hs2_check_bounded_wait", "hs2_full_attn_rows",
    "hs2_select_rows",
]


class Hs2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class PrefillShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("L", ctypes.c_int), ("Hq", ctypes.c_int),
                ("d", ctypes.c_int), ("W", ctypes.c_int), ("k", ctypes.c_int),
                ("scale", ctypes.c_float)]


class DecodeShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Tmax", ctypes.c_int), ("Hq", ctypes.c_int),
                ("d", ctypes.c_int), ("W", ctypes.c_int), ("k", ctypes.c_int),
                ("scale", ctypes.c_float), ("kv", ctypes.c_int)]


_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libhs2.so (built by token_level_top_hs2_b200/build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"hs2 CUDA library not built: {path} is missing "
                           "(run python token_level_top_hs2_b200/build.py)")
    L = ctypes.CDLL(path)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    P, D = ctypes.POINTER(PrefillShape), ctypes.POINTER(DecodeShape)
    L.hs2_status_string.argtypes = [i32]
    L.hs2_status_string.restype = ctypes.c_char_p
    L.hs2_version.argtypes = []
    L.hs2_version.restype = i32
    L.hs2_full_attn_select_workspace.argtypes = [P]
    L.hs2_full_attn_select_workspace.restype = sz
    L.hs2_full_attn_select.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.hs2_full_attn_select.restype = i32
    L.hs2_full_attn.argtypes = [P, vp, vp, vp, vp, vp, vp]
    L.hs2_full_attn.restype = i32
    L.hs2_select.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
    L.hs2_select.restype = i32
    L.hs2_full_attn_rows.argtypes = [P, i32, i32, vp, vp, vp, vp, vp, vp]
    L.hs2_full_attn_rows.restype = i32
    L.hs2_select_rows.argtypes = [P, i32, i32, vp, vp, vp, vp, vp, sz, vp]
    L.hs2_select_rows.restype = i32
    L.hs2_full_attn_select_blocks_workspace.argtypes = [P, i32]
    L.hs2_full_attn_select_blocks_workspace.restype = sz
    L.hs2_full_attn_select_blocks.argtypes = [P, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.hs2_full_attn_select_blocks.restype = i32
    L.hs2_sparse_attn.argtypes = [P, vp, vp, vp, i32, vp, vp, vp, vp, vp]
    L.hs2_sparse_attn.restype = i32
    L.hs2_decode_select_workspace.argtypes = [D]
    L.hs2_decode_select_workspace.restype = sz
    L.hs2_decode_select.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.hs2_decode_select.restype = i32
    L.hs2_decode_sparse.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.hs2_decode_sparse.restype = i32
    L.hs2_decode_select_noalloc.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.hs2_decode_select_noalloc.restype = i32
    L.hs2_decode_stage_workspace.argtypes = [D]
    L.hs2_decode_stage_workspace.restype = sz
    L.hs2_decode_stage.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.hs2_decode_stage.restype = i32
    L.hs2_decode_sparse_staged.argtypes = [D, vp, vp, vp, vp]
    L.hs2_decode_sparse_staged.restype = i32
    L.hs2_selection_overlap.argtypes = [P, vp, vp, vp, vp, vp]
    L.hs2_selection_overlap.restype = i32
    L.hs2_check_bounded_wait.argtypes = [ctypes.c_uint, vp]
    L.hs2_check_bounded_wait.restype = i32
    L.hs2_get_last_device_error.argtypes = [vp]
    L.hs2_get_last_device_error.restype = i32
    _lib = L
    return L


def status_string(status: int) -> str:
    return load().hs2_status_string(status).decode()


_BF16 = (torch.bfloat16,)
_F32 = (torch.float32,)
_I32 = (torch.int32,)


def _ptr(t: Optional[torch.Tensor], name: str = "tensor", dtypes=None, numel=None):
    """Device pointer of a dense CUDA tensor; None stays None (the library
    rejects a missing required pointer itself).

    The kernels read each argument as a dense row-major array of the type and
    extent the C header gives, so a host tensor, a tensor on a CUDA device other
    than the current one, a strided view, another dtype or a buffer of the
    wrong size is refused here instead of being misread or overrun on the
    device."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous (dense, row-major)")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {' or '.join(map(str, dtypes))}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name}: {t.numel()} elements, expected {numel}")
    _check_device(name, t.device)
    return ctypes.c_void_p(t.data_ptr())


def _current_device() -> int:
    return torch.cuda.current_device()


def _check_device(name: str, device: torch.device) -> None:
    """The library launches on the current CUDA device (the one cudaGetDevice
    names) and builds its tensor maps there, so every tensor of a call must
    live on that device: a pointer into another GPU's memory would reach this
    GPU's kernels, which without peer access is an illegal address."""
    if device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor, got device '{device}'")
    cur = _current_device()
    if device.index is not None and device.index != cur:
        raise ValueError(f"{name}: on cuda:{device.index} but the current device is cuda:{cur}; "
                         "make its device current (torch.cuda.device) or move the tensor")


def _kv_dtypes(kv):
    """Element types of K/V storage: bf16 values, or e4m3 codes (as uint8 or
    float8_e4m3fn)."""
    return _BF16 if _kv_code(kv) == HS2_KV_BF16 else (torch.uint8, torch.float8_e4m3fn)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, what: str):
    if status != HS2_OK:
        raise Hs2Error(status, what)


def _kv_code(kv) -> int:
    if kv in (HS2_KV_BF16, "bf16"):
        return HS2_KV_BF16
    if kv in (HS2_KV_E4M3, "e4m3"):
        return HS2_KV_E4M3
    raise ValueError(f"kv must be 'bf16' or 'e4m3', got {kv!r}")


def _u8(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t


def prefill_shape(B, L, Hq, d, W, k, scale=None) -> PrefillShape:
    return PrefillShape(B, L, Hq, d, W, k, 1.0 / math.sqrt(d) if scale is None else scale)


def decode_shape(B, Tmax, Hq, d, W, k, kv="e4m3", scale=None) -> DecodeShape:
    return DecodeShape(B, Tmax, Hq, d, W, k, 1.0 / math.sqrt(d) if scale is None else scale,
                       _kv_code(kv))


def hs2_full_attn_select_workspace(shape: PrefillShape) -> int:
    return load().hs2_full_attn_select_workspace(ctypes.byref(shape))


def hs2_full_attn_select(q, k, v, W: int, k_top: int, *, scale=None, o=None, lse=None, idx=None,
                         workspace=None, want_lse: bool = True, stream=None):
    """q [B,L,Hq,d] bf16, k/v [B,L,d] bf16 (CUDA).  Returns (o, lse or None, idx)."""
    B, L, Hq, d = q.shape
    shape = prefill_shape(B, L, Hq, d, W, k_top, scale)
    dev = q.device
    o = torch.empty_like(q) if o is None else o
    if lse is None and want_lse:
        lse = torch.empty(B, L, Hq, dtype=torch.float32, device=dev)
    idx = torch.empty(B, L, W + k_top, dtype=torch.int32, device=dev) if idx is None else idx
    need = hs2_full_attn_select_workspace(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    n, nh = B * L * d, B * L * Hq
    st = load().hs2_full_attn_select(ctypes.byref(shape), _ptr(q, "q", _BF16),
                                     _ptr(k, "k", _BF16, n), _ptr(v, "v", _BF16, n),
                                     _ptr(o, "o", _BF16, nh * d), _ptr(lse, "lse", _F32, nh),
                                     _ptr(idx, "idx", _I32, B * L * (W + k_top)),
                                     _ptr(workspace, "workspace"),
                                     workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "hs2_full_attn_select")
    return o, lse, idx


def hs2_full_attn(q, k, v, *, W: int = 1, k_top: int = 0, scale=None, o=None, lse=None,
                  stream=None):
    """Exact causal attention only (O and lse).  Returns (o, lse)."""
    B, L, Hq, d = q.shape
    shape = prefill_shape(B, L, Hq, d, W, k_top, scale)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty(B, L, Hq, dtype=torch.float32, device=q.device) if lse is None else lse
    n, nh = B * L * d, B * L * Hq
    st = load().hs2_full_attn(ctypes.byref(shape), _ptr(q, "q", _BF16), _ptr(k, "k", _BF16, n),
                              _ptr(v, "v", _BF16, n), _ptr(o, "o", _BF16, nh * d),
                              _ptr(lse, "lse", _F32, nh), _stream(stream))
    _check(st, "hs2_full_attn")
    return o, lse


def hs2_select(q, k, lse, W: int, k_top: int, *, scale=None, idx=None, workspace=None,
               stream=None):
    """The selection from q, k and the lse of hs2_full_attn.  Returns idx."""
    B, L, Hq, d = q.shape
    shape = prefill_shape(B, L, Hq, d, W, k_top, scale)
    idx = torch.empty(B, L, W + k_top, dtype=torch.int32, device=q.device) if idx is None else idx
    need = hs2_full_attn_select_workspace(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = load().hs2_select(ctypes.byref(shape), _ptr(q, "q", _BF16),
                           _ptr(k, "k", _BF16, B * L * d), _ptr(lse, "lse", _F32, B * L * Hq),
                           _ptr(idx, "idx", _I32, B * L * (W + k_top)),
                           _ptr(workspace, "workspace"),
                           workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "hs2_select")
    return idx


def hs2_full_attn_rows(q, k, v, row0: int, row1: int, *, o, lse, W: int = 1, k_top: int = 0,
                       scale=None, stream=None):
    """hs2_full_attn for query rows [row0, row1) of every sequence, into the
    full-size o [B,L,Hq,d] and lse [B,L,Hq]; reads K/V rows 0..row1-1."""
    B, L, Hq, d = q.shape
    shape = prefill_shape(B, L, Hq, d, W, k_top, scale)
    n, nh = B * L * d, B * L * Hq
    st = load().hs2_full_attn_rows(ctypes.byref(shape), row0, row1, _ptr(q, "q", _BF16),
                                   _ptr(k, "k", _BF16, n), _ptr(v, "v", _BF16, n),
                                   _ptr(o, "o", _BF16, nh * d), _ptr(lse, "lse", _F32, nh),
                                   _stream(stream))
    _check(st, "hs2_full_attn_rows")
    return o, lse


def hs2_select_rows(q, k, lse, W: int, k_top: int, row0: int, row1: int, *, idx, workspace,
                    scale=None, stream=None):
    """hs2_select for query rows [row0, row1) of every sequence, into the
    full-size idx [B,L,W+k]."""
    B, L, Hq, d = q.shape
    shape = prefill_shape(B, L, Hq, d, W, k_top, scale)
    st = load().hs2_select_rows(ctypes.byref(shape), row0, row1, _ptr(q, "q", _BF16),
                                _ptr(k, "k", _BF16, B * L * d), _ptr(lse, "lse", _F32, B * L * Hq),
                                _ptr(idx, "idx", _I32, B * L * (W + k_top)),
                                _ptr(workspace, "workspace"),
                                workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "hs2_select_rows")
    return idx


def hs2_full_attn_select_blocks_workspace(shape: PrefillShape, block: int = 64) -> int:
    return load().hs2_full_attn_select_blocks_workspace(ctypes.byref(shape), block)


def hs2_full_attn_select_blocks(q, k, v, W: int, k_top: int, *, block: int = 64, scale=None,
                                o=None, lse=None, idx=None, workspace=None, want_lse: bool = True,
                                stream=None):
    """Block-level selector variant (HySparse): as hs2_full_attn_select, with the
    k_top global tokens taken as k_top/block whole blocks of largest attention mass."""
    B, L, Hq, d = q.shape
    shape = prefill_shape(B, L, Hq, d, W, k_top, scale)
    dev = q.device
    o = torch.empty_like(q) if o is None else o
    if lse is None and want_lse:
        lse = torch.empty(B, L, Hq, dtype=torch.float32, device=dev)
    idx = torch.empty(B, L, W + k_top, dtype=torch.int32, device=dev) if idx is None else idx
    need = hs2_full_attn_select_blocks_workspace(shape, block)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    n, nh = B * L * d, B * L * Hq
    st = load().hs2_full_attn_select_blocks(ctypes.byref(shape), block, _ptr(q, "q", _BF16),
                                            _ptr(k, "k", _BF16, n), _ptr(v, "v", _BF16, n),
                                            _ptr(o, "o", _BF16, nh * d),
                                            _ptr(lse, "lse", _F32, nh),
                                            _ptr(idx, "idx", _I32, B * L * (W + k_top)),
                                            _ptr(workspace, "workspace"),
                                            workspace.numel() * workspace.element_size(),
                                            _stream(stream))
    _check(st, "hs2_full_attn_select_blocks")
    return o, lse, idx


def hs2_sparse_attn(q, k, v, idx, *, kv="bf16", k_scale=None, v_scale=None, W=None, k_top=None,
                    scale=None, o=None, stream=None):
    """q [B,L,Hq,d] bf16; k/v [B,L,d] bf16 or e4m3 codes; idx [B,L,S]. Returns o."""
    B, L, Hq, d = q.shape
    S = idx.shape[-1]
    if W is None:
        W, k_top = 1, S - 1
    shape = prefill_shape(B, L, Hq, d, W, k_top, scale)
    o = torch.empty_like(q) if o is None else o
    n, kvd = B * L * d, _kv_dtypes(kv)
    st = load().hs2_sparse_attn(ctypes.byref(shape), _ptr(q, "q", _BF16),
                                _ptr(_u8(k), "k", kvd, n), _ptr(_u8(v), "v", kvd, n),
                                _kv_code(kv), _ptr(k_scale, "k_scale", _F32, B * L),
                                _ptr(v_scale, "v_scale", _F32, B * L),
                                _ptr(idx, "idx", _I32, B * L * (W + k_top)),
                                _ptr(o, "o", _BF16, q.numel()), _stream(stream))
    _check(st, "hs2_sparse_attn")
    return o


def hs2_decode_select_workspace(shape: DecodeShape) -> int:
    return load().hs2_decode_select_workspace(ctypes.byref(shape))


def hs2_decode_select(q, k_cache, v_cache, lengths, W: int, k_top: int, *, kv="e4m3",
                      k_scale=None, v_scale=None, scale=None, o=None, lse=None, idx=None,
                      workspace=None, want_lse: bool = True, stream=None):
    """q [B,Hq,d] bf16; caches [B,Tmax,d]; lengths [B] int32 (CUDA). Returns (o, lse, idx)."""
    B, Hq, d = q.shape
    Tmax = k_cache.shape[1]
    shape = decode_shape(B, Tmax, Hq, d, W, k_top, kv, scale)
    dev = q.device
    o = torch.empty_like(q) if o is None else o
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    idx = torch.empty(B, W + k_top, dtype=torch.int32, device=dev) if idx is None else idx
    need = hs2_decode_select_workspace(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    n, kvd = B * Tmax * d, _kv_dtypes(kv)
    st = load().hs2_decode_select(ctypes.byref(shape), _ptr(q, "q", _BF16),
                                  _ptr(_u8(k_cache), "k_cache", kvd, n),
                                  _ptr(_u8(v_cache), "v_cache", kvd, n),
                                  _ptr(k_scale, "k_scale", _F32, B * Tmax),
                                  _ptr(v_scale, "v_scale", _F32, B * Tmax),
                                  _ptr(lengths, "lengths", _I32, B),
                                  _ptr(o, "o", _BF16, q.numel()), _ptr(lse, "lse", _F32, B * Hq),
                                  _ptr(idx, "idx", _I32, B * (W + k_top)),
                                  _ptr(workspace, "workspace"),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "hs2_decode_select")
    return o, lse, idx


def hs2_decode_sparse(q, k_cache, v_cache, lengths, idx, *, kv="e4m3", k_scale=None,
                      v_scale=None, W=None, k_top=None, scale=None, o=None, stream=None):
    """q [B,Hq,d] bf16; idx [B,S] int32. Returns o [B,Hq,d] bf16."""
    B, Hq, d = q.shape
    Tmax = k_cache.shape[1]
    S = idx.shape[-1]
    if W is None:
        W, k_top = 1, S - 1
    shape = decode_shape(B, Tmax, Hq, d, W, k_top, kv, scale)
    o = torch.empty_like(q) if o is None else o
    n, kvd = B * Tmax * d, _kv_dtypes(kv)
    st = load().hs2_decode_sparse(ctypes.byref(shape), _ptr(q, "q", _BF16),
                                  _ptr(_u8(k_cache), "k_cache", kvd, n),
                                  _ptr(_u8(v_cache), "v_cache", kvd, n),
                                  _ptr(k_scale, "k_scale", _F32, B * Tmax),
                                  _ptr(v_scale, "v_scale", _F32, B * Tmax),
                                  _ptr(lengths, "lengths", _I32, B),
                                  _ptr(idx, "idx", _I32, B * (W + k_top)),
                                  _ptr(o, "o", _BF16, q.numel()), _stream(stream))
    _check(st, "hs2_decode_sparse")
    return o


def hs2_selection_overlap(idx_a, idx_b, W: int, k_top: int, *, inter=None, ratio=None,
                          stream=None):
    """idx_a, idx_b [B,L,W+k] int32 selections. Returns (inter [B,L] int32, ratio [B,L] fp32):
    per query row the number of global picks the two share and that number over
    min(k, t-W+1)."""
    B, L, S = idx_a.shape
    # head count, head dim and scale do not enter the overlap; any valid values do
    shape = prefill_shape(B, L, 16, 128, W, k_top)
    dev = idx_a.device
    inter = torch.empty(B, L, dtype=torch.int32, device=dev) if inter is None else inter
    ratio = torch.empty(B, L, dtype=torch.float32, device=dev) if ratio is None else ratio
    S = W + k_top
    st = load().hs2_selection_overlap(ctypes.byref(shape), _ptr(idx_a, "idx_a", _I32, B * L * S),
                                      _ptr(idx_b, "idx_b", _I32, B * L * S),
                                      _ptr(inter, "inter", _I32, B * L),
                                      _ptr(ratio, "ratio", _F32, B * L), _stream(stream))
    _check(st, "hs2_selection_overlap")
    return inter, ratio


def hs2_decode_stage(k_cache, v_cache, lengths, idx, *, Hq: int, W: int, k_top: int,
                     kv="e4m3", k_scale=None, v_scale=None, staged=None, stream=None):
    """Stage the selected rows once for the decode sparse layers.  Returns the
    staged buffer (uint8, CUDA)."""
    B, Tmax, d = k_cache.shape
    shape = decode_shape(B, Tmax, Hq, d, W, k_top, kv)
    need = load().hs2_decode_stage_workspace(ctypes.byref(shape))
    if staged is None:
        staged = torch.empty(max(need, 16), dtype=torch.uint8, device=k_cache.device)
    n, kvd = B * Tmax * d, _kv_dtypes(kv)
    st = load().hs2_decode_stage(ctypes.byref(shape), _ptr(_u8(k_cache), "k_cache", kvd, n),
                                 _ptr(_u8(v_cache), "v_cache", kvd, n),
                                 _ptr(k_scale, "k_scale", _F32, B * Tmax),
                                 _ptr(v_scale, "v_scale", _F32, B * Tmax),
                                 _ptr(lengths, "lengths", _I32, B),
                                 _ptr(idx, "idx", _I32, B * (W + k_top)),
                                 _ptr(staged, "staged"), staged.numel() * staged.element_size(),
                                 _stream(stream))
    _check(st, "hs2_decode_stage")
    return staged


def hs2_decode_sparse_staged(q, staged, Tmax: int, W: int, k_top: int, *, kv="e4m3",
                             scale=None, o=None, stream=None):
    """One decode sparse layer over staged rows.  q [B,Hq,d] bf16. Returns o."""
    B, Hq, d = q.shape
    shape = decode_shape(B, Tmax, Hq, d, W, k_top, kv, scale)
    o = torch.empty_like(q) if o is None else o
    st = load().hs2_decode_sparse_staged(ctypes.byref(shape), _ptr(q, "q", _BF16),
                                         _ptr(staged, "staged"),
                                         _ptr(o, "o", _BF16, q.numel()), _stream(stream))
    _check(st, "hs2_decode_sparse_staged")
    return o


def hs2_check_bounded_wait(limit_us: int = 1000, stream=None) -> None:
    """Launch the check of the bounded in-kernel wait: one thread waits on a
    barrier nothing arrives at and gives up after limit_us microseconds; the
    next hs2_get_last_device_error() then returns HS2_ERR_TIMEOUT."""
    _check(load().hs2_check_bounded_wait(limit_us, _stream(stream)), "hs2_check_bounded_wait")


def hs2_get_last_device_error(stream=None) -> int:
    """Synchronise the stream and return the first pending device-side status."""
    return load().hs2_get_last_device_error(_stream(stream))
