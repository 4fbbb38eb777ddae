"""Thin ctypes binding over libvattn.so: argument marshalling only.

Every function mirrors the C entry point of the same name in include/vattn.h.
Tensor arguments may be contiguous torch tensors (their data_ptr() is
passed; CUDA tensors for device pointers, host tensors for the host-buffer
entry point's q, k, v, o, lse) or raw integer addresses; `stream` defaults to
torch's current CUDA stream.
Every non-OK status raises VattnError.  There is no fallback: if the shared
library is missing the import of this module fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
# VATTN_DEBUG_BUILD=1 loads the debug build (device-side bounds checks; see
# build.py) instead of the default library.
LIB_PATH = os.path.join(_HERE, "libvattn_debug.so" if os.environ.get("VATTN_DEBUG_BUILD") == "1" else "libvattn.so")

VATTN_OK = 0
VATTN_ERR_INVALID_ARG = -1
VATTN_ERR_SHAPE = -2
VATTN_ERR_UNSUPPORTED = -3
VATTN_ERR_ALIGN = -4
VATTN_ERR_CUDA = -5
VATTN_ERR_DEVICE_TIMEOUT = -6
VATTN_ERR_WORKSPACE = -7
VATTN_ERR_DEVICE_BOUNDS = -8

VATTN_OP_DUAL_FWD = 1
VATTN_OP_STA_BWD = 2
VATTN_OP_DUAL_BWD = 3
VATTN_OP_DUAL_SYM_FWD = 4
VATTN_OP_DUAL_SYM_BWD = 5
VATTN_OP_STA_FWD_HOST = 6
VATTN_OP_HIER_FWD = 7
VATTN_OP_HIER_BWD = 8
VATTN_OP_STA_FWD_FP8 = 9
VATTN_OP_DUAL_FWD_FP8 = 10
VATTN_OP_DUAL_SYM_LEARNED_FWD = 11
VATTN_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024

VATTN_DEBUG_SKIP_ARRIVAL = 1


class VattnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"vattn error {code}: {msg}")
        self.code = code


class Geom(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("heads", ctypes.c_int64),
        ("head_dim", ctypes.c_int64),
        ("T", ctypes.c_int32),
        ("H", ctypes.c_int32),
        ("W", ctypes.c_int32),
        ("tile", ctypes.c_int32 * 3),
        ("window", ctypes.c_int32 * 3),
        ("pool", ctypes.c_int32 * 3),
    ]


def make_geom(batch: int, heads: int, head_dim: int, grid: Sequence[int], tile: Sequence[int],
              window: Sequence[int], pool: Sequence[int] = (1, 1, 1)) -> Geom:
    g = Geom()
    g.batch, g.heads, g.head_dim = batch, heads, head_dim
    g.T, g.H, g.W = grid
    g.tile[:] = list(tile)
    g.window[:] = list(window)
    g.pool[:] = list(pool)
    return g


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_INT = ctypes.c_int
_GP = ctypes.POINTER(Geom)

_SIGS = {
    "vattn_tile_permute": [_GP, _P, _P, _I64, _P],
    "vattn_tile_unpermute": [_GP, _P, _P, _I64, _P],
    "vattn_kept_tiles": [_GP, _P, _P],
    "vattn_sta_fwd": [_GP, _P, _P, _P, _F, _P, _P, _P],
    "vattn_pool_kv": [_GP, _P, _P, _P, _P, _P],
    "vattn_global_fwd": [_GP, _P, _P, _P, _F, _P, _P, _P],
    "vattn_dual_fwd": [_GP, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "vattn_sta_bwd": [_GP, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _SZ, _P],
    "vattn_dual_bwd": [_GP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _SZ, _P],
    "vattn_dual_fwd_noalloc": [_GP, _P, _P, _P, _P, _F, _P, _P],
    "vattn_xwin_fwd": [_GP, _INT, _P, _P, _P, _F, _P, _P, _P],
    "vattn_hier_fwd": [_GP, _P, _P, _P, _F, _P, _P, _P, _SZ, _P],
    "vattn_hier_bwd": [_GP, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _SZ, _P],
    "vattn_sta_fwd_raster": [_GP, _P, _P, _P, _F, _P, _P, _P],
    "vattn_dual_fwd_fp8": [_GP, _P, _P, _P, _P, _F, _P, _P, _SZ, _P],
    "vattn_sta_fwd_fp8": [_GP, _P, _P, _P, _F, _P, _P, _P, _SZ, _P],
    "vattn_sta_fwd_host": [_GP, _P, _P, _P, _F, _P, _P, _I64, _P, _SZ, _P],
    "vattn_dual_sym_fwd": [_GP, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "vattn_dual_sym_learned_fwd": [_GP, _P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _P, _SZ, _P],
    "vattn_dual_sym_bwd": [_GP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _SZ, _P],
    "vattn_xwin_bwd": [_GP, _INT, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _SZ, _P],
    "vattn_workspace_size": [_INT, _GP, ctypes.POINTER(_SZ)],
    "vattn_get_status": [_P],
    "vattn_last_error": [],
    "vattn_shutdown": [],
    "vattn_debug_set": [_INT, _I64],
    "vattn_debug_exp2": [_P, _P, _I64, _P],
    "vattn_debug_query_blocks": [_GP, _INT, _P, _I64, _P],
    "vattn_version": [],
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python video_dit_local_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, args in _SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name in ("vattn_last_error", "vattn_version") else ctypes.c_int
    return lib


lib = _load()


def _ptr(x) -> Optional[int]:
    """Device pointer argument: None, a raw address, or a contiguous CUDA tensor."""
    if x is None or isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("a device pointer argument got a host tensor: pass a CUDA tensor")
    if not x.is_contiguous():
        raise ValueError("tensor arguments must be contiguous (the library reads them as dense arrays)")
    return x.data_ptr()


def _hptr(x) -> Optional[int]:
    """Host pointer argument (vattn_sta_fwd_host's q, k, v, o, lse): None, a raw
    address, or a contiguous host tensor."""
    if x is None or isinstance(x, int):
        return x
    if x.is_cuda:
        raise ValueError("a host pointer argument got a CUDA tensor: pass host (ideally pinned) memory")
    if not x.is_contiguous():
        raise ValueError("tensor arguments must be contiguous (the library reads them as dense arrays)")
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    if torch.cuda.is_available():
        return torch.cuda.current_stream().cuda_stream
    return None


def _check(code: int) -> None:
    if code != VATTN_OK:
        raise VattnError(code, lib.vattn_last_error().decode())


def _row_bytes(t) -> int:
    return t.shape[-1] * t.element_size() if t.dim() == 4 else t.element_size()


def vattn_tile_permute(geom: Geom, src, dst, row_bytes: Optional[int] = None, stream=None) -> None:
    rb = _row_bytes(src) if row_bytes is None else row_bytes
    _check(lib.vattn_tile_permute(ctypes.byref(geom), _ptr(src), _ptr(dst), rb, _stream(stream)))


def vattn_tile_unpermute(geom: Geom, src, dst, row_bytes: Optional[int] = None, stream=None) -> None:
    rb = _row_bytes(src) if row_bytes is None else row_bytes
    _check(lib.vattn_tile_unpermute(ctypes.byref(geom), _ptr(src), _ptr(dst), rb, _stream(stream)))


def vattn_kept_tiles(geom: Geom, out, stream=None) -> None:
    _check(lib.vattn_kept_tiles(ctypes.byref(geom), _ptr(out), _stream(stream)))


def vattn_sta_fwd(geom: Geom, q, k, v, scale: float, o, lse=None, stream=None) -> None:
    _check(lib.vattn_sta_fwd(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), scale, _ptr(o), _ptr(lse),
                             _stream(stream)))


def vattn_xwin_fwd(geom: Geom, shifted: int, q, k, v, scale: float, o, lse=None, stream=None) -> None:
    _check(lib.vattn_xwin_fwd(ctypes.byref(geom), int(shifted), _ptr(q), _ptr(k), _ptr(v), scale, _ptr(o), _ptr(lse),
                              _stream(stream)))


def vattn_xwin_bwd(geom: Geom, shifted: int, q, k, v, o, lse, dout, scale: float, dq, dk, dv, workspace,
                   ws_bytes: int = 0, stream=None) -> None:
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_xwin_bwd(ctypes.byref(geom), int(shifted), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                              _ptr(dout), scale, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes,
                              _stream(stream)))


def vattn_dual_sym_fwd(geom: Geom, q, k, v, g, scale: float, o, o_l=None, lse_l=None, qp=None, kp=None, vp=None,
                       o_p=None, lse_p=None, workspace=None, ws_bytes: int = 0, stream=None) -> None:
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_dual_sym_fwd(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(g), scale, _ptr(o), _ptr(o_l),
                                  _ptr(lse_l), _ptr(qp), _ptr(kp), _ptr(vp), _ptr(o_p), _ptr(lse_p), _ptr(workspace),
                                  ws_bytes, _stream(stream)))


def vattn_dual_sym_learned_fwd(geom: Geom, q, k, v, g, wq, wk, wv, w3, scale: float, o, workspace,
                               ws_bytes: int = 0, stream=None) -> None:
    """Learned compressed global branch (inference): weights fp32, taps-major
    ([heads, p_t*p_h*p_w, d] for wq/wk/wv, [heads, 27, d] for w3)."""
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_dual_sym_learned_fwd(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(wq), _ptr(wk),
                                          _ptr(wv), _ptr(w3), scale, _ptr(o), _ptr(workspace), ws_bytes,
                                          _stream(stream)))


def vattn_dual_sym_bwd(geom: Geom, q, k, v, g, o_l, lse_l, qp, kp, vp, o_p, lse_p, dout, scale: float, dq, dk, dv,
                       workspace, ws_bytes: int = 0, stream=None) -> None:
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_dual_sym_bwd(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o_l), _ptr(lse_l),
                                  _ptr(qp), _ptr(kp), _ptr(vp), _ptr(o_p), _ptr(lse_p), _ptr(dout), scale, _ptr(dq),
                                  _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, _stream(stream)))


def vattn_hier_fwd(geom: Geom, q, k, v, scale: float, o, lse=None, workspace=None, ws_bytes: int = 0,
                   stream=None) -> None:
    """Hierarchical local attention (geom.pool = the medium pool factor)."""
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_hier_fwd(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), scale, _ptr(o), _ptr(lse),
                              _ptr(workspace), ws_bytes, _stream(stream)))


def vattn_hier_bwd(geom: Geom, q, k, v, o, lse, dout, scale: float, dq, dk, dv, workspace, ws_bytes: int = 0,
                   stream=None) -> None:
    """Backward of vattn_hier_fwd (geom.pool = the medium pool factor)."""
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_hier_bwd(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), scale,
                              _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, _stream(stream)))


def vattn_sta_fwd_raster(geom: Geom, q, k, v, scale: float, o, lse=None, stream=None) -> None:
    """Sliding-tile forward on raster-order tensors (reorder fused into the kernel)."""
    _check(lib.vattn_sta_fwd_raster(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), scale, _ptr(o), _ptr(lse),
                                    _stream(stream)))


def vattn_dual_fwd_fp8(geom: Geom, q, k, v, g, scale: float, o, workspace, ws_bytes: int = 0, stream=None) -> None:
    """Dual forward with e4m3 Q*K^T in both branches (inference)."""
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_dual_fwd_fp8(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(g), scale, _ptr(o),
                                  _ptr(workspace), ws_bytes, _stream(stream)))


def vattn_sta_fwd_fp8(geom: Geom, q, k, v, scale: float, o, lse=None, workspace=None, ws_bytes: int = 0,
                      stream=None) -> None:
    """Sliding-tile forward with e4m3 Q*K^T (per-head absmax scales), bf16 P*V."""
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_sta_fwd_fp8(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), scale, _ptr(o), _ptr(lse),
                                 _ptr(workspace), ws_bytes, _stream(stream)))


def vattn_sta_fwd_host(geom: Geom, q, k, v, scale: float, o, lse, chunk_slices: int, workspace,
                       ws_bytes: int = 0, stream=None) -> None:
    """Host-buffer sliding-tile forward with copies overlapped by chunks of
    batch*head slices (q, k, v, o, lse: host tensors / addresses, raster)."""
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_sta_fwd_host(ctypes.byref(geom), _hptr(q), _hptr(k), _hptr(v), scale, _hptr(o), _hptr(lse),
                                  int(chunk_slices), _ptr(workspace), ws_bytes, _stream(stream)))


def vattn_pool_kv(geom: Geom, k, v, kp, vp, stream=None) -> None:
    _check(lib.vattn_pool_kv(ctypes.byref(geom), _ptr(k), _ptr(v), _ptr(kp), _ptr(vp), _stream(stream)))


def vattn_global_fwd(geom: Geom, q, kp, vp, scale: float, o, lse=None, stream=None) -> None:
    _check(lib.vattn_global_fwd(ctypes.byref(geom), _ptr(q), _ptr(kp), _ptr(vp), scale, _ptr(o), _ptr(lse),
                                _stream(stream)))


def vattn_dual_fwd(geom: Geom, q, k, v, g, scale: float, o, o_l=None, lse_l=None, o_g=None, lse_g=None,
                   kp=None, vp=None, workspace=None, ws_bytes: int = 0, stream=None) -> None:
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_dual_fwd(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(g), scale, _ptr(o), _ptr(o_l),
                              _ptr(lse_l), _ptr(o_g), _ptr(lse_g), _ptr(kp), _ptr(vp), _ptr(workspace), ws_bytes,
                              _stream(stream)))


def vattn_dual_fwd_noalloc(geom: Geom, q, k, v, g, scale: float, o, stream=None) -> None:
    """vattn_dual_fwd for callers that cannot allocate: the workspace is the
    library's own static device scratch (VATTN_NOALLOC_SCRATCH_BYTES)."""
    _check(lib.vattn_dual_fwd_noalloc(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(g), scale, _ptr(o),
                                      _stream(stream)))


def vattn_sta_bwd(geom: Geom, q, k, v, o, lse, dout, scale: float, dq, dk, dv, workspace, ws_bytes: int = 0,
                  stream=None) -> None:
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_sta_bwd(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), scale,
                             _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, _stream(stream)))


def vattn_dual_bwd(geom: Geom, q, k, v, g, o_l, lse_l, o_g, lse_g, kp, vp, dout, scale: float, dq, dk, dv,
                   dg=None, workspace=None, ws_bytes: int = 0, stream=None) -> None:
    if workspace is not None and not ws_bytes:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.vattn_dual_bwd(ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o_l), _ptr(lse_l),
                              _ptr(o_g), _ptr(lse_g), _ptr(kp), _ptr(vp), _ptr(dout), scale, _ptr(dq), _ptr(dk),
                              _ptr(dv), _ptr(dg), _ptr(workspace), ws_bytes, _stream(stream)))


def vattn_workspace_size(op: int, geom: Geom) -> int:
    n = _SZ(0)
    _check(lib.vattn_workspace_size(op, ctypes.byref(geom), ctypes.byref(n)))
    return n.value


def vattn_get_status(stream=None) -> int:
    """Returns the status code (does not raise)."""
    return lib.vattn_get_status(_stream(stream))


def vattn_last_error() -> str:
    return lib.vattn_last_error().decode()


def vattn_shutdown() -> None:
    """Releases the host pipeline's library streams and events on every device."""
    _check(lib.vattn_shutdown())


def vattn_debug_set(flags: int, timeout_ns: int = 0) -> None:
    _check(lib.vattn_debug_set(flags, timeout_ns))


def vattn_debug_exp2(x, y, n: Optional[int] = None, stream=None) -> None:
    _check(lib.vattn_debug_exp2(_ptr(x), _ptr(y), x.numel() if n is None else n, _stream(stream)))


def vattn_debug_query_blocks(geom: Geom, window_mode: int):
    """Host-side query-block plan of the sliding-tile forward: an int32 tensor
    [n_blocks, 4] = (first tile-major row, rows that exist, straddle flag,
    tile of the key stream).  window_mode: 0 sliding, 1 partition, 2 shifted."""
    import torch
    n = ctypes.c_int64(0)
    _check(lib.vattn_debug_query_blocks(ctypes.byref(geom), window_mode, None, 0, ctypes.byref(n)))
    out = torch.empty((n.value, 4), dtype=torch.int32)
    _check(lib.vattn_debug_query_blocks(ctypes.byref(geom), window_mode, _hptr(out), n.value, ctypes.byref(n)))
    return out


def vattn_version() -> str:
    return lib.vattn_version().decode()
