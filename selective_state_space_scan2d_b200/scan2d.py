"""ctypes binding of the C ABI in include/scan2d.h (libscan2d_b200.so, built in-tree).

Argument marshalling only: every step of the scan runs in the CUDA library.  There is no
CPU path; importing this module without the built library raises ImportError.

    y = scan2d_fwd(x, delta, A, B, C, Dskip)          # torch CUDA tensors, y allocated
    scan2d_fwd(x, delta, A, B, C, Dskip, y=y)         # into a caller-provided y

Tensor layouts (contiguous): x, delta (batch, D, H, W) fp32 or bf16; A (D, N) fp32;
B, C (batch, K, N, H, W) or (batch, N, H, W) for K = 1, dtype of x; Dskip (D,) fp32 or None.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libscan2d_b200.so")

if not os.path.exists(lib_path):
    raise ImportError(
        f"{lib_path} is missing: build it with `python -m selective_state_space_scan2d_b200.build` "
        "(the 2D scan has no CPU fallback)")

_lib = ctypes.CDLL(lib_path)

_vp, _i, _u, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
_lib.scan2d_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _u, _vp]
_lib.scan2d_fwd.restype = _i
_lib.scan2d_fwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _u, _vp]
_lib.scan2d_fwd_noalloc.restype = _i
_lib.scan2d_query_plan.argtypes = [_i, _i, _i, _i, _i, _u, ctypes.POINTER(ctypes.c_longlong), _i]
_lib.scan2d_query_plan.restype = _i
_lib.scan2d_host_staging_bytes.argtypes = [_i, _i, _i, _i, _i, _u]
_lib.scan2d_host_staging_bytes.restype = _sz
_lib.scan2d_fwd_host.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i, _i, _i, _i, _i, _u, _vp]
_lib.scan2d_fwd_host.restype = _i
_lib.scan2d_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                            _i, _i, _i, _i, _i, _u, _vp]
_lib.scan2d_bwd.restype = _i
_lib.scan2d_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _u]
_lib.scan2d_bwd_workspace_bytes.restype = _sz
_lib.scan2d_grid_cells.argtypes = [_vp, _i, _i, _i, _vp, _vp, _vp]
_lib.scan2d_grid_cells.restype = _i
_lib.scan2d_grid_gather.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _u, _vp]
_lib.scan2d_grid_gather.restype = _i
_lib.scan2d_fwd_wsi.argtypes = [_vp] * 9 + [_i, _i, _i, _i, _i, _u, _vp]
_lib.scan2d_fwd_wsi.restype = _i
_lib.scan2d_proj.argtypes = [_vp] * 7 + [_i, _i, _i, _i, _i, _i, _u, _vp]
_lib.scan2d_proj.restype = _i
_lib.scan2d_get_device_error.argtypes = [_vp]
_lib.scan2d_get_device_error.restype = _i
_lib.scan2d_strerror.argtypes = [_i]
_lib.scan2d_strerror.restype = ctypes.c_char_p
_lib.scan2d_version.argtypes = []
_lib.scan2d_version.restype = _i

# flags (include/scan2d.h)
SCAN2D_BF16 = 0x1
SCAN2D_OUT_F32 = 0x2
SCAN2D_VFIRST = 0x8
SCAN2D_OR_TL = 0x10
SCAN2D_OR_TR = 0x20
SCAN2D_OR_BL = 0x40
SCAN2D_OR_BR = 0x80
SCAN2D_E_SCRATCH = -11
SCAN2D_E_WORKSPACE = -12
SCAN2D_NOALLOC_SCRATCH_BYTES = 32 << 20
SCAN2D_BWD_MAX_N = 16
SCAN2D_PROJ_MAX_R = 32


class Scan2dError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {scan2d_strerror(code)} (code {code})")


def scan2d_strerror(code: int) -> str:
    return _lib.scan2d_strerror(int(code)).decode()


def scan2d_version() -> int:
    return int(_lib.scan2d_version())


def flags_for(bf16: bool, orient_mask: int = 1, out_f32: bool = False, vfirst: bool = False) -> int:
    """Flag word for an element type, a 4-bit orientation mask (bit0 TL .. bit3 BR) and the
    scan order (vfirst: vertical scan first)."""
    f = (SCAN2D_BF16 if bf16 else 0) | ((orient_mask & 0xF) << 4)
    if out_f32:
        f |= SCAN2D_OUT_F32
    if vfirst:
        f |= SCAN2D_VFIRST
    return f


def _torch():
    import torch
    return torch


def _stream_handle(stream):
    if stream is None:
        return _torch().cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dims(x, B, A):
    batch, D, H, W = x.shape
    K = B.shape[1] if B.dim() == 5 else 1
    N = A.shape[1]
    return batch, D, H, W, N, K


def _check(x, delta, A, B, C, Dskip, device_kind):
    torch = _torch()
    for name, t in (("x", x), ("delta", delta), ("A", A), ("B", B), ("C", C), ("Dskip", Dskip)):
        if t is None:
            if name != "Dskip":
                raise ValueError(f"{name} is required")
            continue
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if device_kind == "cuda" and not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if device_kind == "cpu" and t.is_cuda:
            raise ValueError(f"{name} must be a host tensor")
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    for name, t in (("delta", delta), ("B", B), ("C", C)):
        if t.dtype != x.dtype:
            raise TypeError(f"{name} must have the dtype of x")
    if A.dtype != torch.float32 or (Dskip is not None and Dskip.dtype != torch.float32):
        raise TypeError("A and Dskip must be float32")


def scan2d_fwd(x, delta, A, B, C, Dskip=None, y=None, flags=None, stream=None):
    """The 2D selective-scan forward on CUDA tensors (asynchronous on `stream`).

    flags defaults to the element type of x and K = B.shape[1] orientations
    (TL; TL+TR; TL+TR+BL; all four).  Returns y."""
    torch = _torch()
    _check(x, delta, A, B, C, Dskip, "cuda")
    batch, D, H, W, N, K = _dims(x, B, A)
    if flags is None:
        flags = flags_for(x.dtype == torch.bfloat16, (1 << K) - 1)
    out_dtype = torch.float32 if (x.dtype == torch.float32 or flags & SCAN2D_OUT_F32) else torch.bfloat16
    if y is None:
        y = torch.empty((batch, D, H, W), dtype=out_dtype, device=x.device)
    elif y.dtype != out_dtype or tuple(y.shape) != (batch, D, H, W) or not y.is_contiguous():
        raise ValueError("y has the wrong dtype, shape or layout")
    rc = _lib.scan2d_fwd(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip), _ptr(y),
                         batch, D, H, W, N, flags, _stream_handle(stream))
    if rc:
        raise Scan2dError(rc, "scan2d_fwd")
    return y


def scan2d_fwd_noalloc(x, delta, A, B, C, Dskip, y, flags=None, stream=None):
    """scan2d_fwd into a caller-provided y, with the library's fixed device scratch instead of
    an allocated workspace: for callers that must not allocate device memory (a runtime whose
    allocator owns the device's memory, an operator interface that forbids allocating during
    execution, a loop that cannot take the synchronisation an allocation may cause).  Calls
    share that scratch, so calls that overlap on the GPU race; shapes that need more than
    SCAN2D_NOALLOC_SCRATCH_BYTES raise Scan2dError (SCAN2D_E_SCRATCH)."""
    torch = _torch()
    _check(x, delta, A, B, C, Dskip, "cuda")
    batch, D, H, W, N, K = _dims(x, B, A)
    if flags is None:
        flags = flags_for(x.dtype == torch.bfloat16, (1 << K) - 1)
    out_dtype = torch.float32 if (x.dtype == torch.float32 or flags & SCAN2D_OUT_F32) else torch.bfloat16
    if y is None or y.dtype != out_dtype or tuple(y.shape) != (batch, D, H, W) or not y.is_contiguous():
        raise ValueError("y must be a contiguous CUDA tensor of the output dtype and shape")
    rc = _lib.scan2d_fwd_noalloc(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip),
                                 _ptr(y), batch, D, H, W, N, flags, _stream_handle(stream))
    if rc:
        raise Scan2dError(rc, "scan2d_fwd_noalloc")
    return y


def scan2d_bwd_workspace_bytes(batch, channels, H, W, N, flags) -> int:
    return int(_lib.scan2d_bwd_workspace_bytes(batch, channels, H, W, N, flags))


def scan2d_bwd(x, delta, A, B, C, Dskip, dy, flags=None, workspace=None, stream=None) -> dict:
    """Gradients of sum(dy * scan2d_fwd(x, delta, A, B, C, Dskip)) on CUDA tensors
    (asynchronous on `stream`): a dict with dx, ddelta (the layout and element type of y),
    dA (channels, N), dB and dC (the layout of B), dDskip (channels,), all fp32 but dx and
    ddelta.  `workspace` (a uint8 CUDA tensor of at least scan2d_bwd_workspace_bytes(...)
    bytes) is allocated here when not given."""
    torch = _torch()
    _check(x, delta, A, B, C, Dskip, "cuda")
    batch, D, H, W, N, K = _dims(x, B, A)
    if flags is None:
        flags = flags_for(x.dtype == torch.bfloat16, (1 << K) - 1)
    out_dtype = torch.float32 if (x.dtype == torch.float32 or flags & SCAN2D_OUT_F32) else torch.bfloat16
    if dy.dtype != out_dtype or tuple(dy.shape) != (batch, D, H, W) or not dy.is_contiguous() or not dy.is_cuda:
        raise ValueError("dy must be a contiguous CUDA tensor of the shape and dtype of y")
    need = scan2d_bwd_workspace_bytes(batch, D, H, W, N, flags)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    dev = x.device
    g = {"dx": torch.empty((batch, D, H, W), dtype=out_dtype, device=dev),
         "ddelta": torch.empty((batch, D, H, W), dtype=out_dtype, device=dev),
         "dA": torch.empty((D, N), dtype=torch.float32, device=dev),
         "dB": torch.empty(tuple(B.shape), dtype=torch.float32, device=dev),
         "dC": torch.empty(tuple(C.shape), dtype=torch.float32, device=dev),
         "dDskip": torch.empty((D,), dtype=torch.float32, device=dev)}
    rc = _lib.scan2d_bwd(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip), _ptr(dy),
                         *(_ptr(g[k]) for k in ("dx", "ddelta", "dA", "dB", "dC", "dDskip")),
                         _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
                         batch, D, H, W, N, flags, _stream_handle(stream))
    if rc:
        raise Scan2dError(rc, "scan2d_bwd")
    return g


def scan2d_grid_cells(coords, H, W, cell_patch=None, n_skipped=None, stream=None):
    """Cell map (H*W int32 CUDA tensor) of a bag whose patch k sits at coords[k] = (row, col)
    (an (npatch, 2) int32 CUDA tensor): the patch index at each cell, -1 where there is none."""
    torch = _torch()
    if coords.dtype != torch.int32 or coords.dim() != 2 or coords.shape[1] != 2 or not coords.is_contiguous():
        raise ValueError("coords must be a contiguous (npatch, 2) int32 tensor")
    if cell_patch is None:
        cell_patch = torch.empty(H * W, dtype=torch.int32, device=coords.device)
    rc = _lib.scan2d_grid_cells(_ptr(coords), coords.shape[0], H, W, _ptr(cell_patch), _ptr(n_skipped),
                                _stream_handle(stream))
    if rc:
        raise Scan2dError(rc, "scan2d_grid_cells")
    return cell_patch


def scan2d_grid_gather(feat, cell_patch, pad, H, W, x=None, stream=None):
    """x (1, channels, H, W): feat[cell_patch[i*W + j]] at each cell, pad where it is -1."""
    torch = _torch()
    npatch, D = feat.shape
    if x is None:
        x = torch.empty((1, D, H, W), dtype=feat.dtype, device=feat.device)
    flags = SCAN2D_BF16 if feat.dtype == torch.bfloat16 else 0
    rc = _lib.scan2d_grid_gather(_ptr(feat), _ptr(cell_patch), _ptr(pad), _ptr(x), npatch, D, H, W, flags,
                                 _stream_handle(stream))
    if rc:
        raise Scan2dError(rc, "scan2d_grid_gather")
    return x


def scan2d_fwd_wsi(feat, cell_patch, pad, delta, A, B, C, Dskip=None, y=None, flags=None, stream=None):
    """scan2d_fwd of one map whose x is read from the bag feat (npatch, channels) through the
    cell map, pad at non-tissue cells; x itself is never written."""
    torch = _torch()
    npatch, D = feat.shape
    _, _, H, W = delta.shape
    N = A.shape[1]
    K = B.shape[1] if B.dim() == 5 else 1
    if flags is None:
        flags = flags_for(delta.dtype == torch.bfloat16, (1 << K) - 1)
    out_dtype = torch.float32 if (delta.dtype == torch.float32 or flags & SCAN2D_OUT_F32) else torch.bfloat16
    if y is None:
        y = torch.empty((1, D, H, W), dtype=out_dtype, device=delta.device)
    rc = _lib.scan2d_fwd_wsi(_ptr(feat), _ptr(cell_patch), _ptr(pad), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                             _ptr(Dskip), _ptr(y), npatch, D, H, W, N, flags, _stream_handle(stream))
    if rc:
        raise Scan2dError(rc, "scan2d_fwd_wsi")
    return y


def scan2d_proj(x, Wx, Wdt, bdt, N, R, delta=None, B=None, C=None, stream=None):
    """delta (like x), B and C ((batch, N, H, W), x's dtype) from x and the projection weights
    Wx (R + 2N, channels), Wdt (channels, R), bdt (channels,), all CUDA tensors."""
    torch = _torch()
    batch, D, H, W = x.shape
    dev = x.device
    if delta is None:
        delta = torch.empty_like(x)
    if B is None:
        B = torch.empty((batch, N, H, W), dtype=x.dtype, device=dev)
    if C is None:
        C = torch.empty((batch, N, H, W), dtype=x.dtype, device=dev)
    flags = SCAN2D_BF16 if x.dtype == torch.bfloat16 else 0
    rc = _lib.scan2d_proj(_ptr(x), _ptr(Wx), _ptr(Wdt), _ptr(bdt), _ptr(delta), _ptr(B), _ptr(C),
                          batch, D, H, W, N, R, flags, _stream_handle(stream))
    if rc:
        raise Scan2dError(rc, "scan2d_proj")
    return delta, B, C


PLAN_FIELDS = ("launches", "grid", "threads", "smem", "nseg", "cols", "wpc", "mode", "ng",
               "workspace", "g", "tma", "link")


def scan2d_query_plan(batch, channels, H, W, N, flags) -> dict:
    """How scan2d_fwd runs a call of this shape (no device needed)."""
    out = (ctypes.c_longlong * len(PLAN_FIELDS))()
    rc = _lib.scan2d_query_plan(batch, channels, H, W, N, flags, out, len(PLAN_FIELDS))
    if rc:
        raise Scan2dError(rc, "scan2d_query_plan")
    return dict(zip(PLAN_FIELDS, (int(v) for v in out)))


def scan2d_host_staging_bytes(batch, channels, H, W, N, flags) -> int:
    return int(_lib.scan2d_host_staging_bytes(batch, channels, H, W, N, flags))


def scan2d_fwd_host(x, delta, A, B, C, Dskip, y, staging, flags=None, stream=None):
    """The forward on HOST tensors (pinned for overlap) through a caller-provided device
    staging buffer (a uint8 CUDA tensor of scan2d_host_staging_bytes(...) bytes).
    Asynchronous on `stream`; y (host) is valid once the stream has completed."""
    torch = _torch()
    _check(x, delta, A, B, C, Dskip, "cpu")
    batch, D, H, W, N, K = _dims(x, B, A)
    if flags is None:
        flags = flags_for(x.dtype == torch.bfloat16, (1 << K) - 1)
    rc = _lib.scan2d_fwd_host(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip),
                              _ptr(y), _ptr(staging), staging.numel() * staging.element_size(),
                              batch, D, H, W, N, flags, _stream_handle(stream))
    if rc:
        raise Scan2dError(rc, "scan2d_fwd_host")
    return y


def scan2d_get_device_error(stream=None) -> int:
    """Synchronise `stream`; return and clear the device's first recorded error (0 = none)."""
    return int(_lib.scan2d_get_device_error(_stream_handle(stream)))


def raw():
    """The ctypes library handle, for calls with plain integer pointers."""
    return _lib
