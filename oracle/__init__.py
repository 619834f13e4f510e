"""fp64 CPU oracle of the 2D selective-scan forward (2DMamba) and its gradients, as a ctypes binding.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The product path (the CUDA
library under ``selective_state_space_scan2d_b200``) shares no code with it.

The arithmetic lives in ``scan2d_oracle.c`` (plain single-threaded C, fp64), written
from the recurrences on the pages ("2DMamba 精读：从小白到博士", section 4.5 (1)
horizontal scan, (2) vertical scan and output).  This module only builds it with gcc and
marshals numpy arrays.

Input conventions (numpy):
  * fp32 tensors are ``float32`` arrays; bf16 tensors are ``uint16`` arrays holding the
    bf16 bit patterns (numpy has no bf16 dtype).  Every stored value is widened exactly.
  * x, delta: (batch, channels, H, W); A: (channels, N) float32; B, C: (batch, K, N, H, W);
    Dskip: (channels,) float32 or None.
  * ``orient_mask``: bit 4 (0x10) selects the vertical-then-horizontal scan order.
  * ``orient_mask`` bits 0-3: bit 0 top-left, bit 1 top-right (flip W), bit 2 bottom-left (flip H),
    bit 3 bottom-right (flip both).  K = number of set bits.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "scan2d_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_scan2d.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C99, -O2, no fast-math) into this folder."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str | None = None):
    """ctypes handle of the oracle library (the default build, or another build at path)."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(path or build())
    vp, fp, dp, ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    i, u = ctypes.c_int, ctypes.c_uint
    common = [vp, vp, fp, vp, vp, fp, dp, i, i, i, i, i, i, u]
    lib.scan2d_oracle_fwd.argtypes = common
    lib.scan2d_oracle_fwd.restype = i
    lib.scan2d_oracle_maps.argtypes = common + [ip, i]
    lib.scan2d_oracle_maps.restype = i
    lib.scan2d_oracle_points.argtypes = common + [ip, i]
    lib.scan2d_oracle_points.restype = i
    lib.scan2d_oracle_bwd.argtypes = [vp, vp, fp, vp, vp, fp, dp, dp, dp, dp, dp, dp, dp,
                                      i, i, i, i, i, i, u, i]
    lib.scan2d_oracle_bwd.restype = i
    lib.scan2d_oracle_version.argtypes = []
    lib.scan2d_oracle_version.restype = i
    if path is None:
        _lib = lib
    return lib


def _load(lib=None):
    return lib if lib is not None else load_library()


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _prepare(x, delta, A, B, C, Dskip, orient_mask):
    x = np.ascontiguousarray(x)
    delta = np.ascontiguousarray(delta)
    B = np.ascontiguousarray(B)
    C = np.ascontiguousarray(C)
    A = np.ascontiguousarray(A, dtype=np.float32)
    if Dskip is not None:
        Dskip = np.ascontiguousarray(Dskip, dtype=np.float32)
    if x.dtype == np.uint16:
        is_bf16 = 1
    elif x.dtype == np.float32:
        is_bf16 = 0
    else:
        raise TypeError("x must be float32 or uint16 (bf16 bits)")
    for name, t in (("delta", delta), ("B", B), ("C", C)):
        if t.dtype != x.dtype:
            raise TypeError(f"{name} must have the dtype of x")
    batch, channels, H, W = x.shape
    if delta.shape != x.shape:
        raise ValueError("delta must have the shape of x")
    K = bin(orient_mask & 0xF).count("1")
    if B.ndim == 4:                      # (batch, N, H, W) is the K = 1 layout
        B = B.reshape(B.shape[0], 1, *B.shape[1:])
        C = C.reshape(C.shape[0], 1, *C.shape[1:])
    if B.shape[0] != batch or B.shape[1] != K or B.shape[3:] != (H, W) or C.shape != B.shape:
        raise ValueError(f"B, C must be (batch, K={K}, N, H, W); got {B.shape}, {C.shape}")
    N = B.shape[2]
    if A.shape != (channels, N):
        raise ValueError("A must be (channels, N)")
    if Dskip is not None and Dskip.shape != (channels,):
        raise ValueError("Dskip must be (channels,)")
    return x, delta, A, B, C, Dskip, (batch, channels, H, W, N, is_bf16)


def scan2d_fwd(x, delta, A, B, C, Dskip=None, orient_mask: int = 1, lib=None) -> np.ndarray:
    """Full fp64 output y (batch, channels, H, W)."""
    x, delta, A, B, C, Dskip, dims = _prepare(x, delta, A, B, C, Dskip, orient_mask)
    y = np.empty(x.shape, dtype=np.float64)
    rc = _load(lib).scan2d_oracle_fwd(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip),
                                   _ptr(y), *dims, orient_mask)
    if rc:
        raise RuntimeError(f"oracle error {rc}")
    return y


def scan2d_maps(x, delta, A, B, C, Dskip, maps, orient_mask: int = 1, lib=None) -> np.ndarray:
    """fp64 output of the listed (b, d) maps only: shape (len(maps), H, W)."""
    x, delta, A, B, C, Dskip, dims = _prepare(x, delta, A, B, C, Dskip, orient_mask)
    m = np.ascontiguousarray(np.asarray(maps, dtype=np.int32).reshape(-1, 2))
    y = np.empty((m.shape[0], dims[2], dims[3]), dtype=np.float64)
    rc = _load(lib).scan2d_oracle_maps(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip),
                                    _ptr(y), *dims, orient_mask, _ptr(m), m.shape[0])
    if rc:
        raise RuntimeError(f"oracle error {rc}")
    return y


def scan2d_points(x, delta, A, B, C, Dskip, points, orient_mask: int = 1, lib=None) -> np.ndarray:
    """fp64 output at the listed (b, d, i, j) positions only."""
    x, delta, A, B, C, Dskip, dims = _prepare(x, delta, A, B, C, Dskip, orient_mask)
    p = np.ascontiguousarray(np.asarray(points, dtype=np.int32).reshape(-1, 4))
    y = np.empty(p.shape[0], dtype=np.float64)
    rc = _load(lib).scan2d_oracle_points(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                      _ptr(Dskip), _ptr(y), *dims, orient_mask, _ptr(p), p.shape[0])
    if rc:
        raise RuntimeError(f"oracle error {rc}")
    return y


def scan2d_bwd(x, delta, A, B, C, Dskip, dy, orient_mask: int = 1, majorant: bool = False,
               lib=None) -> dict:
    """fp64 gradients of sum(dy * y) with respect to every input: a dict with dx, ddelta
    (batch, channels, H, W), dA (channels, N), dB, dC (batch, K, N, H, W) and dDskip
    (channels,).  majorant=True returns, for each output, the sum of the magnitudes of the
    terms that make it up (the scale of any evaluation's rounding error)."""
    x, delta, A, B, C, Dskip, dims = _prepare(x, delta, A, B, C, Dskip, orient_mask)
    batch, channels, H, W, N, _ = dims
    K = B.shape[1]
    dy = np.ascontiguousarray(dy, dtype=np.float64)
    if dy.shape != x.shape:
        raise ValueError("dy must have the shape of x")
    out = {"dx": np.empty(x.shape), "ddelta": np.empty(x.shape), "dA": np.empty((channels, N)),
           "dB": np.empty((batch, K, N, H, W)), "dC": np.empty((batch, K, N, H, W)),
           "dDskip": np.empty(channels)}
    rc = _load(lib).scan2d_oracle_bwd(_ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip),
                                   _ptr(dy), *(_ptr(out[k]) for k in ("dx", "ddelta", "dA", "dB", "dC", "dDskip")),
                                   *dims, orient_mask, int(bool(majorant)))
    if rc:
        raise RuntimeError(f"oracle error {rc}")
    return out


def wsi_grid(feat, coords, pad, H: int, W: int):
    """The map of a whole-slide image from its bag of patches ("2DMamba 精读", section 四.2,
    the 2DMambaMIL framework, steps 3-4: each patch feature goes back to its grid position;
    cells without a patch hold the learnable non-tissue token).  Patches are placed in index
    order, so when two name one cell the later one stays; patches outside the grid are left
    out and counted.  Returns x (1, channels, H, W) of feat's dtype, the cell map (H*W int32,
    -1 at non-tissue cells) and the number of patches left out."""
    feat = np.asarray(feat)
    npatch, channels = feat.shape
    cell = np.full((H, W), -1, dtype=np.int32)
    skipped = 0
    for k in range(npatch):
        r, c = int(coords[k][0]), int(coords[k][1])
        if 0 <= r < H and 0 <= c < W:
            cell[r, c] = k
        else:
            skipped += 1
    x = np.empty((1, channels, H, W), dtype=feat.dtype)
    for r in range(H):
        for c in range(W):
            x[0, :, r, c] = feat[cell[r, c]] if cell[r, c] >= 0 else pad
    return x, cell.reshape(-1), skipped


def softplus(z):
    """log(1 + e^z), evaluated without overflow."""
    return np.logaddexp(0.0, z)


def proj(x, Wx, Wdt, bdt, N: int, R: int):
    """The input-dependent parameters of the scan from x (Mamba's selective projection, the
    reading of "2DMamba 精读", section 四.4: the parameters follow the current input): per
    position, u = Wx x (R + 2N values), B = u[R:R+N], C = u[R+N:], delta = softplus(Wdt u[:R]
    + bdt).  x: (batch, D, H, W) float32 or bf16 bits; returns fp64 delta (batch, D, H, W),
    B and C (batch, N, H, W)."""
    xf = np.asarray(x)
    if xf.dtype == np.uint16:
        xf = (xf.astype(np.uint32) << 16).view(np.float32)
    xf = xf.astype(np.float64)
    batch, D, H, W = xf.shape
    Wx = np.asarray(Wx, dtype=np.float64)
    Wdt = np.asarray(Wdt, dtype=np.float64)
    bdt = np.asarray(bdt, dtype=np.float64)
    if Wx.shape != (R + 2 * N, D) or Wdt.shape != (D, R) or bdt.shape != (D,):
        raise ValueError("weights must be Wx (R + 2N, D), Wdt (D, R), bdt (D,)")
    u = np.einsum("jd,bdhw->bjhw", Wx, xf)
    z = np.einsum("dr,brhw->bdhw", Wdt, u[:, :R]) + bdt[None, :, None, None]
    return softplus(z), u[:, R:R + N].copy(), u[:, R + N:].copy()


def version() -> int:
    return _load().scan2d_oracle_version()
