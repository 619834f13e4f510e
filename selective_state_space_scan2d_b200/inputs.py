"""Seeded synthetic inputs for the 2D selective scan, shared by the tests, the benchmark
and the CPU oracle runs.  numpy only; this module holds none of the scan's arithmetic.

The workloads are synthetic stand-ins for the pages' data sets (whole-slide images from
TCGA / BRACS / PANDA, ImageNet-1K and ADE20K feature maps), which are not available here.
Their shapes follow the pages: SSM width D = 128 and state size N = 16 (papernotes.org
notes, "训练策略"), the 14x14 map used for the padding discussion ("SegmentedBlockScan"),
and giga-pixel whole-slide grids.

Recipe (every tensor from its own PCG64 stream keyed by (seed, tensor id)):
  x      ~ N(0, 1)                                     (batch, D, H, W)
  delta  = softplus(u), u ~ U(lo, hi)                  (batch, D, H, W)
  A[d,n] = -(n + 1), or -U(0.5, 16) for the random-A variant
  B, C   ~ N(0, 1)                                     (batch, K, N, H, W), shared over D
  Dskip  ~ N(0, 1)                                     (D,)
  WSI mask: N(0,1) noise on the H x W grid, Gaussian-smoothed (sigma 8, truncated at 3
  sigma, reflecting boundary), the round(0.35 * H * W) lowest cells are "non-tissue"; every
  non-tissue cell of x holds one shared pad vector p[d] ~ N(0, 1).
bf16 tensors are produced by rounding the fp32 draws to nearest-even and are returned as
uint16 bit patterns (numpy has no bf16 dtype).
"""
from __future__ import annotations

import dataclasses

import numpy as np

ORIENT_TL, ORIENT_TR, ORIENT_BL, ORIENT_BR = 1, 2, 4, 8

_TENSOR_ID = {"x": 1, "delta": 2, "B": 3, "C": 4, "Dskip": 5, "pad": 6, "mask": 7, "A": 8, "dy": 9,
              "order": 10, "Wx": 11, "Wdt": 12, "bdt": 13}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    channels: int
    N: int
    H: int
    W: int
    dtype: str = "f32"                 # "f32" or "bf16" for x, delta, B, C (and y)
    orient_mask: int = ORIENT_TL
    delta_lo: float = -4.0
    delta_hi: float = -1.0
    wsi_mask: bool = False
    random_A: bool = False
    dskip: bool = True
    vfirst: bool = False               # scan order: vertical first (not an input, a flag)

    @property
    def K(self) -> int:
        return bin(self.orient_mask & 0xF).count("1")

    @property
    def elements(self) -> int:
        return self.batch * self.channels * self.H * self.W

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # 1 x 4 x 8 x 8, N = 4, fp32: the small case the oracle checks exhaustively.
    "tiny": Workload("tiny", 1, 4, 4, 8, 8),
    # 1 x 128 x 160 x 224 (35,840 patches), fp32, ~35% non-tissue cells hold a pad vector.
    "wsi": Workload("wsi", 1, 128, 16, 160, 224, wsi_mask=True),
    # 256 x 384 x 14 x 14, bf16: H*W = 196 is not a multiple of 32.
    "small": Workload("small", 256, 384, 16, 14, 14, dtype="bf16"),
    # 64 x 192 x 56 x 56, bf16, four corner orientations with their own B_k, C_k.
    "vision": Workload("vision", 64, 192, 16, 56, 56, dtype="bf16", orient_mask=0xF),
    # 1 x 128 x 1024 x 1024 (1,048,576 patches), fp32, long-range decay.
    "giga": Workload("giga", 1, 128, 16, 1024, 1024, delta_lo=-5.0, delta_hi=-2.0),
}


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TENSOR_ID[name]])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _softplus_f32(u: np.ndarray) -> np.ndarray:
    return np.logaddexp(np.float32(0.0), u).astype(np.float32)


def _gaussian_smooth_reflect(a: np.ndarray, sigma: float) -> np.ndarray:
    """Separable Gaussian filter, kernel truncated at 3 sigma, reflecting boundary."""
    r = int(3.0 * sigma + 0.5)
    t = np.arange(-r, r + 1, dtype=np.float64)
    k = np.exp(-0.5 * (t / sigma) ** 2)
    k /= k.sum()
    out = a.astype(np.float64)
    for axis in (0, 1):
        pad = [(0, 0), (0, 0)]
        pad[axis] = (r, r)
        p = np.pad(out, pad, mode="symmetric")
        acc = np.zeros_like(out)
        for o, w in enumerate(k):
            sl = [slice(None), slice(None)]
            sl[axis] = slice(o, o + out.shape[axis])
            acc += w * p[tuple(sl)]
        out = acc
    return out


def wsi_tissue_mask(H: int, W: int, seed: int = 0, frac_empty: float = 0.35) -> np.ndarray:
    """Boolean (H, W) map, True where a cell is non-tissue (holds the pad vector)."""
    noise = _rng(seed, "mask").standard_normal((H, W))
    sm = _gaussian_smooth_reflect(noise, 8.0)
    n_empty = int(round(frac_empty * H * W))
    order = np.argsort(sm, axis=None, kind="stable")
    mask = np.zeros(H * W, dtype=bool)
    mask[order[:n_empty]] = True
    return mask.reshape(H, W)


def make_inputs(w: Workload | str, seed: int = 0) -> dict:
    """All inputs of one workload as numpy arrays, plus its metadata.

    Returns a dict with x, delta, A, B, C, Dskip (None when the workload has no skip term),
    'workload' and 'orient_mask'.  B and C are always 5-D: (batch, K, N, H, W)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    shp = (w.batch, w.channels, w.H, w.W)
    x = _rng(seed, "x").standard_normal(shp, dtype=np.float32)
    if w.wsi_mask:
        mask = wsi_tissue_mask(w.H, w.W, seed)
        pad = _rng(seed, "pad").standard_normal(w.channels, dtype=np.float32)
        x[:, :, mask] = pad[None, :, None]
    u = _rng(seed, "delta").random(shp, dtype=np.float32)
    u = np.float32(w.delta_lo) + np.float32(w.delta_hi - w.delta_lo) * u
    delta = _softplus_f32(u)
    if w.random_A:
        A = -(np.float32(0.5) + np.float32(15.5) * _rng(seed, "A").random((w.channels, w.N), dtype=np.float32))
    else:
        A = -np.tile(np.arange(1, w.N + 1, dtype=np.float32), (w.channels, 1))
    bshp = (w.batch, w.K, w.N, w.H, w.W)
    B = _rng(seed, "B").standard_normal(bshp, dtype=np.float32)
    C = _rng(seed, "C").standard_normal(bshp, dtype=np.float32)
    Dskip = _rng(seed, "Dskip").standard_normal(w.channels, dtype=np.float32) if w.dskip else None
    if w.dtype == "bf16":
        x, delta, B, C = (f32_to_bf16_bits(t) for t in (x, delta, B, C))
    elif w.dtype != "f32":
        raise ValueError(w.dtype)
    return dict(x=x, delta=delta, A=np.ascontiguousarray(A, dtype=np.float32), B=B, C=C,
                Dskip=Dskip, workload=w, orient_mask=w.orient_mask, vfirst=w.vfirst)


def make_cotangent(w: Workload | str, seed: int = 0, out_f32: bool = False) -> np.ndarray:
    """A seeded cotangent dy for the gradients: N(0, 1) values of y's shape, as bf16 bits
    when y is bf16 (bf16 inputs without fp32 output), else float32."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    dy = _rng(seed, "dy").standard_normal((w.batch, w.channels, w.H, w.W), dtype=np.float32)
    return f32_to_bf16_bits(dy) if (w.dtype == "bf16" and not out_f32) else dy


def make_wsi_bag(w: Workload | str, seed: int = 0) -> dict:
    """The workload's map as a bag of patches: the tissue cells of make_inputs' mask in a
    seeded random order, their features feat (npatch, channels) = x at those cells, their
    coordinates (npatch, 2) int32 (row, column) and the non-tissue token pad (channels), so
    that placing the bag on the grid gives back make_inputs' x exactly."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    if w.batch != 1 or not w.wsi_mask:
        raise ValueError("a bag describes one whole-slide map (batch 1, wsi_mask)")
    d = make_inputs(w, seed)
    mask = wsi_tissue_mask(w.H, w.W, seed)
    rows, cols = np.nonzero(~mask)
    order = _rng(seed, "order").permutation(rows.size)
    rows, cols = rows[order], cols[order]
    feat = np.ascontiguousarray(d["x"][0][:, rows, cols].T)
    coords = np.ascontiguousarray(np.stack([rows, cols], axis=1).astype(np.int32))
    pad = _rng(seed, "pad").standard_normal(w.channels, dtype=np.float32)
    if w.dtype == "bf16":
        pad = f32_to_bf16_bits(pad)
    return dict(d, feat=feat, coords=coords, pad=pad, tissue=~mask)


def make_proj_weights(channels: int, N: int, R: int, seed: int = 0) -> dict:
    """Weights of the input projections: Wx (R + 2N, channels) ~ N(0, 1/channels), Wdt
    (channels, R) ~ N(0, 1/R), and bdt = log(e^dt - 1) with dt = exp(U(log 1e-3, log 1e-1)), so
    that delta starts near the step sizes of the other workloads.  All float32."""
    Wx = _rng(seed, "Wx").standard_normal((R + 2 * N, channels), dtype=np.float32) / np.float32(np.sqrt(channels))
    Wdt = _rng(seed, "Wdt").standard_normal((channels, R), dtype=np.float32) / np.float32(np.sqrt(R))
    dt = np.exp(np.log(1e-3) + (np.log(1e-1) - np.log(1e-3)) * _rng(seed, "bdt").random(channels))
    bdt = np.log(np.expm1(dt)).astype(np.float32)
    return dict(Wx=np.ascontiguousarray(Wx), Wdt=np.ascontiguousarray(Wdt), bdt=bdt, R=R)
