"""Parity of the CUDA gradients (scan2d_bwd, through the C ABI) with the fp64 oracle.

Bound, element by element, for every gradient g with oracle value r and oracle majorant m (the
sum of the magnitudes of the terms that make up r, so m bounds the rounding error of any
evaluation order):  |g - r| <= RTOL * m + 1e-6, with RTOL = 1e-4 for fp32 results and 1e-2
for bf16 results (dx and ddelta when y is bf16: one bf16 rounding is 2^-9 of |r| <= m).
"""
import numpy as np
import pytest

from selective_state_space_scan2d_b200 import inputs

from scan2d_testlib import to_torch, workload

pytestmark = pytest.mark.gpu

RTOL_F32 = 1e-4
RTOL_BF16 = 1e-2
NAMES = ("dx", "ddelta", "dA", "dB", "dC", "dDskip")


def _dy_torch(dy):
    import torch
    if dy.dtype == np.uint16:
        return torch.from_numpy(dy.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(dy).cuda()


def _dy_f64(dy):
    return inputs.bf16_bits_to_f32(dy).astype(np.float64) if dy.dtype == np.uint16 else dy.astype(np.float64)


def _gpu_bwd(d, dy, out_f32=False):
    from selective_state_space_scan2d_b200 import scan2d
    t = to_torch(d)
    flags = scan2d.flags_for(d["x"].dtype == np.uint16, d["orient_mask"], out_f32=out_f32,
                             vfirst=d.get("vfirst", False))
    g = scan2d.scan2d_bwd(t["x"], t["delta"], t["A"], t["B"], t["C"], t["Dskip"], _dy_torch(dy), flags=flags)
    assert scan2d.scan2d_get_device_error() == 0
    return {k: v.detach().float().cpu().numpy().astype(np.float64) for k, v in g.items()}


def _check(g, ref, maj, bf16_out, label, skip=()):
    worst = {}
    for k in NAMES:
        if k in skip:
            continue
        rtol = RTOL_BF16 if (bf16_out and k in ("dx", "ddelta")) else RTOL_F32
        bound = rtol * maj[k] + 1e-6
        err = np.abs(g[k].reshape(ref[k].shape) - ref[k])
        ratio = err / bound
        w = float(np.max(ratio))
        worst[k] = w
        if not (w <= 1.0) or not np.all(np.isfinite(g[k])):
            idx = np.unravel_index(int(np.nanargmax(ratio)), ratio.shape)
            raise AssertionError(f"{label} {k}: {int((ratio > 1).sum())} of {ratio.size} outside the bound; "
                                 f"worst {w:.3g}x at {idx}: got {g[k].reshape(ref[k].shape)[idx]!r}, "
                                 f"want {ref[k][idx]!r} (majorant {maj[k][idx]!r})")
    return worst


# (workload, overrides, out_f32): ragged channel groups, ragged and odd strips, every
# orientation set, N = 4 / 8 / 16, with and without Dskip
CASES = {
    "f32_tl_ragged": ("giga", dict(batch=2, channels=12, H=9, W=21), False),
    "f32_all4": ("giga", dict(channels=8, H=7, W=16, orient_mask=0xF), False),
    "f32_tr_bl_odd": ("tiny", dict(batch=2, channels=5, N=8, H=6, W=13, orient_mask=0b0110), False),
    "f32_n4_nodskip": ("tiny", dict(channels=9, H=10, W=11, dskip=False), False),
    "f32_br_random_A": ("giga", dict(channels=8, H=12, W=24, orient_mask=0b1000, random_A=True), False),
    "bf16_vision_like": ("vision", dict(batch=2, channels=16, H=10, W=14), False),
    "bf16_out_f32": ("vision", dict(batch=1, channels=8, H=9, W=16, orient_mask=0b0101), True),
    "bf16_k1_aligned": ("small", dict(batch=3, channels=16, H=8, W=24), False),
    "f32_h1": ("giga", dict(channels=8, H=1, W=37), False),
    "f32_w1": ("giga", dict(channels=8, H=23, W=1, orient_mask=0b0011), False),
    "f32_wide": ("giga", dict(channels=16, H=6, W=200), False),
    "f32_n13_odd_states": ("tiny", dict(batch=1, channels=11, N=13, H=7, W=19, orient_mask=0b0101), False),
    "bf16_n5_odd_states": ("vision", dict(batch=1, channels=8, N=5, H=6, W=12), False),
    # the vertical-first scan order
    "f32_vf_ragged": ("giga", dict(batch=2, channels=12, H=9, W=21, vfirst=True), False),
    "f32_vf_all4": ("giga", dict(channels=8, H=7, W=16, orient_mask=0xF, vfirst=True), False),
    "f32_vf_n4_nodskip": ("tiny", dict(channels=9, H=10, W=11, dskip=False, vfirst=True), False),
    "bf16_vf_vision_like": ("vision", dict(batch=2, channels=16, H=10, W=14, vfirst=True), False),
    "f32_vf_wide_br": ("giga", dict(channels=16, H=6, W=200, orient_mask=0b1000, vfirst=True), False),
}


def _mask(d):
    return d["orient_mask"] | (0x10 if d.get("vfirst") else 0)


@pytest.mark.parametrize("case", sorted(CASES))
def test_bwd_parity(oracle_mod, case):
    name, kw, out_f32 = CASES[case]
    w = workload(name, **kw)
    d = inputs.make_inputs(w, seed=3)
    dy = inputs.make_cotangent(w, seed=3, out_f32=out_f32)
    g = _gpu_bwd(d, dy, out_f32)
    args = (d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], _dy_f64(dy), _mask(d))
    ref = oracle_mod.scan2d_bwd(*args)
    maj = oracle_mod.scan2d_bwd(*args, majorant=True)
    _check(g, ref, maj, w.dtype == "bf16" and not out_f32, case)


def test_bwd_repeatable_and_workspace_reused(oracle_mod):
    """Two calls with one caller-provided workspace give the same results (up to the order of
    the atomic sums) and do not depend on what the workspace held before."""
    import torch
    from selective_state_space_scan2d_b200 import scan2d
    w = workload("giga", batch=1, channels=16, H=20, W=40, orient_mask=0b1001)
    d = inputs.make_inputs(w, seed=5)
    dy = inputs.make_cotangent(w, seed=5)
    t = to_torch(d)
    flags = scan2d.flags_for(False, d["orient_mask"])
    ws = torch.full((scan2d.scan2d_bwd_workspace_bytes(1, 16, 20, 40, 16, flags),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    g1 = scan2d.scan2d_bwd(t["x"], t["delta"], t["A"], t["B"], t["C"], t["Dskip"], _dy_torch(dy), flags=flags,
                           workspace=ws)
    g2 = scan2d.scan2d_bwd(t["x"], t["delta"], t["A"], t["B"], t["C"], t["Dskip"], _dy_torch(dy), flags=flags,
                           workspace=ws)
    torch.cuda.synchronize()
    for k in ("dx", "ddelta"):
        assert torch.equal(g1[k], g2[k]), k
    for k in ("dA", "dB", "dC", "dDskip"):
        torch.testing.assert_close(g1[k], g2[k], rtol=1e-5, atol=1e-6)


def test_bwd_rejects_small_workspace():
    import torch
    from selective_state_space_scan2d_b200 import scan2d
    w = workload("tiny")
    d = inputs.make_inputs(w, seed=1)
    t = to_torch(d)
    dy = _dy_torch(inputs.make_cotangent(w, seed=1))
    flags = scan2d.flags_for(False, 1)
    need = scan2d.scan2d_bwd_workspace_bytes(1, 4, 8, 8, 4, flags)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(scan2d.Scan2dError) as e:
        scan2d.scan2d_bwd(t["x"], t["delta"], t["A"], t["B"], t["C"], t["Dskip"], dy, flags=flags, workspace=small)
    assert e.value.code == scan2d.SCAN2D_E_WORKSPACE


def _crop(d, rows, cols, channels=None):
    """Inputs restricted to a rectangle of rows x cols (and optionally some channels)."""
    c = dict(d)
    ch = slice(None) if channels is None else channels
    for k in ("x", "delta"):
        c[k] = np.ascontiguousarray(d[k][:, ch][:, :, rows][:, :, :, cols])
    for k in ("B", "C"):
        c[k] = np.ascontiguousarray(d[k][:, :, :, rows][:, :, :, :, cols])
    c["A"] = np.ascontiguousarray(d["A"][ch])
    c["Dskip"] = None if d["Dskip"] is None else np.ascontiguousarray(d["Dskip"][ch])
    return c


def test_bwd_full_size_giga_sampled(oracle_mod):
    """The giga-pixel map at full size (1 x 128 x 1024 x 1024, N = 16, fp32, one launch
    sequence as timed): dx, ddelta, dA, dDskip of two whole channels against the oracle on
    those channels; dC on the top-left 16 x 16 corner (h there depends only on the rectangle
    above and to the left) and dB on the bottom-right corner (the adjoint there depends only
    on the rectangle below and to the right), both summed over all 128 channels."""
    w = inputs.WORKLOADS["giga"]
    d = inputs.make_inputs(w, seed=0)
    dy = inputs.make_cotangent(w, seed=0)
    g = _gpu_bwd(d, dy)
    dyf = _dy_f64(dy)
    for ch in (5, 126):
        c = _crop(d, slice(None), slice(None), [ch])
        args = (c["x"], c["delta"], c["A"], c["B"], c["C"], c["Dskip"], dyf[:, [ch]], 1)
        ref = oracle_mod.scan2d_bwd(*args)
        maj = oracle_mod.scan2d_bwd(*args, majorant=True)
        sub = {"dx": g["dx"][:, [ch]], "ddelta": g["ddelta"][:, [ch]], "dA": g["dA"][[ch]],
               "dDskip": g["dDskip"][[ch]], "dB": None, "dC": None}
        _check(sub, ref, maj, False, f"giga channel {ch}", skip=("dB", "dC"))
    H, W, r = w.H, w.W, 16
    c = _crop(d, slice(0, r), slice(0, r))
    args = (c["x"], c["delta"], c["A"], c["B"], c["C"], c["Dskip"], np.ascontiguousarray(dyf[:, :, :r, :r]), 1)
    ref, maj = oracle_mod.scan2d_bwd(*args), oracle_mod.scan2d_bwd(*args, majorant=True)
    got = g["dC"].reshape(1, 1, 16, H, W)[..., :r, :r]
    err = np.abs(got - ref["dC"]) / (RTOL_F32 * maj["dC"] + 1e-6)
    assert float(err.max()) <= 1.0, f"dC corner: worst {float(err.max()):.3g}x the bound"
    c = _crop(d, slice(H - r, H), slice(W - r, W))
    args = (c["x"], c["delta"], c["A"], c["B"], c["C"], c["Dskip"],
            np.ascontiguousarray(dyf[:, :, H - r:, W - r:]), 1)
    ref, maj = oracle_mod.scan2d_bwd(*args), oracle_mod.scan2d_bwd(*args, majorant=True)
    got = g["dB"].reshape(1, 1, 16, H, W)[..., H - r:, W - r:]
    err = np.abs(got - ref["dB"]) / (RTOL_F32 * maj["dB"] + 1e-6)
    assert float(err.max()) <= 1.0, f"dB corner: worst {float(err.max()):.3g}x the bound"


def test_bwd_full_size_vision_sampled(oracle_mod):
    """The vision stage at full size (64 x 192 x 56 x 56, N = 16, bf16, four orientations):
    every per-batch gradient (dx, ddelta, dB, dC) of two batch elements against the oracle
    on those elements; dDskip, a plain sum over batch and positions, against numpy."""
    w = inputs.WORKLOADS["vision"]
    d = inputs.make_inputs(w, seed=0)
    dy = inputs.make_cotangent(w, seed=0)
    g = _gpu_bwd(d, dy)
    dyf = _dy_f64(dy)
    for b in (0, 63):
        c = dict(d)
        for k in ("x", "delta", "B", "C"):
            c[k] = np.ascontiguousarray(d[k][[b]])
        args = (c["x"], c["delta"], c["A"], c["B"], c["C"], c["Dskip"], dyf[[b]], d["orient_mask"])
        ref = oracle_mod.scan2d_bwd(*args)
        maj = oracle_mod.scan2d_bwd(*args, majorant=True)
        sub = {k: g[k][[b]] for k in ("dx", "ddelta", "dB", "dC")}
        _check(sub, ref, maj, True, f"vision batch {b}", skip=("dA", "dDskip"))
    xf = inputs.bf16_bits_to_f32(d["x"]).astype(np.float64)
    want = np.einsum("bdij,bdij->d", dyf, xf)
    scale = np.einsum("bdij,bdij->d", np.abs(dyf), np.abs(xf))
    assert np.all(np.abs(g["dDskip"] - want) <= RTOL_F32 * scale + 1e-6)
