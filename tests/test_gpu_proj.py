"""The input projections on the GPU (scan2d_proj, through the C ABI) against the fp64 oracle.

Bound, element by element, with m the magnitude sum of the terms (|Wx|·|x| for B and C;
|Wdt|·(|Wx|·|x|) + |bdt| for delta's argument, and softplus' slope is at most 1):
|g - r| <= 1e-5·m + 1e-6 for fp32 outputs, and 1e-2·(|r| + m) + 1e-6 when the outputs are bf16
(one bf16 rounding is 2^-9 of |r|)."""
import numpy as np
import pytest

from selective_state_space_scan2d_b200 import inputs

from scan2d_testlib import TOL, assert_parity, to_torch, y_to_f64

pytestmark = pytest.mark.gpu


def _dev(a):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _f64(a):
    return inputs.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def _majorants(x, w, N, R):
    xa = np.abs(_f64(x))
    ua = np.einsum("jd,bdhw->bjhw", np.abs(w["Wx"].astype(np.float64)), xa)
    za = np.einsum("dr,brhw->bdhw", np.abs(w["Wdt"].astype(np.float64)), ua[:, :R]) + \
        np.abs(w["bdt"].astype(np.float64))[None, :, None, None]
    return za, ua[:, R:R + N], ua[:, R + N:]


def _check(got, ref, maj, bf16, label):
    got = np.asarray(got, np.float64)
    bound = (1e-2 * (np.abs(ref) + maj) if bf16 else 1e-5 * maj) + 1e-6
    ratio = np.abs(got - ref) / bound
    worst = float(ratio.max())
    assert worst <= 1.0 and np.all(np.isfinite(got)), f"{label}: worst {worst:.3g}x the bound"


def _run(x, w, N, R):
    from selective_state_space_scan2d_b200 import scan2d
    d, B, C = scan2d.scan2d_proj(_dev(x), _dev(w["Wx"]), _dev(w["Wdt"]), _dev(w["bdt"]), N, R)
    return [t.float().cpu().numpy() for t in (d, B, C)]


@pytest.mark.parametrize("dtype,D,N,R,H,W", [("f32", 128, 16, 8, 9, 37), ("f32", 40, 5, 3, 7, 11),
                                              ("bf16", 192, 16, 12, 6, 14), ("f32", 384, 16, 24, 3, 20),
                                              ("f32", 4, 4, 1, 8, 8)])
def test_proj_parity(oracle_mod, dtype, D, N, R, H, W):
    w0 = inputs.WORKLOADS["giga"].scaled(batch=2, channels=D, N=N, H=H, W=W, dtype=dtype)
    x = inputs.make_inputs(w0, seed=3)["x"]
    w = inputs.make_proj_weights(D, N, R, seed=3)
    got = _run(x, w, N, R)
    ref = oracle_mod.proj(x, w["Wx"], w["Wdt"], w["bdt"], N, R)
    maj = _majorants(x, w, N, R)
    for name, g, r, m in zip(("delta", "B", "C"), got, ref, maj):
        _check(g, r, m, dtype == "bf16", f"{dtype} D={D} {name}")


def test_proj_full_size_giga_sampled(oracle_mod):
    """1 x 128 x 1024 x 1024 fp32, as timed: every output at 64 sampled positions."""
    w0 = inputs.WORKLOADS["giga"]
    x = inputs.make_inputs(w0, seed=0)["x"]
    w = inputs.make_proj_weights(w0.channels, w0.N, 8, seed=0)
    got = _run(x, w, w0.N, 8)
    rng = np.random.default_rng(9)
    ii, jj = rng.integers(0, w0.H, 64), rng.integers(0, w0.W, 64)
    xs = np.ascontiguousarray(x[:, :, ii, jj][:, :, None, :])          # the sampled positions as a 1 x 64 map
    ref = oracle_mod.proj(xs, w["Wx"], w["Wdt"], w["bdt"], w0.N, 8)
    maj = _majorants(xs, w, w0.N, 8)
    for name, g, r, m in zip(("delta", "B", "C"), got, ref, maj):
        _check(g[:, :, ii, jj][:, :, None, :], r, m, False, f"giga {name}")


def test_proj_feeds_the_scan(oracle_mod):
    """delta, B, C from scan2d_proj go straight into scan2d_fwd; y meets the forward's bound
    against the oracle's scan of the oracle's projections (rounded to what the GPU stored)."""
    from selective_state_space_scan2d_b200 import scan2d
    w0 = inputs.WORKLOADS["giga"].scaled(channels=32, H=12, W=40)
    d = inputs.make_inputs(w0, seed=1)
    w = inputs.make_proj_weights(32, 16, 8, seed=1)
    t = to_torch(d)
    delta, B, C = scan2d.scan2d_proj(t["x"], _dev(w["Wx"]), _dev(w["Wdt"]), _dev(w["bdt"]), 16, 8)
    y = scan2d.scan2d_fwd(t["x"], delta, t["A"], B, C, t["Dskip"])
    ref = oracle_mod.scan2d_fwd(d["x"], delta.cpu().numpy(), d["A"], B.cpu().numpy()[:, None],
                                C.cpu().numpy()[:, None], d["Dskip"], 1)
    assert_parity(y_to_f64(y), ref, TOL["f32"], "proj -> scan")
