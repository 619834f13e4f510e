"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each pin is an independent route to the same number:
  * the unrolled closed form (a sum over source positions of path products), by brute
    force on small maps ("2DMamba 精读", section 五.3; product form for varying Abar);
  * the two scans written as lower-triangular linear systems and solved by LAPACK;
  * the Manhattan-distance form for constant Abar, and the pages' 3x3 worked example;
  * the 1D Mamba recurrence when H = 1 or W = 1 ("2DMamba 精读", section 四.4);
  * linearity in x, B = 0, C picking one state, and orientations as flips of the input.
A last test plants plausible mistakes in a copy of the oracle and checks that every one
of them is caught by at least one pin.
"""
import json
import os
import subprocess

import numpy as np
import pytest

from selective_state_space_scan2d_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(a):
    if a.dtype == np.uint16:
        return inputs.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


# ----------------------------------------------------------------------------------------
# independent routes
# ----------------------------------------------------------------------------------------
def closed_form_map(x, dl, A, B, C, D):
    """One map, one orientation (top-left), brute force over all source positions:
    h[i,j] = sum_{i'<=i, j'<=j} prod_{k=i'+1..i} Abar[k,j] * prod_{l=j'+1..j} Abar[i',l]
             * Bbar[i',j'] x[i',j'];   y = sum_n C[n] h[n] + D x."""
    H, W = x.shape
    y = D * x.copy()
    for n in range(A.shape[0]):
        a = np.exp(dl * A[n])
        u = dl * B[n] * x
        for i in range(H):
            for j in range(W):
                s = 0.0
                for ip in range(i + 1):
                    down = np.prod(a[ip + 1:i + 1, j])
                    for jp in range(j + 1):
                        right = np.prod(a[ip, jp + 1:j + 1])
                        s += down * right * u[ip, jp]
                y[i, j] += C[n, i, j] * s
    return y


def linsolve_map(x, dl, A, B, C, D):
    """One map, top-left: hh = M_h^{-1} u and h = M_v^{-1} hh with
    M_h = I - diag(Abar) S_left and M_v = I - diag(Abar) S_up, solved by numpy.linalg."""
    H, W = x.shape
    L = H * W
    y = (D * x).ravel().copy()
    for n in range(A.shape[0]):
        a = np.exp(dl * A[n]).ravel()
        u = (dl * B[n] * x).ravel()
        Mh = np.eye(L)
        Mv = np.eye(L)
        for p in range(L):
            i, j = divmod(p, W)
            if j > 0:
                Mh[p, p - 1] = -a[p]
            if i > 0:
                Mv[p, p - W] = -a[p]
        h = np.linalg.solve(Mv, np.linalg.solve(Mh, u))
        y += C[n].ravel() * h
    return y.reshape(H, W)


def closed_form_map_vfirst(x, dl, A, B, C, D):
    """Vertical-then-horizontal order, brute force: the path from (i', j') runs down column
    j' to row i, then right along row i:
    h[i,j] = sum prod_{l=j'+1..j} Abar[i,l] * prod_{k=i'+1..i} Abar[k,j'] * Bbar x[i',j']."""
    H, W = x.shape
    y = D * x.copy()
    for n in range(A.shape[0]):
        a = np.exp(dl * A[n])
        u = dl * B[n] * x
        for i in range(H):
            for j in range(W):
                s = 0.0
                for jp in range(j + 1):
                    right = np.prod(a[i, jp + 1:j + 1])
                    for ip in range(i + 1):
                        down = np.prod(a[ip + 1:i + 1, jp])
                        s += right * down * u[ip, jp]
                y[i, j] += C[n, i, j] * s
    return y


def recurrence_1d(a, u):
    """Textbook 1D selective recurrence h_t = a_t h_{t-1} + u_t, h_{-1} = 0."""
    h = np.zeros_like(u)
    prev = 0.0
    for t in range(u.shape[0]):
        prev = a[t] * prev + u[t]
        h[t] = prev
    return h


def _small(name="tiny", seed=0, **kw):
    w = inputs.WORKLOADS[name].scaled(**kw)
    return inputs.make_inputs(w, seed)


def _map_args(d, b, ch, k=0):
    x = _f64(d["x"][b, ch])
    dl = _f64(d["delta"][b, ch])
    A = d["A"][ch].astype(np.float64)
    B = _f64(d["B"][b, k])
    C = _f64(d["C"][b, k])
    D = 0.0 if d["Dskip"] is None else float(d["Dskip"][ch])
    return x, dl, A, B, C, D


def _fwd(oracle_mod, d, lib=None, mask=None):
    return oracle_mod.scan2d_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"],
                                 d["orient_mask"] if mask is None else mask, lib=lib)


# ----------------------------------------------------------------------------------------
# pins (each takes an optional ctypes lib so the mutation test can rerun them)
# ----------------------------------------------------------------------------------------
def pin_closed_form(oracle_mod, lib=None):
    for (H, W, N, seed) in [(8, 8, 4, 0), (5, 7, 3, 1), (6, 3, 2, 2)]:
        d = _small(H=H, W=W, N=N, channels=2, batch=1, seed=seed)
        y = _fwd(oracle_mod, d, lib)
        for ch in range(2):
            ref = closed_form_map(*_map_args(d, 0, ch))
            np.testing.assert_allclose(y[0, ch], ref, rtol=1e-12, atol=1e-12)


def pin_linsolve(oracle_mod, lib=None):
    d = _small(H=7, W=9, N=3, channels=2, batch=2, seed=3, random_A=True)
    y = _fwd(oracle_mod, d, lib)
    for b in range(2):
        for ch in range(2):
            ref = linsolve_map(*_map_args(d, b, ch))
            np.testing.assert_allclose(y[b, ch], ref, rtol=1e-11, atol=1e-11)


def pin_manhattan_constant(oracle_mod, lib=None):
    """Constant delta and A: h[i,j] = sum a^{(i-i')+(j-j')} Bbar x  (pages' printed form)."""
    d = _small(H=6, W=9, N=2, channels=1, batch=1, seed=4)
    d["delta"][:] = np.float32(0.3)
    y = _fwd(oracle_mod, d, lib)
    x, dl, A, B, C, D = _map_args(d, 0, 0)
    H, W = x.shape
    ii, jj = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    ref = D * x
    for n in range(A.shape[0]):
        a = np.exp(dl[0, 0] * A[n])        # the stored fp32 value of delta
        u = dl * B[n] * x
        h = np.zeros((H, W))
        for i in range(H):
            for j in range(W):
                m = (ii <= i) & (jj <= j)
                h[i, j] = np.sum(a ** ((i - ii[m]) + (j - jj[m])) * u[m])
        ref = ref + C[n] * h
    np.testing.assert_allclose(y[0, 0], ref, rtol=1e-12, atol=1e-12)


def pin_golden_3x3(oracle_mod, lib=None):
    g = json.load(open(os.path.join(GOLDEN, "manhattan_3x3.json")))
    H, W = g["H"], g["W"]
    si, sj = (v - 1 for v in g["source_1based"])
    ti, tj = (v - 1 for v in g["target_1based"])
    dval, aval = 0.25, -1.5
    x = np.zeros((1, 1, H, W), np.float32)
    x[0, 0, si, sj] = 1.0
    delta = np.full((1, 1, H, W), dval, np.float32)
    A = np.array([[aval]], np.float32)
    B = np.ones((1, 1, 1, H, W), np.float32)
    C = np.zeros((1, 1, 1, H, W), np.float32)
    C[0, 0, 0, ti, tj] = 1.0
    y = oracle_mod.scan2d_fwd(x, delta, A, B, C, None, 1, lib=lib)
    abar = np.exp(np.float64(np.float32(dval)) * np.float64(np.float32(aval)))
    bbar_x = np.float64(np.float32(dval))
    assert y[0, 0, ti, tj] == pytest.approx(abar ** g["power_2d"] * bbar_x, rel=1e-13)
    # the flattened 1D sequence of the same map decays with the sequence distance
    flat = recurrence_1d(np.full(H * W, abar), np.eye(H * W)[si * W + sj] * bbar_x)
    assert flat[ti * W + tj] == pytest.approx(abar ** g["power_1d_flattened"] * bbar_x, rel=1e-13)
    assert g["power_2d"] == (ti - si) + (tj - sj)


def pin_1d_reduction(oracle_mod, lib=None):
    for (H, W) in [(1, 13), (11, 1)]:
        d = _small(H=H, W=W, N=3, channels=2, batch=1, seed=5, random_A=True)
        y = _fwd(oracle_mod, d, lib)
        for ch in range(2):
            x, dl, A, B, C, D = _map_args(d, 0, ch)
            ref = D * x.ravel()
            for n in range(A.shape[0]):
                h = recurrence_1d(np.exp(dl * A[n]).ravel(), (dl * B[n] * x).ravel())
                ref = ref + C[n].ravel() * h
            np.testing.assert_allclose(y[0, ch].ravel(), ref, rtol=1e-12, atol=1e-12)


def pin_linearity_and_special(oracle_mod, lib=None):
    d = _small(H=5, W=6, N=3, channels=3, batch=2, seed=6)
    y1 = _fwd(oracle_mod, d, lib)
    Dx = d["Dskip"][None, :, None, None].astype(np.float64) * d["x"].astype(np.float64)
    d2 = dict(d)
    d2["x"] = (d["x"] * np.float32(2.0)).astype(np.float32)
    y2 = _fwd(oracle_mod, d2, lib)
    np.testing.assert_allclose(y2 - 2 * Dx, 2 * (y1 - Dx), rtol=1e-12, atol=1e-12)
    # B = 0: only the skip term remains
    d3 = dict(d)
    d3["B"] = np.zeros_like(d["B"])
    np.testing.assert_array_equal(_fwd(oracle_mod, d3, lib), Dx)
    # C = e_n at one position picks that state's h; compare with the closed form
    d4 = dict(d)
    d4["C"] = np.zeros_like(d["C"])
    d4["C"][:, :, 1] = 1.0
    d4["Dskip"] = None
    y4 = _fwd(oracle_mod, d4, lib)
    x, dl, A, B, C, D = _map_args(d4, 1, 2)
    ref = closed_form_map(x, dl, A[1:2], B[1:2], C[1:2], 0.0)
    np.testing.assert_allclose(y4[1, 2], ref, rtol=1e-12, atol=1e-12)


def pin_orientations(oracle_mod, lib=None):
    """Four orientations = four top-left scans of the flipped map, flipped back, + D x once."""
    d = _small(H=5, W=7, N=2, channels=2, batch=1, seed=7, orient_mask=0xF)
    y = _fwd(oracle_mod, d, lib)
    ref = d["Dskip"][None, :, None, None].astype(np.float64) * d["x"].astype(np.float64)
    for k, (fh, fw) in enumerate([(0, 0), (0, 1), (1, 0), (1, 1)]):
        axes = tuple(ax for ax, f in ((2, fh), (3, fw)) if f)
        fl = (lambda a: np.flip(a, axes).copy()) if axes else (lambda a: a.copy())
        flb = (lambda a: np.flip(a, tuple(ax + 1 for ax in axes)).copy()) if axes else (lambda a: a.copy())
        yk = oracle_mod.scan2d_fwd(fl(d["x"]), fl(d["delta"]), d["A"], flb(d["B"][:, k:k + 1]),
                                   flb(d["C"][:, k:k + 1]), None, 1)
        ref = ref + fl(yk)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
    # and a subset mask uses B_k, C_k in set-bit order
    d2 = dict(d)
    d2["B"] = d["B"][:, [1, 3]].copy()
    d2["C"] = d["C"][:, [1, 3]].copy()
    y2 = _fwd(oracle_mod, d2, lib, mask=0b1010)
    d3 = dict(d)
    d3["B"] = d["B"][:, [1]].copy()
    d3["C"] = d["C"][:, [1]].copy()
    d4 = dict(d)
    d4["B"] = d["B"][:, [3]].copy()
    d4["C"] = d["C"][:, [3]].copy()
    Dx = d["Dskip"][None, :, None, None].astype(np.float64) * d["x"].astype(np.float64)
    ysum = _fwd(oracle_mod, d3, lib, mask=0b0010) + _fwd(oracle_mod, d4, lib, mask=0b1000) - Dx
    np.testing.assert_allclose(y2, ysum, rtol=1e-12, atol=1e-12)


VFIRST = 0x10     # oracle mask bit: vertical-then-horizontal scan order


def pin_vfirst_closed_form(oracle_mod, lib=None):
    """Vertical-first order ("scan order" ablation, papernotes.org): brute-force path sums."""
    for (H, W, N, seed) in [(6, 5, 3, 11), (4, 8, 2, 12)]:
        d = _small(H=H, W=W, N=N, channels=2, batch=1, seed=seed, random_A=True)
        y = _fwd(oracle_mod, d, lib, mask=1 | VFIRST)
        for ch in range(2):
            np.testing.assert_allclose(y[0, ch], closed_form_map_vfirst(*_map_args(d, 0, ch)),
                                       rtol=1e-12, atol=1e-12)


def pin_vfirst_transpose(oracle_mod, lib=None):
    """Vertical-first on a map = horizontal-first on the transposed map, transposed back
    (flip W and flip H trade places under the transpose)."""
    d = _small(H=5, W=7, N=3, channels=2, batch=2, seed=13, random_A=True)
    T = lambda a: np.swapaxes(a, -1, -2).copy()
    for o, o_t in ((0, 0), (1, 2), (2, 1), (3, 3)):          # TL, TR, BL, BR -> TL, BL, TR, BR
        y = _fwd(oracle_mod, d, lib, mask=(1 << o) | VFIRST)
        yt = oracle_mod.scan2d_fwd(T(d["x"]), T(d["delta"]), d["A"], T(d["B"]), T(d["C"]), d["Dskip"],
                                   1 << o_t, lib=lib)
        np.testing.assert_allclose(y, T(yt), rtol=1e-12, atol=1e-12)
    # the order matters when Abar varies (the two orders are different operators)
    yh = _fwd(oracle_mod, d, lib, mask=1)
    yv = _fwd(oracle_mod, d, lib, mask=1 | VFIRST)
    assert np.max(np.abs(yh - yv)) > 1e-6


def pin_points_and_maps(oracle_mod, lib=None):
    d = _small(H=9, W=11, N=3, channels=3, batch=2, seed=8, orient_mask=0b1101)
    y = _fwd(oracle_mod, d, lib)
    pts = [(0, 0, 0, 0), (1, 2, 8, 10), (0, 1, 4, 0), (1, 0, 0, 10), (1, 1, 5, 6)]
    yp = oracle_mod.scan2d_points(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], pts,
                                  d["orient_mask"], lib=lib)
    np.testing.assert_allclose(yp, [y[p] for p in pts], rtol=1e-13, atol=1e-13)
    ym = oracle_mod.scan2d_maps(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"],
                                [(1, 2), (0, 1)], d["orient_mask"], lib=lib)
    np.testing.assert_array_equal(ym[0], y[1, 2])
    np.testing.assert_array_equal(ym[1], y[0, 1])


# ----------------------------------------------------------------------------------------
# gradients: the pages give no backward pass, so its oracle is pinned by routes that do not
# share its adjoint recurrences (automatic differentiation, finite differences)
# ----------------------------------------------------------------------------------------
def torch_forward(x, dl, A, B, C, D, mask):
    """The forward written once more with torch fp64 tensors, every (b, d, n) at once and a
    Python loop over positions: orientations as flips of the inputs and of y."""
    import torch
    batch, ch, H, W = x.shape
    y = D[None, :, None, None] * x
    k = 0
    for o in range(4):
        if not (mask >> o) & 1:
            continue
        dims = ([3] if o & 1 else []) + ([2] if o & 2 else [])
        fl = (lambda t: torch.flip(t, dims)) if dims else (lambda t: t)
        xf, df = fl(x), fl(dl)
        Bf, Cf = fl(B[:, k]), fl(C[:, k])                          # (batch, N, H, W)
        a = torch.exp(df[:, :, None] * A[None, :, :, None, None])   # (batch, ch, N, H, W)
        u = df[:, :, None] * Bf[:, None] * xf[:, :, None]
        rows = []
        col = [torch.zeros_like(a[..., 0, 0]) for _ in range(W)]
        for i in range(H):
            run = torch.zeros_like(a[..., 0, 0])
            out = []
            for j in range(W):
                if not mask & 0x10:
                    run = a[..., i, j] * run + u[..., i, j]           # horizontal
                    col[j] = a[..., i, j] * col[j] + run            # vertical
                    h = col[j]
                else:
                    col[j] = a[..., i, j] * col[j] + u[..., i, j]   # vertical first
                    run = a[..., i, j] * run + col[j]
                    h = run
                out.append((Cf[:, None, :, i, j] * h).sum(2))
            rows.append(torch.stack(out, -1))
        y = y + fl(torch.stack(rows, -2))
        k += 1
    return y


def _bwd(oracle_mod, d, dy, lib=None, mask=None, majorant=False):
    return oracle_mod.scan2d_bwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], dy,
                                 d["orient_mask"] if mask is None else mask, majorant=majorant, lib=lib)


def pin_bwd_autograd(oracle_mod, lib=None):
    """Every gradient against torch's reverse-mode differentiation of the forward above,
    both scan orders, one and four orientations; the majorant bounds each gradient."""
    import torch
    for seed, mask, dtype in ((21, 0b0001, "f32"), (22, 0b1111, "f32"), (23, 0b1011 | VFIRST, "bf16"),
                              (24, 0b0001 | VFIRST, "f32")):
        d = _small(H=5, W=6, N=3, channels=2, batch=2, seed=seed, dtype=dtype, orient_mask=mask & 0xF)
        dy = np.random.default_rng(seed).standard_normal(d["x"].shape)
        T = {k: torch.tensor(_f64(d[k]), requires_grad=True) for k in ("x", "delta", "B", "C")}
        TA = torch.tensor(d["A"].astype(np.float64), requires_grad=True)
        TD = torch.tensor(d["Dskip"].astype(np.float64), requires_grad=True)
        y = torch_forward(T["x"], T["delta"], TA, T["B"], T["C"], TD, mask)
        np.testing.assert_allclose(y.detach().numpy(), _fwd(oracle_mod, d, lib, mask=mask),
                                   rtol=1e-12, atol=1e-12)
        (y * torch.tensor(dy)).sum().backward()
        g = _bwd(oracle_mod, d, dy, lib, mask=mask)
        want = {"dx": T["x"].grad, "ddelta": T["delta"].grad, "dA": TA.grad, "dB": T["B"].grad,
                "dC": T["C"].grad, "dDskip": TD.grad}
        maj = _bwd(oracle_mod, d, dy, lib, mask=mask, majorant=True)
        for name, ref in want.items():
            np.testing.assert_allclose(g[name], ref.numpy(), rtol=1e-10, atol=1e-12, err_msg=name)
            assert np.all(maj[name] >= np.abs(g[name]) * (1 - 1e-12)), name


def pin_bwd_finite_difference(oracle_mod, lib=None):
    """Central differences of sum(dy * y) through the forward oracle, at a few entries of
    every input, against the gradients."""
    d = _small(H=4, W=5, N=2, channels=2, batch=1, seed=31, orient_mask=0b0110)
    rng = np.random.default_rng(31)
    dy = rng.standard_normal(d["x"].shape)
    g = _bwd(oracle_mod, d, dy, lib)
    loss = lambda dd: float(np.sum(dy * _fwd(oracle_mod, dd, lib)))
    for name, gname in (("x", "dx"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC"),
                        ("Dskip", "dDskip")):
        for _ in range(3):
            idx = tuple(int(rng.integers(0, n)) for n in d[name].shape)
            plus, minus = dict(d), dict(d)
            plus[name], minus[name] = d[name].copy(), d[name].copy()
            v = float(d[name][idx])
            eps = 1e-2 * max(abs(v), 0.1)
            plus[name][idx] = np.float32(v + eps)
            minus[name][idx] = np.float32(v - eps)
            step = float(plus[name][idx]) - float(minus[name][idx])
            fd = (loss(plus) - loss(minus)) / step
            assert abs(fd - g[gname][idx]) <= 2e-4 * (1 + abs(fd)), (name, idx, fd, g[gname][idx])


PINS = [pin_closed_form, pin_linsolve, pin_manhattan_constant, pin_golden_3x3,
        pin_1d_reduction, pin_linearity_and_special, pin_orientations, pin_vfirst_closed_form,
        pin_vfirst_transpose, pin_points_and_maps, pin_bwd_autograd, pin_bwd_finite_difference]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(oracle_mod, pin):
    pin(oracle_mod)


def test_bf16_inputs_widen_exactly(oracle_mod):
    d = _small(H=6, W=5, N=3, channels=2, batch=1, seed=9, dtype="bf16", orient_mask=0b0110)
    y = _fwd(oracle_mod, d)
    f = dict(d)
    for k in ("x", "delta", "B", "C"):
        f[k] = inputs.bf16_bits_to_f32(d[k])
    np.testing.assert_array_equal(y, _fwd(oracle_mod, f))


def test_bf16_rounding_is_nearest_even():
    v = np.array([1.0, 1.00390625, 1.005859375, -2.5, 3.0e-3], np.float32)
    bits = inputs.f32_to_bf16_bits(v)
    back = inputs.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins
    assert back[0] == 1.0 and back[1] == 1.0
    assert back[2] == np.float32(1.0078125)
    assert back[3] == -2.5
    assert abs(back[4] - 3.0e-3) <= 3.0e-3 * 2 ** -8


def test_oracle_rejects_bad_arguments(oracle_mod):
    d = _small()
    with pytest.raises((RuntimeError, ValueError)):
        _fwd(oracle_mod, d, mask=0)
    with pytest.raises(RuntimeError):
        oracle_mod.scan2d_points(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"],
                                 [(0, 0, 8, 0)], 1)


# ----------------------------------------------------------------------------------------
# planted mistakes: a copy of the oracle with one plausible error must fail some pin
# ----------------------------------------------------------------------------------------
MUTATIONS = {
    "vertical_without_decay": ("hcol[jj] = abar * hcol[jj] + hh;", "hcol[jj] = hcol[jj] + hh;"),
    "bbar_without_delta": ("hh = abar * hh + (dl * Bv) * xv;", "hh = abar * hh + Bv * xv;"),
    "exp_sign": ("exp(dl * An)", "exp(-dl * An)"),
    "no_skip_term": ("ym[pos] += Dd * load(x, map + pos, is_bf16);", "(void)Dd;"),
    "flip_w_ignored": ("const int j = flipW ? W - 1 - jj : jj;", "const int j = jj;"),
    "C_transposed": ("load(p->C, bc + pos, p->is_bf16)",
                     "load(p->C, bc + ((size_t)j * H + i) % ((size_t)H * W), p->is_bf16)"),
    "vertical_adds_bbar_again": ("hcol[jj] = abar * hcol[jj] + hh;",
                                 "hcol[jj] = abar * hcol[jj] + hh + (dl * Bv) * xv;"),
    "horizontal_carry_not_reset": ("double hh = 0.0;                               /* hh[i, -1] = 0 */",
                                   "static double hh; if (ii == 0) hh = 0.0;"),
    "state_index_off_by_one": ("const double An = (double)p->A[(size_t)d * N + n];",
                               "const double An = (double)p->A[(size_t)d * N + (n + 1) % N];"),
    "vfirst_ignored": ("const int vfirst = p->vfirst;", "const int vfirst = 0;"),
    "vfirst_vertical_without_decay": ("hcol[jj] = abar * hcol[jj] + (dl * Bv) * xv;",
                                      "hcol[jj] = hcol[jj] + (dl * Bv) * xv;"),
    "bwd_drop_first_scan_term": ("const double dabar = g2[t] * s2_prev + g1[t] * s1_prev;",
                                 "const double dabar = g2[t] * s2_prev;"),
    "bwd_adjoint_unshifted_decay": ("g2[t] = Cv * gy + (has_d ? a[AT(ii + 1, jj)] * g2[AT(ii + 1, jj)] : 0.0);",
                                    "g2[t] = Cv * gy + (has_d ? a[t] * g2[AT(ii + 1, jj)] : 0.0);"),
    "bwd_dB_without_delta": ("dB[bc + pos] += g1[t] * dl * xv;", "dB[bc + pos] += g1[t] * xv;"),
    "bwd_ddelta_sign": ("ddelta[map + pos] += dabar * a[t] * Af + g1[t] * Bv * xv;",
                        "ddelta[map + pos] += -dabar * a[t] * Af + g1[t] * Bv * xv;"),
    "bwd_dC_first_state": ("dC[bc + pos] += gy * s2[t];", "dC[bc + pos] += gy * s1[t];"),
    "bwd_skip_missing": ("dx[map + pos] += Dd * gy;", "(void)Dd;"),
    "bwd_vfirst_adjoint_order": ("g1[t] = g2[t] + (has_d ? a[AT(ii + 1, jj)] * g1[AT(ii + 1, jj)] : 0.0);",
                                 "g1[t] = g2[t] + (has_r ? a[AT(ii, jj + 1)] * g1[AT(ii, jj + 1)] : 0.0);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(oracle_mod, tmp_path, name):
    src = open(os.path.join(os.path.dirname(oracle_mod.__file__), "scan2d_oracle.c")).read()
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, f"mutation anchor missing: {old}"
    mutated = src.replace(old, new)
    c = tmp_path / "mut.c"
    so = tmp_path / "libmut.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"])
    lib = oracle_mod.load_library(str(so))
    caught = []
    for pin in PINS:
        try:
            pin(oracle_mod, lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"


# ----------------------------------------------------------------------------------------
# the whole-slide grid ("2DMamba 精读", section 四.2, steps 3-4): a worked example typed out
# by hand, and the round trip through the seeded bag generator
# ----------------------------------------------------------------------------------------
def test_wsi_grid_worked_example(oracle_mod):
    feat = np.array([[1, 2], [3, 4], [5, 6], [7, 8]], dtype=np.float32)
    coords = np.array([[0, 1], [1, 2], [0, 1], [5, 0]], dtype=np.int32)   # patch 2 repeats a cell,
    pad = np.array([-1, -2], dtype=np.float32)                            # patch 3 is off the grid
    x, cell, skipped = oracle_mod.wsi_grid(feat, coords, pad, 2, 3)
    assert skipped == 1
    np.testing.assert_array_equal(cell, [-1, 2, -1, -1, -1, 1])
    want = np.array([[[-1, 5, -1], [-1, -1, 3]],
                     [[-2, 6, -2], [-2, -2, 4]]], dtype=np.float32)[None]
    np.testing.assert_array_equal(x, want)


def test_wsi_grid_round_trip(oracle_mod):
    for dtype in ("f32", "bf16"):
        w = inputs.WORKLOADS["wsi"].scaled(channels=5, H=19, W=26, dtype=dtype)
        b = inputs.make_wsi_bag(w, 4)
        x, cell, skipped = oracle_mod.wsi_grid(b["feat"], b["coords"], b["pad"], w.H, w.W)
        assert skipped == 0
        np.testing.assert_array_equal(x, b["x"])
        assert int((cell >= 0).sum()) == b["feat"].shape[0] == int(b["tissue"].sum())
        # every non-tissue cell holds the token
        assert np.all(x[0][:, ~b["tissue"]] == b["pad"][:, None])


# ----------------------------------------------------------------------------------------
# input projections (reading of "2DMamba 精读", section 四.4): special cases with closed forms
# and a second library route (torch)
# ----------------------------------------------------------------------------------------
def test_proj_special_cases(oracle_mod):
    import math
    rng = np.random.default_rng(5)
    D, N, R = 6, 3, 2
    x = rng.standard_normal((2, D, 3, 4)).astype(np.float32)
    bdt = np.array([-3.0, -1.0, 0.0, 0.5, 2.0, 30.0], np.float32)
    # Wdt = 0: delta is softplus(bdt) everywhere; softplus(0) = ln 2 and softplus(30) ~ 30
    Wx = rng.standard_normal((R + 2 * N, D)).astype(np.float32)
    delta, B, C = oracle_mod.proj(x, Wx, np.zeros((D, R), np.float32), bdt, N, R)
    for d in range(D):
        want = math.log1p(math.exp(float(bdt[d])))
        np.testing.assert_allclose(delta[:, d], want, rtol=1e-15, atol=0)
    assert abs(oracle_mod.softplus(0.0) - math.log(2.0)) < 1e-15
    # unit rows select channels: B[n] = x[c_n], C[n] = -x[c'_n]
    Wsel = np.zeros((R + 2 * N, D), np.float32)
    picks = [4, 0, 5]
    for n, c in enumerate(picks):
        Wsel[R + n, c] = 1.0
        Wsel[R + N + n, (c + 1) % D] = -1.0
    _, B, C = oracle_mod.proj(x, Wsel, np.zeros((D, R), np.float32), bdt, N, R)
    for n, c in enumerate(picks):
        np.testing.assert_array_equal(B[:, n], x[:, c].astype(np.float64))
        np.testing.assert_array_equal(C[:, n], -x[:, (c + 1) % D].astype(np.float64))


def test_proj_against_torch(oracle_mod):
    import torch
    rng = np.random.default_rng(6)
    D, N, R = 10, 4, 3
    x = rng.standard_normal((2, D, 5, 7)).astype(np.float32)
    w = inputs.make_proj_weights(D, N, R, seed=2)
    delta, B, C = oracle_mod.proj(x, w["Wx"], w["Wdt"], w["bdt"], N, R)
    xt = torch.tensor(x, dtype=torch.float64).permute(0, 2, 3, 1)          # (b, h, w, D)
    u = xt @ torch.tensor(w["Wx"], dtype=torch.float64).T                   # (b, h, w, R + 2N)
    z = u[..., :R] @ torch.tensor(w["Wdt"], dtype=torch.float64).T + torch.tensor(w["bdt"], dtype=torch.float64)
    np.testing.assert_allclose(delta, torch.nn.functional.softplus(z).permute(0, 3, 1, 2).numpy(), rtol=1e-12)
    np.testing.assert_allclose(B, u[..., R:R + N].permute(0, 3, 1, 2).numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(C, u[..., R + N:].permute(0, 3, 1, 2).numpy(), rtol=1e-12, atol=1e-14)


def test_bwd_single_cell_closed_form(oracle_mod):
    """A 1 x 1 map: y = sum_n C_n dt B_n x + D x, so every gradient has a closed form
    (Abar never multiplies anything, so dA = 0)."""
    rng = np.random.default_rng(12)
    N = 3
    x = rng.standard_normal((1, 1, 1, 1)).astype(np.float32)
    dt = np.abs(rng.standard_normal((1, 1, 1, 1))).astype(np.float32)
    A = -rng.random((1, N)).astype(np.float32)
    B = rng.standard_normal((1, 1, N, 1, 1)).astype(np.float32)
    C = rng.standard_normal((1, 1, N, 1, 1)).astype(np.float32)
    D = rng.standard_normal(1).astype(np.float32)
    dy = rng.standard_normal((1, 1, 1, 1))
    for mask in (1, 1 | VFIRST):
        g = oracle_mod.scan2d_bwd(x, dt, A, B, C, D, dy, mask)
        xs, ds, gys = float(x[0, 0, 0, 0]), float(dt[0, 0, 0, 0]), float(dy[0, 0, 0, 0])
        Bv = B[0, 0, :, 0, 0].astype(np.float64)
        Cv = C[0, 0, :, 0, 0].astype(np.float64)
        np.testing.assert_allclose(g["dx"][0, 0, 0, 0], gys * (ds * np.dot(Bv, Cv) + float(D[0])), rtol=1e-14)
        np.testing.assert_allclose(g["ddelta"][0, 0, 0, 0], gys * xs * np.dot(Bv, Cv), rtol=1e-14)
        np.testing.assert_array_equal(g["dA"], 0.0)
        np.testing.assert_allclose(g["dB"][0, 0, :, 0, 0], gys * Cv * ds * xs, rtol=1e-14)
        np.testing.assert_allclose(g["dC"][0, 0, :, 0, 0], gys * Bv * ds * xs, rtol=1e-14)
        np.testing.assert_allclose(g["dDskip"][0], gys * xs, rtol=1e-14)
