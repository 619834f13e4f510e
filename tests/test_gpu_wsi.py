"""The whole-slide grid on the GPU, through the C ABI: the cell map and the gathered map are
bit-exact against the oracle's grid (pure data movement), and the scan that reads x through
the cell map (scan2d_fwd_wsi) meets the forward's bound against the fp64 oracle run on the
oracle's map: |y - y_ref| <= TOL * (1 + |y_ref|)."""
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


def _bits(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def _grid_gpu(feat, coords, pad, H, W):
    import torch
    from selective_state_space_scan2d_b200 import scan2d
    c = _dev(coords)
    skipped = torch.zeros(1, dtype=torch.int32, device="cuda")
    cell = scan2d.scan2d_grid_cells(c, H, W, n_skipped=skipped)
    x = scan2d.scan2d_grid_gather(_dev(feat), cell, _dev(pad), H, W)
    torch.cuda.synchronize()
    return _bits(x), cell.cpu().numpy(), int(skipped.item())


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_grid_bit_exact(oracle_mod, dtype):
    w = inputs.WORKLOADS["wsi"].scaled(channels=40, H=21, W=37, dtype=dtype)   # ragged tiles
    b = inputs.make_wsi_bag(w, 7)
    x, cell, sk = _grid_gpu(b["feat"], b["coords"], b["pad"], w.H, w.W)
    xr, cellr, skr = oracle_mod.wsi_grid(b["feat"], b["coords"], b["pad"], w.H, w.W)
    assert sk == skr == 0
    np.testing.assert_array_equal(cell, cellr)
    np.testing.assert_array_equal(x, xr)


def test_grid_duplicates_outside_and_empty(oracle_mod):
    rng = np.random.default_rng(3)
    H, W, D = 9, 11, 33
    coords = np.stack([rng.integers(-2, H + 2, 300), rng.integers(-2, W + 2, 300)], 1).astype(np.int32)
    feat = rng.standard_normal((300, D)).astype(np.float32)
    pad = rng.standard_normal(D).astype(np.float32)
    x, cell, sk = _grid_gpu(feat, coords, pad, H, W)
    xr, cellr, skr = oracle_mod.wsi_grid(feat, coords, pad, H, W)
    assert sk == skr > 0
    np.testing.assert_array_equal(cell, cellr)
    np.testing.assert_array_equal(x, xr)
    # an empty bag: every cell holds the token
    x0, cell0, sk0 = _grid_gpu(np.zeros((0, D), np.float32), np.zeros((0, 2), np.int32), pad, H, W)
    assert sk0 == 0 and np.all(cell0 == -1)
    np.testing.assert_array_equal(x0, np.broadcast_to(pad[None, :, None, None], (1, D, H, W)))


def test_grid_full_size_wsi(oracle_mod):
    """1 x 128 x 160 x 224, fp32, the workload's own mask: bit-exact."""
    w = inputs.WORKLOADS["wsi"]
    b = inputs.make_wsi_bag(w, 0)
    x, cell, sk = _grid_gpu(b["feat"], b["coords"], b["pad"], w.H, w.W)
    assert sk == 0
    np.testing.assert_array_equal(x, b["x"])
    np.testing.assert_array_equal(cell >= 0, b["tissue"].reshape(-1))


def _flags(w):
    from selective_state_space_scan2d_b200 import scan2d
    return scan2d.flags_for(w.dtype == "bf16", w.orient_mask)


def _fwd_wsi(b, w):
    from selective_state_space_scan2d_b200 import scan2d
    t = to_torch(b)
    cell = scan2d.scan2d_grid_cells(_dev(b["coords"]), w.H, w.W)
    y = scan2d.scan2d_fwd_wsi(_dev(b["feat"]), cell, _dev(b["pad"]), t["delta"], t["A"], t["B"], t["C"], t["Dskip"],
                              flags=_flags(w))
    assert scan2d.scan2d_get_device_error() == 0
    return y, t


@pytest.mark.parametrize("dtype,mask", [("f32", 1), ("bf16", 0xF), ("f32", 0b0110)])
def test_fused_forward_parity(oracle_mod, dtype, mask):
    from selective_state_space_scan2d_b200 import scan2d
    w = inputs.WORKLOADS["wsi"].scaled(channels=24, H=19, W=45, dtype=dtype, orient_mask=mask)
    b = inputs.make_wsi_bag(w, 2)
    y, t = _fwd_wsi(b, w)
    xr, _, _ = oracle_mod.wsi_grid(b["feat"], b["coords"], b["pad"], w.H, w.W)
    ref = oracle_mod.scan2d_fwd(xr, b["delta"], b["A"], b["B"], b["C"], b["Dskip"], mask)
    assert_parity(y_to_f64(y), ref, TOL[dtype], f"fused wsi {dtype} mask {mask}")
    # the map written by the grid step and scanned by scan2d_fwd gives the same y within the bound
    x = scan2d.scan2d_grid_gather(_dev(b["feat"]), scan2d.scan2d_grid_cells(_dev(b["coords"]), w.H, w.W),
                                  _dev(b["pad"]), w.H, w.W)
    y2 = scan2d.scan2d_fwd(x, t["delta"], t["A"], t["B"], t["C"], t["Dskip"], flags=_flags(w))
    assert_parity(y_to_f64(y2), ref, TOL[dtype], "unfused")


def test_fused_forward_full_size_wsi_sampled(oracle_mod):
    """The workload at full size (1 x 128 x 160 x 224, fp32): y at sampled positions, each
    computed by the oracle over the rectangle that reaches it."""
    w = inputs.WORKLOADS["wsi"]
    b = inputs.make_wsi_bag(w, 0)
    y, _ = _fwd_wsi(b, w)
    y = y_to_f64(y)
    rng = np.random.default_rng(11)
    pts = [(0, int(d), int(i), int(j)) for d, i, j in zip(rng.integers(0, w.channels, 24),
                                                           rng.integers(0, w.H, 24), rng.integers(0, w.W, 24))]
    pts += [(0, 0, 0, 0), (0, 127, w.H - 1, w.W - 1)]
    ref = oracle_mod.scan2d_points(b["x"], b["delta"], b["A"], b["B"], b["C"], b["Dskip"], pts, 1)
    got = np.array([y[p] for p in pts])
    assert_parity(got, ref, TOL["f32"], "fused wsi full size")
