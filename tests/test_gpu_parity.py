"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, element by element,
on identical seeded inputs.  Bound: |y - y_ref| <= 1e-5 (1 + |y_ref|) for fp32 inputs and
2e-2 (1 + |y_ref|) for bf16 inputs."""
import numpy as np
import pytest

from selective_state_space_scan2d_b200 import inputs
from scan2d_cases import CASES
from scan2d_testlib import TOL, assert_parity, max_violation, run_gpu, to_torch, workload, y_to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _oracle_full(oracle_mod, d, mask=None):
    if mask is None:
        mask = d["orient_mask"] | (0x10 if d.get("vfirst") else 0)   # oracle bit 4: vertical first
    return oracle_mod.scan2d_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], mask)


def _check_full(oracle_mod, d, flags=None, mask=None):
    y = y_to_f64(run_gpu(d, flags))
    torch.cuda.synchronize()
    ref = _oracle_full(oracle_mod, d, mask)
    v = assert_parity(y, ref, TOL[d["workload"].dtype], d["workload"].name)
    from selective_state_space_scan2d_b200 import scan2d
    assert scan2d.scan2d_get_device_error() == 0
    return v


@pytest.mark.parametrize("case", sorted(CASES))
def test_parity_small(oracle_mod, case):
    name, kw = CASES[case]
    d = inputs.make_inputs(workload(name, **kw), seed=11)
    _check_full(oracle_mod, d)


def test_bf16_with_fp32_output(oracle_mod):
    from selective_state_space_scan2d_b200 import scan2d
    d = inputs.make_inputs(workload("vision", batch=1, channels=9, H=12, W=20), seed=3)
    y = run_gpu(d, flags=scan2d.flags_for(True, 0xF, out_f32=True))
    assert y.dtype == torch.float32
    ref = _oracle_full(oracle_mod, d)
    assert max_violation(y_to_f64(y), ref, TOL["bf16"]) <= 1.0


def test_repeat_is_bitwise_identical():
    d = inputs.make_inputs(workload("tiny", batch=1, channels=16, N=16, H=33, W=300), seed=5)
    a = run_gpu(d)
    b = run_gpu(d)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_two_streams_concurrently(oracle_mod):
    """Each stream gets its own workspace: concurrent chained launches stay correct."""
    d1 = inputs.make_inputs(workload("tiny", batch=1, channels=8, N=16, H=30, W=400), seed=1)
    d2 = inputs.make_inputs(workload("tiny", batch=1, channels=8, N=16, H=30, W=400), seed=2)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s1):
        y1 = run_gpu(d1, stream=s1)
    with torch.cuda.stream(s2):
        y2 = run_gpu(d2, stream=s2)
    torch.cuda.synchronize()
    for d, y in ((d1, y1), (d2, y2)):
        assert max_violation(y_to_f64(y), _oracle_full(oracle_mod, d), TOL["f32"]) <= 1.0


def test_host_entry_point_matches_device():
    from selective_state_space_scan2d_b200 import scan2d
    d = inputs.make_inputs(workload("small", batch=4, channels=24, H=14, W=14), seed=4)
    yd = run_gpu(d)
    t = to_torch(d, device="cpu")
    t = {k: (v.pin_memory() if v is not None else None) for k, v in t.items()}
    flags = scan2d.flags_for(True, 1)
    nbytes = scan2d.scan2d_host_staging_bytes(4, 24, 14, 14, 16, flags)
    staging = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    yh = torch.empty(4, 24, 14, 14, dtype=torch.bfloat16).pin_memory()
    scan2d.scan2d_fwd_host(t["x"], t["delta"], t["A"], t["B"], t["C"], t["Dskip"], yh, staging, flags)
    torch.cuda.synchronize()
    assert torch.equal(yh, yd.cpu())


# ---- full-size workloads, same launch configuration as the benchmark ----------------------
FULL = {
    # workload: (number of whole maps checked, number of extra points)
    "wsi": (3, 24),
    "small": (48, 24),
    "vision": (12, 24),
    "giga": (2, 12),
}


@pytest.mark.parametrize("name", sorted(FULL))
def test_full_size_sampled(oracle_mod, name):
    w = inputs.WORKLOADS[name]
    d = inputs.make_inputs(w, seed=0)
    y = run_gpu(d)
    torch.cuda.synchronize()
    from selective_state_space_scan2d_b200 import scan2d
    assert scan2d.scan2d_get_device_error() == 0
    rng = np.random.default_rng(123)
    nmaps, npts = FULL[name]
    maps = {(int(rng.integers(w.batch)), int(rng.integers(w.channels))) for _ in range(nmaps)}
    maps.add((w.batch - 1, w.channels - 1))
    maps = sorted(maps)
    ym = oracle_mod.scan2d_maps(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], maps,
                                d["orient_mask"])
    tol = TOL[w.dtype]
    for m, (b, ch) in enumerate(maps):
        got = y[b, ch].to("cpu", torch.float64).numpy()
        assert_parity(got, ym[m], tol, f"{name} map {(b, ch)}")
    pts = [(w.batch - 1, w.channels - 1, w.H - 1, w.W - 1), (0, 0, w.H - 1, 0), (0, 0, 0, w.W - 1)]
    for _ in range(npts):
        pts.append((int(rng.integers(w.batch)), int(rng.integers(w.channels)),
                    int(rng.integers(w.H)), int(rng.integers(w.W))))
    yp = oracle_mod.scan2d_points(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], pts,
                                  d["orient_mask"])
    got = np.array([float(y[p]) for p in pts])
    assert_parity(got, yp, tol, f"{name} points")


def test_full_size_random_A_giga_shape(oracle_mod):
    """The kernel is not specialised to A = -(n+1): random A at the giga shape."""
    w = inputs.WORKLOADS["giga"].scaled(random_A=True)
    d = inputs.make_inputs(w, seed=1)
    y = run_gpu(d)
    torch.cuda.synchronize()
    maps = [(0, 5), (0, 127)]
    ym = oracle_mod.scan2d_maps(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], maps, 1)
    for m, (b, ch) in enumerate(maps):
        got = y[b, ch].to("cpu", torch.float64).numpy()
        assert_parity(got, ym[m], TOL["f32"], f"random-A map {(b, ch)}")


def test_workspace_reuse_across_shapes(oracle_mod):
    """A chained call after calls of other shapes on the same stream: the earlier calls'
    carry values must never be read as the later call's flags."""
    s = torch.cuda.Stream()
    big = inputs.make_inputs(workload("tiny", batch=1, channels=16, N=16, H=24, W=1024), seed=21)
    small = inputs.make_inputs(workload("tiny", batch=1, channels=32, N=16, H=24, W=200), seed=22)
    with torch.cuda.stream(s):
        run_gpu(big, stream=s)
        run_gpu(small, stream=s)
        y = run_gpu(big, stream=s)
    s.synchronize()
    from selective_state_space_scan2d_b200 import scan2d
    assert scan2d.scan2d_get_device_error(s) == 0
    assert_parity(y_to_f64(y), _oracle_full(oracle_mod, big), TOL["f32"], "reuse")


def test_full_size_vfirst_giga_shape(oracle_mod):
    """Vertical-then-horizontal order at the giga shape, in the launch configuration of the
    default order (the flag changes only the math inside a row)."""
    w = inputs.WORKLOADS["giga"].scaled(vfirst=True)
    d = inputs.make_inputs(w, seed=2)
    y = run_gpu(d)
    torch.cuda.synchronize()
    from selective_state_space_scan2d_b200 import scan2d
    assert scan2d.scan2d_get_device_error() == 0
    maps = [(0, 3), (0, 126)]
    ym = oracle_mod.scan2d_maps(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], maps, 1 | 0x10)
    for m, (b, ch) in enumerate(maps):
        got = y[b, ch].to("cpu", torch.float64).numpy()
        assert_parity(got, ym[m], TOL["f32"], f"vertical-first map {(b, ch)}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unaligned_buffers_use_plain_loads(oracle_mod, dtype):
    """Buffers that start one element past a 16-byte boundary cannot be staged by TMA: the
    call takes the plain-load path for a shape that would otherwise use TMA."""
    from selective_state_space_scan2d_b200 import scan2d
    name = "small" if dtype == "bf16" else "tiny"
    w = workload(name, batch=1, channels=8, N=16, H=9, W=64)
    d = inputs.make_inputs(w, seed=8)
    t = to_torch(d)

    def shifted(a):               # same values, storage starting one element later
        buf = torch.empty(a.numel() + 1, dtype=a.dtype, device=a.device)
        v = buf[1:].view(a.shape)
        v.copy_(a)
        return v
    s = {k: (shifted(v) if k in ("x", "delta", "B", "C") else v) for k, v in t.items()}
    assert s["x"].data_ptr() % 16 != 0
    y = scan2d.scan2d_fwd(s["x"], s["delta"], s["A"], s["B"], s["C"], s["Dskip"],
                          flags=scan2d.flags_for(dtype == "bf16", 1))
    torch.cuda.synchronize()
    assert scan2d.scan2d_get_device_error() == 0
    assert_parity(y_to_f64(y), _oracle_full(oracle_mod, d), TOL[dtype], f"unaligned {dtype}")
