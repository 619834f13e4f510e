"""scan2d_fwd_noalloc: the forward for callers that must not allocate device memory.

Such callers include runtimes whose allocator has reserved the device memory they may use,
operator or plugin interfaces that forbid allocating inside their execute call, and
latency-bound loops that cannot take the device-wide synchronisation of cudaMalloc/cudaFree.
scan2d_fwd would allocate a per-stream workspace on first need; scan2d_fwd_noalloc takes the
same scratch from one fixed device array inside the library instead.

These tests call it through the C ABI on shapes whose plan needs scratch memory (the
cross-block carry ring; the fp32 accumulator of several orientations with bf16 output) and
compare it with scan2d_fwd, within the parity bound of the other tests, on two calls in a
row of each shape, with calls of other shapes in between.  The file is named to be
collected last; it passes on its own in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest

from selective_state_space_scan2d_b200 import inputs
from scan2d_cases import CASES
from scan2d_testlib import TOL, assert_parity, to_torch, workload, y_to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

# shapes whose launch plan uses scratch: global carry rings (TMA and plain loads), and the
# fp32 accumulator of four orientations with bf16 output
SCRATCH_CASES = ("f32_global_ring_tma", "bf16_k4_across_blocks", "f32_long_chain_backpressure")


def _args(t, y):
    return [t["x"].data_ptr(), t["delta"].data_ptr(), t["A"].data_ptr(), t["B"].data_ptr(),
            t["C"].data_ptr(), t["Dskip"].data_ptr() if t["Dskip"] is not None else None,
            y.data_ptr()]


def _call_noalloc(t, y, w, flags, stream):
    from selective_state_space_scan2d_b200 import scan2d
    return scan2d.raw().scan2d_fwd_noalloc(*_args(t, y), w.batch, w.channels, w.H, w.W, w.N,
                                           flags, ctypes.c_void_p(stream.cuda_stream))


def test_noalloc_matches_scan2d_fwd_on_two_calls_in_a_row():
    from selective_state_space_scan2d_b200 import scan2d
    stream = torch.cuda.current_stream()
    # every scratch shape twice in a row, then the first one again after the others
    order = [c for c in SCRATCH_CASES for _ in range(2)] + [SCRATCH_CASES[0]] * 2
    prepared = {}
    for case in SCRATCH_CASES:
        name, kw = CASES[case]
        w = workload(name, **kw)
        flags = scan2d.flags_for(w.dtype == "bf16", w.orient_mask)
        assert scan2d.scan2d_query_plan(w.batch, w.channels, w.H, w.W, w.N, flags)["workspace"] > 0
        d = inputs.make_inputs(w, seed=31)
        t = to_torch(d)
        ref = scan2d.scan2d_fwd(t["x"], t["delta"], t["A"], t["B"], t["C"], t["Dskip"], flags=flags)
        torch.cuda.synchronize()
        prepared[case] = (w, flags, t, y_to_f64(ref))
    for n, case in enumerate(order):
        w, flags, t, ref = prepared[case]
        y = torch.full((w.batch, w.channels, w.H, w.W), float("nan"),
                       dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32, device="cuda")
        rc = _call_noalloc(t, y, w, flags, stream)
        assert rc == 0, scan2d.scan2d_strerror(rc)
        assert scan2d.scan2d_get_device_error(stream) == 0
        assert_parity(y_to_f64(y), ref, TOL[w.dtype], f"call {n}: {case}")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from selective_state_space_scan2d_b200 import scan2d
    # four orientations, bf16 output, maps too large for shared memory: the fp32 accumulator
    # alone (8 x 1024 x 1100 floats, 36 MB) exceeds the fixed scratch
    w = inputs.Workload("too_large", batch=1, channels=8, N=16, H=1024, W=1100, dtype="bf16",
                        orient_mask=0xF)
    flags = scan2d.flags_for(True, 0xF)
    assert scan2d.scan2d_query_plan(1, 8, 1024, 1100, 16, flags)["workspace"] > scan2d.SCAN2D_NOALLOC_SCRATCH_BYTES
    xy = torch.empty(1, 8, 1024, 1100, dtype=torch.bfloat16, device="cuda")
    bc = torch.empty(1, 4, 16, 1024, 1100, dtype=torch.bfloat16, device="cuda")
    t = {"x": xy, "delta": xy, "A": torch.empty(8, 16, device="cuda"), "B": bc, "C": bc, "Dskip": None}
    y = torch.empty_like(xy)
    rc = _call_noalloc(t, y, w, flags, torch.cuda.current_stream())
    assert rc == scan2d.SCAN2D_E_SCRATCH
    assert "SCAN2D_NOALLOC_SCRATCH_BYTES" in scan2d.scan2d_strerror(rc)
    torch.cuda.synchronize()
