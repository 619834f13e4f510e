"""Helpers shared by the GPU tests: numpy inputs -> torch CUDA tensors, the parity bound."""
import numpy as np

from selective_state_space_scan2d_b200 import inputs

# Parity bound, element by element: |y_gpu - y_ref| <= TOL * (1 + |y_ref|)
TOL = {"f32": 1e-5, "bf16": 2e-2}


def to_torch(d, device="cuda"):
    import torch

    def conv(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(a).to(device)

    return {k: conv(d[k]) for k in ("x", "delta", "A", "B", "C", "Dskip")}


def y_to_f64(y):
    import torch
    return y.detach().to("cpu", torch.float64).numpy()


def run_gpu(d, flags=None, stream=None):
    from selective_state_space_scan2d_b200 import scan2d
    t = to_torch(d)
    if flags is None:
        flags = scan2d.flags_for(d["x"].dtype == np.uint16, d["orient_mask"], vfirst=d.get("vfirst", False))
    return scan2d.scan2d_fwd(t["x"], t["delta"], t["A"], t["B"], t["C"], t["Dskip"],
                             flags=flags, stream=stream)


def max_violation(y, ref, tol):
    """max over elements of |y - ref| / (tol * (1 + |ref|)); <= 1 passes."""
    return float(np.max(np.abs(y - ref) / (tol * (1.0 + np.abs(ref)))))


def assert_parity(y, ref, tol, label=""):
    """Element-wise bound |y - ref| <= tol (1 + |ref|), with a diagnosis on failure."""
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    ratio = np.abs(y - ref) / (tol * (1.0 + np.abs(ref)))
    worst = float(np.nanmax(ratio)) if ratio.size else 0.0
    if not (worst <= 1.0) or not np.all(np.isfinite(y)):
        bad = ratio > 1.0
        idx = np.unravel_index(int(np.nanargmax(ratio)), ratio.shape)
        raise AssertionError(
            f"{label}: parity violated at {int(bad.sum())} of {ratio.size} elements; worst "
            f"{worst:.3g}x the bound at {tuple(int(v) for v in idx)}: got {y[idx]!r}, "
            f"want {ref[idx]!r}; non-finite outputs: {int((~np.isfinite(y)).sum())}")
    return worst


def workload(name, **kw):
    w = inputs.WORKLOADS[name]
    return w.scaled(**kw) if kw else w
