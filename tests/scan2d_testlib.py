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
        flags = scan2d.flags_for(d["x"].dtype == np.uint16, d["orient_mask"])
    return scan2d.scan2d_fwd(t["x"], t["delta"], t["A"], t["B"], t["C"], t["Dskip"],
                             flags=flags, stream=stream)


def max_violation(y, ref, tol):
    """max over elements of |y - ref| / (tol * (1 + |ref|)); <= 1 passes."""
    return float(np.max(np.abs(y - ref) / (tol * (1.0 + np.abs(ref)))))


def workload(name, **kw):
    w = inputs.WORKLOADS[name]
    return w.scaled(**kw) if kw else w
