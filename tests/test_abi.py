"""C-ABI library: builds, loads, exports every function include/scan2d.h declares, and rejects
bad arguments on the host before touching a device.  No compute calls (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "scan2d.h")


def _header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(scan2d_\w+)\s*\(", text)
    return sorted(set(names))


def _header_macros():
    text = open(HEADER).read()
    return {m.group(1): int(m.group(2), 0)
            for m in re.finditer(r"#define\s+(SCAN2D_\w+)\s+(-?(?:0x[0-9a-fA-F]+|\d+))u?", text)}


@pytest.fixture(scope="module")
def lib():
    from selective_state_space_scan2d_b200 import build
    build.build()
    from selective_state_space_scan2d_b200 import scan2d
    return scan2d


def test_every_declared_symbol_is_exported(lib):
    declared = _header_functions()
    assert {"scan2d_fwd", "scan2d_fwd_host", "scan2d_get_device_error", "scan2d_strerror",
            "scan2d_version", "scan2d_host_staging_bytes"} <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", lib.lib_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(scan2d_\w+)$", out, flags=re.M))
    missing = [n for n in declared if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    raw = ctypes.CDLL(lib.lib_path)
    for n in declared:
        assert getattr(raw, n) is not None


def test_binding_constants_match_header(lib):
    m = _header_macros()
    for name in ("SCAN2D_BF16", "SCAN2D_OUT_F32", "SCAN2D_OR_TL", "SCAN2D_OR_TR",
                 "SCAN2D_OR_BL", "SCAN2D_OR_BR"):
        assert getattr(lib, name) == m[name], name
    assert lib.SCAN2D_E_SCRATCH == m["SCAN2D_E_SCRATCH"]
    assert lib.SCAN2D_VFIRST == m["SCAN2D_VFIRST"]
    assert lib.SCAN2D_NOALLOC_SCRATCH_BYTES == m["SCAN2D_NOALLOC_SCRATCH_BYTES"]
    assert lib.flags_for(True, 0xF, out_f32=True) == (m["SCAN2D_BF16"] | m["SCAN2D_OUT_F32"] | m["SCAN2D_OR_ALL"])


def test_version_and_strerror(lib):
    assert lib.scan2d_version() >= 100
    m = _header_macros()
    codes = [v for k, v in m.items() if k.startswith("SCAN2D_E_")]
    texts = {lib.scan2d_strerror(c) for c in codes}
    assert len(texts) == len(codes), "every error code has its own text"
    assert lib.scan2d_strerror(12345) == "unknown error"


# fake, 256-byte aligned "device" addresses: the host checks reject the call before any use
P = 1 << 20


@pytest.mark.parametrize("args,code", [
    # (batch, channels, H, W, N, flags), expected error
    ((0, 4, 8, 8, 4, 0x10), "SCAN2D_E_DIMS"),
    ((1, 0, 8, 8, 4, 0x10), "SCAN2D_E_DIMS"),
    ((1, 4, 0, 8, 4, 0x10), "SCAN2D_E_DIMS"),
    ((1, 4, 8, -3, 4, 0x10), "SCAN2D_E_DIMS"),
    ((1, 4, 65536, 65536, 4, 0x10), "SCAN2D_E_DIMS"),
    ((1, 4, 8, 8, 0, 0x10), "SCAN2D_E_N"),
    ((1, 4, 8, 8, 65, 0x10), "SCAN2D_E_N"),
    ((1, 4, 8, 8, 4, 0x100), "SCAN2D_E_FLAGS"),
    ((1, 4, 8, 8, 4, 0x2), "SCAN2D_E_FLAGS"),        # OUT_F32 without BF16
    ((1, 4, 8, 8, 4, 0x4), "SCAN2D_E_FLAGS"),        # reserved bit
])
def test_host_rejects_bad_shapes(lib, args, code):
    m = _header_macros()
    rc = lib.raw().scan2d_fwd(P, P, P, P, P, None, P, *args, None)
    assert rc == m[code]


def test_host_rejects_null_and_misaligned(lib):
    m = _header_macros()
    r = lib.raw()
    dims = (1, 4, 8, 8, 4)
    for k in range(7):
        if k == 5:
            continue                                   # Dskip may be NULL
        ptrs = [P] * 7
        ptrs[k] = None
        assert r.scan2d_fwd(*ptrs, *dims, 0x10, None) == m["SCAN2D_E_NULL"]
    assert r.scan2d_fwd(P + 2, P, P, P, P, None, P, *dims, 0x10, None) == m["SCAN2D_E_ALIGN"]
    assert r.scan2d_fwd(P, P, P + 2, P, P, None, P, *dims, 0x10, None) == m["SCAN2D_E_ALIGN"]
    # bf16 buffers need 2-byte alignment only; fp32 y with OUT_F32 needs 4
    assert r.scan2d_fwd(P, P, P, P + 1, P, None, P, *dims, 0x11, None) == m["SCAN2D_E_ALIGN"]
    assert r.scan2d_fwd(P, P, P, P, P, None, P + 2, *dims, 0x13, None) == m["SCAN2D_E_ALIGN"]


def test_staging_size_and_host_checks(lib):
    m = _header_macros()
    n = lib.scan2d_host_staging_bytes(1, 4, 8, 8, 4, 0x10)
    # x, delta, y: 256 floats each; A 16 floats; B, C 256 floats; Dskip 4 -> rounded to 256 B
    assert n == 256 * 4 * 3 + 256 + 256 * 4 * 2 + 256
    assert lib.scan2d_host_staging_bytes(1, 4, 8, 8, 4, 0x1F1) == 0
    r = lib.raw()
    assert r.scan2d_fwd_host(P, P, P, P, P, None, P, P, n - 1, 1, 4, 8, 8, 4, 0x10, None) == m["SCAN2D_E_STAGING"]
    assert r.scan2d_fwd_host(P, P, P, P, P, None, P, P + 16, n, 1, 4, 8, 8, 4, 0x10, None) == m["SCAN2D_E_ALIGN"]


def test_bwd_workspace_size_and_host_checks(lib):
    m = _header_macros()
    assert lib.SCAN2D_E_WORKSPACE == m["SCAN2D_E_WORKSPACE"]
    assert lib.SCAN2D_BWD_MAX_N == m["SCAN2D_BWD_MAX_N"]
    # channels are padded to a group of 8; hsave: N floats per element of strips padded to 8
    # columns (8 channels * 64 * 4 states * 4 bytes); five strip-carry arrays of H * strips * N
    # floats per channel (8 * 1 * 4 * 8 channels * 4 bytes), each rounded up to 256 bytes
    n = lib.scan2d_bwd_workspace_bytes(1, 4, 8, 8, 4, 0x10)
    assert n == 8 * 64 * 4 * 4 + 5 * 8 * 4 * 8 * 4
    # bf16 y with several orientations adds two fp32 accumulators of the element count
    nb = lib.scan2d_bwd_workspace_bytes(1, 4, 8, 8, 4, 0x31)
    assert nb == n + 2 * 4 * 64 * 4
    assert lib.scan2d_bwd_workspace_bytes(1, 4, 8, 8, 17, 0x10) == 0
    r = lib.raw()
    dims = (1, 4, 8, 8, 4)
    call = lambda *ptrs, size=n, flags=0x10, d=dims: r.scan2d_bwd(*ptrs, size, *d, flags, None)
    good = [P] * 14
    good[5] = None                                     # Dskip may be NULL
    assert call(*good, flags=0x14) == m["SCAN2D_E_FLAGS"]          # a reserved bit
    assert call(*good, d=(1, 4, 8, 8, 17)) == m["SCAN2D_E_N"]
    assert call(*good, size=n - 1) == m["SCAN2D_E_WORKSPACE"]
    for k in (0, 6, 7, 13):
        bad = list(good)
        bad[k] = None
        assert call(*bad) == m["SCAN2D_E_NULL"], k
    bad = list(good)
    bad[13] = P + 16                                   # workspace must be 256-byte aligned
    assert call(*bad) == m["SCAN2D_E_ALIGN"]


def test_grid_host_checks(lib):
    m = _header_macros()
    r = lib.raw()
    assert r.scan2d_grid_cells(P, -1, 8, 8, P, None, None) == m["SCAN2D_E_DIMS"]
    assert r.scan2d_grid_cells(P, 4, 0, 8, P, None, None) == m["SCAN2D_E_DIMS"]
    assert r.scan2d_grid_cells(None, 4, 8, 8, P, None, None) == m["SCAN2D_E_NULL"]
    assert r.scan2d_grid_cells(P, 4, 8, 8, None, None, None) == m["SCAN2D_E_NULL"]
    assert r.scan2d_grid_cells(P, 4, 8, 8, P + 2, None, None) == m["SCAN2D_E_ALIGN"]
    assert r.scan2d_grid_gather(P, P, P, P, 4, 8, 8, 8, 0x10, None) == m["SCAN2D_E_FLAGS"]
    assert r.scan2d_grid_gather(P, P, P, P, 4, 0, 8, 8, 0, None) == m["SCAN2D_E_DIMS"]
    assert r.scan2d_grid_gather(P, P, None, P, 4, 8, 8, 8, 0, None) == m["SCAN2D_E_NULL"]
    assert r.scan2d_grid_gather(P + 2, P, P, P, 4, 8, 8, 8, 0, None) == m["SCAN2D_E_ALIGN"]
    # the fused forward checks the bag's arguments before the scan's
    args = (P, P, P, P, P, P, P, None, P)
    assert r.scan2d_fwd_wsi(*args, -1, 4, 8, 8, 4, 0x10, None) == m["SCAN2D_E_DIMS"]
    assert r.scan2d_fwd_wsi(P, None, P, P, P, P, P, None, P, 3, 4, 8, 8, 4, 0x10, None) == m["SCAN2D_E_NULL"]
    assert r.scan2d_fwd_wsi(*args, 3, 4, 8, 8, 4, 0x14, None) == m["SCAN2D_E_FLAGS"]


def test_proj_host_checks(lib):
    m = _header_macros()
    assert lib.SCAN2D_PROJ_MAX_R == m["SCAN2D_PROJ_MAX_R"]
    r = lib.raw()
    ptrs = [P] * 7
    assert r.scan2d_proj(*ptrs, 1, 8, 4, 4, 4, 2, 0x10, None) == m["SCAN2D_E_FLAGS"]
    assert r.scan2d_proj(*ptrs, 1, 8, 4, 4, 17, 2, 0, None) == m["SCAN2D_E_N"]
    assert r.scan2d_proj(*ptrs, 1, 8, 4, 4, 4, 33, 0, None) == m["SCAN2D_E_DIMS"]
    assert r.scan2d_proj(*ptrs, 0, 8, 4, 4, 4, 2, 0, None) == m["SCAN2D_E_DIMS"]
    for k in range(7):
        bad = list(ptrs)
        bad[k] = None
        assert r.scan2d_proj(*bad, 1, 8, 4, 4, 4, 2, 0, None) == m["SCAN2D_E_NULL"], k
    bad = list(ptrs)
    bad[1] = P + 2
    assert r.scan2d_proj(*bad, 1, 8, 4, 4, 4, 2, 0, None) == m["SCAN2D_E_ALIGN"]


def test_valid_call_without_a_gpu_fails_loudly(lib):
    """No CPU fallback: with valid arguments and no usable device the call is an error."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    m = _header_macros()
    r = lib.raw()
    assert r.scan2d_fwd(P, P, P, P, P, None, P, 1, 4, 8, 8, 4, 0x10, None) == m["SCAN2D_E_DEVICE"]
    n = lib.scan2d_bwd_workspace_bytes(1, 4, 8, 8, 4, 0x10)
    assert r.scan2d_bwd(P, P, P, P, P, None, P, P, P, P, P, P, None, P, n, 1, 4, 8, 8, 4, 0x10, None) == m["SCAN2D_E_DEVICE"]
    assert r.scan2d_fwd_wsi(P, P, P, P, P, P, P, None, P, 3, 4, 8, 8, 4, 0x10, None) == m["SCAN2D_E_DEVICE"]
    assert r.scan2d_grid_cells(P, 4, 8, 8, P, None, None) == m["SCAN2D_E_DEVICE"]
    assert r.scan2d_grid_gather(P, P, P, P, 4, 8, 8, 8, 0, None) == m["SCAN2D_E_DEVICE"]
    assert r.scan2d_proj(P, P, P, P, P, P, P, 1, 8, 4, 4, 4, 2, 0, None) == m["SCAN2D_E_DEVICE"]
    x = torch.zeros(1, 4, 8, 8)
    with pytest.raises(ValueError):
        lib.scan2d_fwd(x, x, torch.zeros(4, 4), torch.zeros(1, 4, 8, 8), torch.zeros(1, 4, 8, 8))
