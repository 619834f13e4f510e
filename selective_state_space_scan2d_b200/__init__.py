"""B200-native 2D selective-scan forward (2DMamba) behind a small C-ABI library.

``selective_state_space_scan2d_b200.scan2d`` is the binding to the CUDA library; it is
imported on first use of one of its names so that the numpy-only input generator
(``selective_state_space_scan2d_b200.inputs``) can be imported without the library.
"""
_BINDING_NAMES = {
    "scan2d_fwd", "scan2d_fwd_host", "scan2d_get_device_error", "scan2d_strerror",
    "scan2d_version", "scan2d_host_staging_bytes", "scan2d_query_plan", "lib_path", "Scan2dError", "flags_for", "raw",
    "SCAN2D_BF16", "SCAN2D_OUT_F32", "SCAN2D_OR_TL", "SCAN2D_OR_TR", "SCAN2D_OR_BL",
    "SCAN2D_OR_BR", "scan2d_fwd_noalloc", "SCAN2D_E_SCRATCH", "SCAN2D_NOALLOC_SCRATCH_BYTES",
    "SCAN2D_VFIRST", "scan2d_bwd", "scan2d_bwd_workspace_bytes", "SCAN2D_E_WORKSPACE",
    "SCAN2D_BWD_MAX_N", "scan2d_grid_cells", "scan2d_grid_gather", "scan2d_fwd_wsi",
    "scan2d_proj", "SCAN2D_PROJ_MAX_R",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import scan2d
        return getattr(scan2d, name)
    raise AttributeError(name)
