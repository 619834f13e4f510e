"""The small GPU parity cases are chosen to reach every code path of the library; this
checks that claim from the host-side plan (no GPU needed)."""
import pytest

from selective_state_space_scan2d_b200 import inputs


@pytest.fixture(scope="module")
def plans():
    from selective_state_space_scan2d_b200 import build
    build.build()
    from selective_state_space_scan2d_b200 import scan2d
    from scan2d_cases import CASES
    out = {}
    for case, (name, kw) in CASES.items():
        w = inputs.WORKLOADS[name].scaled(**kw) if kw else inputs.WORKLOADS[name]
        flags = scan2d.flags_for(w.dtype == "bf16", w.orient_mask)
        out[case] = scan2d.scan2d_query_plan(w.batch, w.channels, w.H, w.W, w.N, flags)
    return out


def test_every_path_is_exercised(plans):
    ps = list(plans.values())
    assert any(p["tma"] == 1 for p in ps) and any(p["tma"] == 0 for p in ps)
    assert any(p["nseg"] > 1 and p["tma"] == 1 for p in ps), "chained blocks, TMA staging"
    assert any(p["nseg"] > 1 and p["tma"] == 0 for p in ps), "chained blocks, plain staging"
    assert any(p["nseg"] > 1 and p["mode"] == 0 and p["tma"] == 1 for p in ps)
    assert any(p["mode"] == 1 for p in ps), "orientations summed in shared memory"
    assert any(p["mode"] == 2 for p in ps), "one launch per orientation"
    assert {p["ng"] for p in ps} >= {1, 2, 4, 8, 16}, "every states-per-lane variant"
    assert {p["g"] for p in ps} == {1, 2}, "one and two channels per lane"
    assert any(p["wpc"] > 1 and p["nseg"] == 1 for p in ps), "several strips in one block"
    assert any(p["tma"] == 1 and p["mode"] == 0 and p["g"] == 2 for p in ps)
    assert any(p["link"] == 1 and p["tma"] == 1 for p in ps), "cluster-linked chain, TMA"
    assert any(p["link"] == 1 and p["tma"] == 0 for p in ps), "cluster-linked chain, plain"
    assert any(p["link"] == 2 and p["tma"] == 1 for p in ps), "global-ring chain, TMA"
    assert any(p["link"] == 2 and p["tma"] == 0 for p in ps), "global-ring chain, plain"
    assert any(p["link"] == 1 and p["nseg"] == 16 for p in ps), "the largest cluster"
    split = [p for p in ps if p["mode"] == 1 and p["threads"] > 256]
    assert any(p["tma"] == 1 for p in split) and any(p["tma"] == 0 for p in split), \
        "two chain slots splitting the orientations, TMA and plain staging"


def test_long_chain_hits_ring_back_pressure(plans):
    # 40 rows > the 16-row carry ring, 9+ segments: producers must wait for consumers
    # 37-40 rows > the 16-row global ring and the 4-row shared-memory ring
    for case in ("f32_long_chain_backpressure", "f32_global_ring_tma"):
        assert plans[case]["link"] == 2 and plans[case]["nseg"] > 16
    assert plans["f32_global_ring_tma"]["tma"] == 1
    assert plans["f32_long_chain_backpressure_tma"]["link"] == 1
