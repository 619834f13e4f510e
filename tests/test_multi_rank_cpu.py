"""The multi-GPU logic of bench.py on CPU: world-size-2 gloo ranks (replicas, weak scaling).

Every (b, d) map is independent, so ranks share no data; the only cross-rank step is the
max of the per-rank device times, and the whole-job rate is N x elements / that time."""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms, e2e = bench.max_over_ranks(times[rank])
        value = bench.whole_job_gelem(1000, world, ms)
        torch.distributed.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{ms} {e2e} {value}\n")
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_rate(tmp_path):
    import torch.multiprocessing as mp
    times = [(2.0, 9.0), (3.0, 4.0)]          # per-rank (device ms, e2e ms)
    mp.start_processes(_rank_main, args=(2, _free_port(), times, str(tmp_path)), nprocs=2,
                       start_method="spawn", join=True)
    for rank in range(2):
        ms, e2e, value = map(float, (tmp_path / f"rank{rank}.txt").read_text().split())
        assert ms == 3.0 and e2e == 9.0           # every rank sees the slowest rank's times
        assert value == pytest.approx(2 * 1000 / 3e-3 / 1e9)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.whole_job_gelem(10**9, 1, 1000.0) == pytest.approx(1.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    from selective_state_space_scan2d_b200 import inputs
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup, gpus = 3, 3, 2
    bench.run_reference(Args, inputs.WORKLOADS["tiny"])      # returns without work or output
    assert capsys.readouterr().out == ""
