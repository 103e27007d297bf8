"""The N > 1 path of bench.py on CPU: two gloo ranks reduce their device times
with a max and report whole-job throughput as all ranks' work over the
slowest rank's time.  No attention data crosses ranks (each rank owns an
independent problem), so the only collectives are these timing reductions."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    import bench
    assert bench.dist_env() == (rank, world, rank)
    my_ms = [12.0, 15.5][rank]
    bench.barrier()
    mx = bench.reduce_max(my_ms)
    value = bench.aggregate_value(bench.step_flops(bench.WORKLOAD), world, mx)
    out[rank] = (mx, value)
    dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    import bench
    expect = bench.step_flops(bench.WORKLOAD) * 2 / (15.5e-3) / 1e12
    for r in range(world):
        mx, value = out[r]
        assert mx == 15.5
        assert value == pytest.approx(expect, rel=1e-12)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def test_work_accounting_matches_the_stated_convention():
    import bench
    w = dict(bench.WORKLOAD)
    assert bench.fwd_flops(w) == pytest.approx(549.755813888e9)
    assert bench.bwd_flops(w) == pytest.approx(1374.38953472e9)
    assert bench.visible_keys(0, w) == 1 and bench.visible_keys(8191, w) == 8192
