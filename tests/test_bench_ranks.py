"""Host logic of the multi-GPU bench path, run as two gloo ranks on the CPU:
every rank gets its own inputs, the timed duration is the max over ranks, and
the reported value counts every rank's tokens over that duration. The oracle
(reference) arm runs on rank 0 only."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    rk = bench.Ranks()
    local_ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
    ms = rk.max_over_ranks(local_ms)
    res = {"rank": rk.rank, "world": rk.world, "seed": rk.seed(0), "ms": ms,
           "value": rk.value(bench.TOKENS_PER_STEP, 4, ms)}
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks_take_the_max_and_count_every_rank(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(2)]
    import bench
    for x in r:
        assert x["world"] == 2
        assert x["ms"] == 15.0                       # the slower rank's time on both ranks
        assert x["value"] == pytest.approx(bench.TOKENS_PER_STEP * 2 * 4 / 15e-3)
    assert r[0]["seed"] != r[1]["seed"]              # independent shards get distinct inputs


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup, gpus, seed = 1, 1, 2, 0
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""             # rank 1 prints nothing and does no work


def test_single_rank_defaults():
    import bench
    rk = bench.Ranks(env={})
    assert (rk.world, rk.rank, rk.local) == (1, 0, 0)
    assert rk.max_over_ranks(3.5) == 3.5
    assert rk.value(100, 10, 1000.0) == pytest.approx(1000.0)
