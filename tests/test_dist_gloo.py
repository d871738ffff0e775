"""The N > 1 benchmark path on CPU: two ``gloo`` ranks in spawned processes.

The hot path shards as independent replicas (each rank runs the whole block on
its own token batch, weights replicated); the only cross-rank steps are the
timing reductions.  These tests check that the replicas' inputs are shared
where they must be and distinct where they must be, and that the whole-job
throughput takes the slowest rank's time."""
import hashlib
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _digest(d) -> str:
    h = hashlib.sha256()
    for k in sorted(d):
        if d[k] is not None:
            h.update(k.encode())
            h.update(np.ascontiguousarray(d[k]).tobytes())
    return h.hexdigest()


def _worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist

    import bench
    from w8a8_int8_quantized_norm_b200 import synthetic as S

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (world, rank, rank)
        inp = bench.rank_inputs(S.SMALL, seed=3, rank=rank)
        digests = [_digest(inp.W), _digest(inp.x_cal), _digest(inp.gamma), _digest(inp.beta),
                   _digest(inp.x)]
        gathered = [None] * world
        dist.all_gather_object(gathered, digests)
        # rank r takes r + 1 seconds for 10 units
        t_max = bench.max_over_ranks(float(rank + 1), world)
        value, t = bench.aggregate(10.0, float(rank + 1), world)
        with open(os.path.join(outdir, "rank%d.txt" % rank), "w") as f:
            f.write(repr((gathered, t_max, value, t)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(world, tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    out = []
    for r in range(world):
        with open(tmp_path / ("rank%d.txt" % r)) as f:
            out.append(eval(f.read()))
    return out


@pytest.mark.timeout(300)
def test_two_rank_replicas_and_timing(tmp_path):
    world = 2
    out = _run(world, tmp_path)
    for gathered, t_max, value, t in out:
        # every rank sees the same gathered table
        assert gathered == out[0][0]
        # weights, calibration tokens and norm parameters are replicated ...
        for field in range(4):
            assert gathered[0][field] == gathered[1][field]
        # ... the runtime token batches are the ranks' own
        assert gathered[0][4] != gathered[1][4]
        # the slowest rank's time, and the whole job's units over it
        assert t_max == 2.0 and t == 2.0
        assert value == pytest.approx(10.0 * world / 2.0)


def test_rank0_tokens_match_single_gpu_run():
    sys.path.insert(0, ROOT)
    import bench
    from w8a8_int8_quantized_norm_b200 import synthetic as S
    a = bench.rank_inputs(S.SMALL, seed=5, rank=0)
    b = S.make_inputs(S.SMALL, seed=5)
    assert _digest(a.x) == _digest(b.x) and _digest(a.W) == _digest(b.W)


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    called = []
    monkeypatch.setattr(bench, "run_reference", lambda *a: called.append(a))
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]) == 0
    assert called == [] and capsys.readouterr().out == ""
