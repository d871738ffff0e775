"""The N > 1 benchmark path on CPU: two ``gloo`` ranks in spawned processes.

The hot path shards as independent replicas (each rank runs the whole block on
its own token batch, weights replicated); the only cross-rank steps are the
timing reductions.  These tests check that the replicas' inputs are shared
where they must be and distinct where they must be, that the whole-job
throughput takes the slowest rank's time, and that token shards run through
the whole block on separate ranks gather to the unsharded block's outputs."""
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


def _tiny_blocks():
    """Small blocks with every kind of site: a LayerNorm MLP (fc1 -> ReLU ->
    requant -> fc2) and an RMSNorm block with the SiLU(gate) * up site."""
    from w8a8_int8_quantized_norm_b200 import synthetic as S
    blocks = [
        S.Workload(name="dp-shard-mlp-layernorm-24x96x160", M=24, M_cal=32, dtype="bf16",
                   alpha=0.5,
                   sites=(S.Site("ffn_norm", 96, S.NORM_LAYER, True),
                          S.Site("fc1_act", 160, S.NORM_NONE, False, calibrated=False)),
                   linears=(S.Linear("fc1", "ffn_norm", 160, relu=True),
                            S.Linear("fc2", "fc1_act", 96, source="fc1")),
                   outliers=S.OutlierLaw(count=3, factor=60.0)),
        S.Workload(name="dp-shard-rms-silu-21x64x96", M=21, M_cal=32, dtype="bf16", alpha=0.8,
                   sites=(S.Site("mlp_norm", 64, S.NORM_RMS, True),
                          S.Site("mlp_act", 48, S.NORM_NONE, False, calibrated=False,
                                 act="silu_mul")),
                   linears=(S.Linear("gate_up", "mlp_norm", 96),
                            S.Linear("down", "mlp_act", 64, source="gate_up")),
                   outliers=S.OutlierLaw(count=2, factor=50.0)),
    ]
    for w in blocks:
        S.WORKLOADS.setdefault(w.name, w)
    return [S.WORKLOADS[w.name] for w in blocks]


def _shard_rows(M, world, rank):
    """Rank r's contiguous share of M token rows (the first M % world ranks
    take one more)."""
    base, extra = divmod(M, world)
    lo = rank * base + min(rank, extra)
    return np.arange(lo, lo + base + (1 if rank < extra else 0))


def _shard_worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist

    import _oracle_pipeline as OP
    import oracle
    from w8a8_int8_quantized_norm_b200 import synthetic as S

    oracle.build()
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        result = {}
        for w in _tiny_blocks():
            inp = S.make_inputs(w, seed=11)
            prep = OP.prepare(w, inp)  # every rank: the replicated offline rows
            res = OP.forward_rows(w, prep, inp, _shard_rows(w.M, world, rank))
            mine = {l.name: res["linears"][l.name]["out"] for l in w.linears}
            mine.update({s.name + ".xs": res["sites"][s.name]["xs"] for s in w.sites})
            gathered = [None] * world
            dist.all_gather_object(gathered, mine)
            result[w.name] = gathered
        with open(os.path.join(outdir, "shard%d.pkl" % rank), "wb") as f:
            import pickle
            pickle.dump(result, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3])
def test_token_shards_gather_to_the_unsharded_block(tmp_path, world):
    """Each rank runs its share of the tokens through the whole block (norm +
    per-token quantisation, INT8 GEMM, epilogue, the ReLU requant and the
    SiLU(gate) * up sites) with the replicated weights and smoothing factors;
    the outputs gathered in rank order equal one process's run over all
    tokens, bit for bit: every step after the offline rows is row-local."""
    import pickle

    import torch.multiprocessing as mp
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import _oracle_pipeline as OP
    import oracle
    from w8a8_int8_quantized_norm_b200 import synthetic as S

    mp.start_processes(_shard_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    outs = []
    for r in range(world):
        with open(tmp_path / ("shard%d.pkl" % r), "rb") as f:
            outs.append(pickle.load(f))
    oracle.build()
    for w in _tiny_blocks():
        inp = S.make_inputs(w, seed=11)
        whole = OP.forward_rows(w, OP.prepare(w, inp), inp, np.arange(w.M))
        for r in range(world):  # every rank gathered the same table
            assert all(a.keys() == b.keys() and all(np.array_equal(a[k], b[k]) for k in a)
                       for a, b in zip(outs[r][w.name], outs[0][w.name]))
        gathered = outs[0][w.name]
        assert sum(g[w.linears[0].name].shape[0] for g in gathered) == w.M
        for lin in w.linears:
            got = np.concatenate([g[lin.name] for g in gathered])
            assert np.array_equal(got, whole["linears"][lin.name]["out"]), lin.name
        for site in w.sites:
            got = np.concatenate([g[site.name + ".xs"] for g in gathered])
            assert np.array_equal(got.view(np.uint32),
                                  whole["sites"][site.name]["xs"].view(np.uint32)), site.name
