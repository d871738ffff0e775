"""The row split of a W8A8 Linear over ranks (ksplit), on CPU: two ``gloo``
ranks in spawned processes, each holding half of the input channels.

The split's steps run on the oracle here (an op set given to ksplit, so the
module's sequence of steps and collectives is what runs); the all-reduces are
real gloo collectives.  Every rank must end with the unsplit layer's codes,
scales and output bit for bit: the oracle's linear over all K, with its
per-output-channel weights."""
import os
import pickle
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The split's steps on the oracle, on torch CPU tensors."""

    @staticmethod
    def row_absmax(x):
        import torch
        return torch.from_numpy(np.abs(x.numpy()).max(axis=1).astype(np.float32))

    @staticmethod
    def quant_given(x, row_absmax):
        import torch
        import oracle
        xv, am = x.numpy(), row_absmax.numpy()
        steps = np.array([oracle.step_of(a) for a in am], np.float32)
        q = np.concatenate([oracle.quantize_with_step(xv[m:m + 1], steps[m])
                            for m in range(xv.shape[0])])
        return torch.from_numpy(q), torch.from_numpy(steps)

    @staticmethod
    def gemm_i32(Xq, Wq):
        import torch
        import oracle
        return torch.from_numpy(oracle.gemm_i64(Xq.numpy(), Wq.numpy()))

    @staticmethod
    def dequant(acc, x_scale, w_scale, epi="bf16"):
        import torch
        import oracle
        _, out = oracle.epilogue(acc.numpy(), x_scale.numpy(), w_scale.numpy(),
                                 epi == "bf16_relu")
        return torch.from_numpy(out.view(np.int16))


def _inputs(M=7, N=40, K=96, seed=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, [5, 77]] *= np.float32(40.0)  # outliers in both halves
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    return x, W


def _worker(rank, world, port, outdir, relu):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch
    import torch.distributed as dist

    from test_ksplit_gloo import OracleOps, _inputs
    from w8a8_int8_quantized_norm_b200 import ksplit

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        x, W = _inputs()
        K = x.shape[1]
        cuts = [0, 48, K] if world == 2 else [0, 32, 48, K]  # uneven slices
        sl = slice(cuts[rank], cuts[rank + 1])
        xs = torch.from_numpy(np.ascontiguousarray(x[:, sl]))
        Ws = torch.from_numpy(np.ascontiguousarray(W[:, sl]))
        rmax, rsum = ksplit.torch_reducers()
        Wq, ws = ksplit.quantize_weight_shard(Ws, reduce_max=rmax, ops=OracleOps)
        out = ksplit.linear_shard(xs, Wq, ws, "bf16_relu" if relu else "bf16",
                                  reduce_max=rmax, reduce_sum=rsum, ops=OracleOps)
        # the step of each token as this rank saw it
        am = ksplit.shard_row_max(xs, OracleOps)
        rmax(am)
        _, xsc = OracleOps.quant_given(xs, am)
        with open(os.path.join(outdir, "rank%d.pkl" % rank), "wb") as f:
            pickle.dump({"Wq": Wq.numpy(), "ws": ws.numpy(), "out": out.numpy(),
                         "x_scale": xsc.numpy(), "slice": (sl.start, sl.stop)}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,relu", [(2, False), (3, True)])
def test_row_split_equals_the_unsplit_layer(tmp_path, world, relu):
    import torch.multiprocessing as mp

    import oracle
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), relu), nprocs=world,
                       join=True, start_method="spawn")
    x, W = _inputs()
    Wq_o, ws_o = oracle.quantize_weights(W, None)
    Xq_o, xs_o, acc_o, _, out_o = oracle.linear(x, oracle.NORM_NONE, None, None, 1e-5,
                                                Wq_o, ws_o, relu)
    for r in range(world):
        with open(tmp_path / ("rank%d.pkl" % r), "rb") as f:
            got = pickle.load(f)
        a, b = got["slice"]
        assert np.array_equal(got["ws"].view(np.uint32), ws_o.view(np.uint32))
        assert np.array_equal(got["Wq"], Wq_o[:, a:b])
        assert np.array_equal(got["x_scale"].view(np.uint32), xs_o.view(np.uint32))
        assert np.array_equal(got["out"].view(np.uint16), out_o)
