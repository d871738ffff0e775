"""The allocation-free GEMM entry point (sq_w8a8_gemm_dequant_noalloc).

Some callers cannot allocate device memory at the moment they launch the
GEMM -- an inference-engine plugin whose enqueue path must not allocate, or a
serving loop whose memory a framework reserved up front.  This entry point
takes no workspace: its split-K partial sums live in a fixed array owned by the
library.  The tests check, through the C ABI, that two calls in a row give the
same output as the allocating entry point with a caller-provided workspace
and as the oracle, that an automatic plan too big for the array falls back to
whole tiles, and that a plan needing more scratch than the array holds (or an
output of the wrong shape) is refused.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_int8_quantized_norm_b200 import sq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sq.lib()


def _problem(rng, M, N, K):
    Xq = torch.from_numpy(rng.integers(-127, 128, (M, K)).astype(np.int8)).cuda()
    Wq = torch.from_numpy(rng.integers(-127, 128, (N, K)).astype(np.int8)).cuda()
    xs = torch.from_numpy((rng.random(M) * 0.05 + 1e-3).astype(np.float32)).cuda()
    ws = torch.from_numpy((rng.random(N) * 0.002 + 1e-5).astype(np.float32)).cuda()
    return Xq, Wq, xs, ws


@pytest.mark.parametrize("epi", ["bf16", "i32"])
def test_noalloc_matches_allocating_entry_point_twice(epi):
    rng = np.random.default_rng(99)
    M, N, K = 16, 1024, 8192  # decode tiles with split-K: the scratch is used
    assert 0 < sq.gemm_workspace_size(M, N, K, 0) <= sq.NOALLOC_SCRATCH_BYTES
    dt = torch.int32 if epi == "i32" else torch.bfloat16
    for _ in range(2):  # two calls in a row, different inputs each time
        Xq, Wq, xs, ws = _problem(rng, M, N, K)
        ref = sq.w8a8_gemm_dequant(Xq, Wq, xs, ws, epi)
        out = torch.full((M, N), 7, dtype=dt, device="cuda")
        sq.w8a8_gemm_dequant_noalloc(Xq, Wq, xs, ws, out, epi)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        _check_oracle(out, Xq, Wq, xs, ws, epi)
    assert sq.get_device_error() == 0


def _check_oracle(out, Xq, Wq, xs, ws, epi):
    """The output against the oracle: the exact integer sums, or the
    oracle's epilogue of them bit for bit."""
    acc = oracle.gemm_i64(Xq.cpu().numpy(), Wq.cpu().numpy())
    if epi == "i32":
        assert np.array_equal(out.cpu().numpy().astype(np.int64), acc)
    else:
        _, ref = oracle.epilogue(acc, xs.cpu().numpy(), ws.cpu().numpy())
        assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), ref)


def test_noalloc_automatic_plan_falls_back_to_whole_tiles():
    """With split_k = 0, a decode plan whose stream-K slots would not fit the
    library's array runs whole tiles (no scratch) and gives the same bits as
    the allocating entry point's whole-tile plan."""
    rng = np.random.default_rng(5)
    M, N, K = 128, 8192, 8192
    assert sq.gemm_workspace_size(M, N, K, 0) > sq.NOALLOC_SCRATCH_BYTES
    Xq, Wq, xs, ws = _problem(rng, M, N, K)
    ref = sq.w8a8_gemm_dequant(Xq, Wq, xs, ws, "bf16", split_k=1)
    out = torch.full((M, N), 3, dtype=torch.bfloat16, device="cuda")
    sq.w8a8_gemm_dequant_noalloc(Xq, Wq, xs, ws, out, "bf16")
    torch.cuda.synchronize()
    assert sq.get_device_error() == 0
    assert torch.equal(out, ref)
    _check_oracle(out, Xq, Wq, xs, ws, "bf16")


def test_noalloc_rejects_an_output_of_the_wrong_shape():
    rng = np.random.default_rng(6)
    Xq, Wq, xs, ws = _problem(rng, 4, 256, 128)
    for bad in (torch.empty((4, 255), dtype=torch.bfloat16, device="cuda"),
                torch.empty((4, 256), dtype=torch.int32, device="cuda"),
                torch.empty((256, 4), dtype=torch.bfloat16, device="cuda").t()):
        with pytest.raises(ValueError):
            sq.w8a8_gemm_dequant_noalloc(Xq, Wq, xs, ws, bad, "bf16")


def test_noalloc_refuses_plans_beyond_its_scratch():
    M, N, K = 128, 57344, 8192
    need = sq.gemm_workspace_size(M, N, K, 8)
    assert need > sq.NOALLOC_SCRATCH_BYTES
    Xq = torch.zeros((M, K), dtype=torch.int8, device="cuda")
    Wq = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    xs = torch.zeros(M, dtype=torch.float32, device="cuda")
    ws = torch.zeros(N, dtype=torch.float32, device="cuda")
    out = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sq.SQError) as e:
        sq.w8a8_gemm_dequant_noalloc(Xq, Wq, xs, ws, out, "bf16", path_hint=2, split_k=8)
    assert e.value.status == 7  # SQ_ERR_WORKSPACE, nothing launched
    assert torch.count_nonzero(out) == 0
