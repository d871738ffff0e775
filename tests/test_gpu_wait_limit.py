"""Failure detection in the GEMM pipeline without a GPU fault.

A poll limit of one makes the tensor-core pipeline's first unfinished wait give
up: the kernel records SQ_ERR_PIPELINE_TIMEOUT in the device error word, lets
every copy and MMA it issued finish, frees its tensor memory and returns.  The
host reads the status; the context stays usable, which the next (normal) call
on the same shapes shows by producing the exact result."""
import numpy as np
import pytest
import torch

import oracle
from w8a8_int8_quantized_norm_b200 import sq

from _parity import to_gpu

pytestmark = pytest.mark.gpu

TIMEOUT = 6  # SQ_ERR_PIPELINE_TIMEOUT


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sq.lib()
    assert sq.get_device_error() == 0
    yield
    sq.set_wait_limit(0)
    assert sq.get_device_error() == 0


# (M, N, K, path hint, split-K): CTA-pair prefill tiles, single-SM prefill
# tiles, decode tiles on the automatic stream-K plan (partial sums in the
# workspace, then the fix-up kernel launched as a programmatic dependent), and
# decode tiles with an explicit split into four K slices plus the reduction
# kernel.  K is long enough that an accumulator is never ready at the
# epilogue's first probe.
CASES = [(512, 1024, 16384, 1, 0), (512, 1024, 16384, 3, 0), (16, 2048, 16384, 2, 0),
         (16, 2048, 16384, 2, 4)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%dx%dx%d-path%d-split%d" % c)
def test_wait_limit_reports_timeout_then_recovers(case):
    M, N, K, path, split = case
    rng = np.random.default_rng(7 + path)
    A = rng.integers(-127, 128, (M, K)).astype(np.int8)
    B = rng.integers(-127, 128, (N, K)).astype(np.int8)
    a, b = to_gpu(A), to_gpu(B)
    out = torch.zeros((M, N), dtype=torch.int32, device=a.device)
    try:
        sq.set_wait_limit(1)
        sq.w8a8_gemm_dequant(a, b, None, None, "i32", out=out, path_hint=path, split_k=split)
        status = sq.get_device_error()
    finally:
        sq.set_wait_limit(0)
    assert status == TIMEOUT, sq.status_string(status)
    # the error word was read and cleared; a normal call is exact again
    assert sq.get_device_error() == 0
    sq.w8a8_gemm_dequant(a, b, None, None, "i32", out=out, path_hint=path, split_k=split)
    assert sq.get_device_error() == 0
    assert np.array_equal(out.cpu().numpy().astype(np.int64), oracle.gemm_i64(A, B))
