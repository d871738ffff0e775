"""Helpers of the GPU-vs-oracle parity tests.

Exactness contract (the library's documented arithmetic):
* INT8 codes, INT32 accumulators, every fp32 scale and the folded norm
  parameters are bit-identical to the oracle's;
* bf16 outputs are within 1 bf16 ulp of the oracle's fp32 value (they are
  expected to be identical).
Two inputs of that arithmetic are reductions the GPU orders differently from
the oracle: the norm's row sums (fp64, tree order; the oracle sums exactly)
and fp64 ``pow`` (CUDA's vs glibc's, both within a few ulps).  A row or
channel may therefore differ only where the oracle certifies a near-tie: a
perturbation of the fp64 input within the stated error bound changes the fp32
result.  Such cases are counted, checked with a 1-code / 1-ulp tolerance and
expected to be absent.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

U64 = 2.0 ** -53


def to_gpu(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _stats32(S1, S2, K, kind, eps):
    ms = S2 / K
    if kind == oracle.NORM_RMS:
        v = ms + eps
        mu = 0.0
    else:
        mu64 = S1 / K
        var = max(0.0, ms - mu64 * mu64)
        v = var + eps
        mu = mu64
    return np.float32(mu), np.float32(1.0 / np.sqrt(v))


def norm_near_tie_rows(x: np.ndarray, kind: int, eps: float) -> np.ndarray:
    """Rows whose fp32 (mu, r) could change under any fp64 summation order:
    the sums move by at most (K-1) u sum|terms| (a bound valid for every
    order)."""
    if kind == oracle.NORM_NONE:
        return np.zeros(x.shape[0], bool)
    S1, S2, SA = oracle.row_sums(x)
    K = x.shape[1]
    e = float(np.float32(eps))
    flags = np.zeros(x.shape[0], bool)
    for m in range(x.shape[0]):
        b1 = (K + 2) * U64 * SA[m]
        b2 = (K + 2) * U64 * S2[m]
        ref = _stats32(S1[m], S2[m], K, kind, e)
        for d1 in (-b1, b1):
            for d2 in (-b2, b2):
                if _stats32(S1[m] + d1, max(S2[m] + d2, 0.0), K, kind, e) != ref:
                    flags[m] = True
    return flags


def scale_near_tie_channels(s64: np.ndarray, ulps: float = 4.0) -> np.ndarray:
    """Channels whose fp32 smoothing factor could change if the fp64 value
    moved by `ulps` fp64 ulps (CUDA's and glibc's pow may differ that much)."""
    lo = (s64 * (1 - ulps * U64)).astype(np.float32)
    hi = (s64 * (1 + ulps * U64)).astype(np.float32)
    return lo != hi


def compare_rows_quant(Xq_g, xs_g, Xq_o, xs_o, tie_rows):
    """Bit-exact comparison of per-row INT8 codes and scales; rows flagged as
    near-ties may differ by one code / a few ulps.  Returns the number of
    tolerated rows."""
    bad_rows = np.nonzero((Xq_g != Xq_o).any(axis=1) | (xs_g.view(np.uint32) != xs_o.view(np.uint32)))[0]
    unexplained = [int(m) for m in bad_rows if not tie_rows[m]]
    assert not unexplained, "rows differ from the oracle without a near-tie: %s" % unexplained[:10]
    for m in bad_rows:
        assert np.abs(Xq_g[m].astype(np.int32) - Xq_o[m]).max() <= 1
        assert abs(float(xs_g[m]) - float(xs_o[m])) <= 4 * np.spacing(np.float32(xs_o[m]))
    return len(bad_rows)


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two bf16 bit arrays (same-sign values)."""
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7fff), b & 0x7fff)
    return np.abs(key(a_bits) - key(b_bits))
