"""LLM.int8()'s mixed-precision decomposition as a comparator of the
smoothed W8A8 layer ("LLM.int8() and SmoothQuant" -- "Fix 1: give the
outliers their own lane (LLM.int8())", "going deeper -- LLM.int8()
decomposition").

The channels whose max |x| over the batch reaches tau (6 in the paper) are
multiplied in 16-bit; the others go through the same per-token INT8 codes,
INT8 GEMM and per-output-channel weight scales as the W8A8 layer; the two
results are added.  Every step runs in libsq.so; this module sequences the
five calls and owns their buffers.
"""
from __future__ import annotations

import torch

from . import sq


class LLMInt8Linear:
    """One Linear, W [N, K] (bf16 or fp32) on the device.  ``prepare``
    quantises W once per output channel; ``forward`` runs the decomposition on
    a batch x [M, K]."""

    def __init__(self, W: torch.Tensor, tau: float = 6.0):
        self.W = W
        self.tau = float(tau)
        N, K = W.shape
        dev = W.device
        self.Wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        self.w_scale = torch.empty(N, dtype=torch.float32, device=dev)
        self.col = torch.empty(K, dtype=torch.float32, device=dev)
        self.mask = torch.empty(K, dtype=torch.float32, device=dev)
        self.idx = torch.empty(K, dtype=torch.int32, device=dev)
        self.count = torch.zeros(1, dtype=torch.int32, device=dev)

    def prepare(self, stream=None) -> "LLMInt8Linear":
        sq.smooth_quantize_weights(self.W, None, Wq=self.Wq, w_scale=self.w_scale, stream=stream)
        return self

    def launches(self, M: int) -> int:
        """Kernels of this library one forward on M tokens launches: column
        max, outlier list, codes, the GEMM's plan, the merge (the column max's
        zeroing is a memset)."""
        return 4 + sq.gemm_plan(M, self.W.shape[0], self.W.shape[1], 0, 0).launches

    def forward(self, x: torch.Tensor, epi: str = "bf16", out=None, stream=None):
        """Returns the bf16 output [M, N]; the stages stay in ``self.stages``."""
        # max_t |x[t, j]|: the column-max pass of the weights, run on x (it
        # spreads any number of rows over the SMs with few atomics)
        sq.weight_column_max([x], w_max=self.col, stream=stream)
        sq.llmint8_outliers(self.col, self.tau, self.mask, self.idx, self.count, stream=stream)
        Xq, xs = sq.norm_smooth_quant_per_token(x, sq.NORM_NONE, self.mask, None, 0.0,
                                                stream=stream)
        acc = sq.w8a8_gemm_dequant(Xq, self.Wq, None, None, "i32", stream=stream)
        out = sq.llmint8_combine(acc, xs, self.w_scale, x, self.W, self.idx, self.count, epi,
                                 out=out, stream=stream)
        self.stages = {"Xq": Xq, "x_scale": xs, "acc": acc}
        return out
