"""A SmoothQuant W8A8 block run through the C ABI: offline preparation
(calibration, smoothing factors, fold, weight quantisation) and the runtime
forward (norm + per-token quant, INT8 GEMM + dequant epilogue).

Which Linears are smoothed follows "SmoothQuant, in depth" -- "Where the scales
go in a decoder block": projections fed by a norm share one s folded into that
norm; o_proj / down_proj style inputs (no norm in front) are not smoothed but
still quantised per token.  A Linear with no norm in front that *is* smoothed
gets its 1/s as a per-channel multiplier (the fold with gamma = 1).

Every arithmetic step runs in libsq.so; this module only sequences the calls
and owns the device buffers (allocated once, reused by every forward).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

from . import sq
from .synthetic import Workload


@dataclasses.dataclass
class SiteState:
    norm: int
    K: int
    act_max: Optional[torch.Tensor] = None
    s: Optional[torch.Tensor] = None
    gamma_folded: Optional[torch.Tensor] = None
    beta_folded: Optional[torch.Tensor] = None


@dataclasses.dataclass
class LinearState:
    Wq: torch.Tensor
    w_scale: torch.Tensor


@dataclasses.dataclass
class Prepared:
    workload: Workload
    sites: Dict[str, SiteState]
    linears: Dict[str, LinearState]


def prepare(w: Workload, x_cal: Dict[str, torch.Tensor], W: Dict[str, torch.Tensor],
            gamma: Dict[str, Optional[torch.Tensor]], beta: Dict[str, Optional[torch.Tensor]],
            stream=None) -> Prepared:
    """Offline steps: calibrate every smoothed site, compute its s from the
    weights of all Linears reading it, fold 1/s, smooth and quantise every
    weight (unsmoothed Linears with s = 1)."""
    sites: Dict[str, SiteState] = {}
    for site in w.sites:
        st = SiteState(norm=site.norm, K=site.K)
        if site.smoothed:
            g, b = gamma.get(site.name), beta.get(site.name)
            st.act_max = sq.calibrate_absmax(x_cal[site.name], site.norm, g, b, w.eps,
                                             stream=stream)
            ws = [W[l.name] for l in w.linears_of(site.name)]
            st.s, st.gamma_folded, st.beta_folded = sq.compute_smooth_scales(
                st.act_max, ws, w.alpha, w.clamp_eps, g, b, stream=stream)
        else:
            st.gamma_folded, st.beta_folded = gamma.get(site.name), beta.get(site.name)
        sites[site.name] = st
    linears: Dict[str, LinearState] = {}
    for lin in w.linears:
        Wq, wsc = sq.smooth_quantize_weights(W[lin.name], sites[lin.site].s, stream=stream)
        linears[lin.name] = LinearState(Wq, wsc)
    return Prepared(w, sites, linears)


class Forward:
    """Runtime path with preallocated buffers for M tokens."""

    def __init__(self, prep: Prepared, M: int, device, epi_raw: bool = False):
        self.prep = prep
        self.M = M
        w = prep.workload
        self.xq: Dict[str, torch.Tensor] = {}
        self.xs: Dict[str, torch.Tensor] = {}
        self.out: Dict[str, torch.Tensor] = {}
        self.ws: Dict[str, Optional[torch.Tensor]] = {}
        for site in w.sites:
            self.xq[site.name] = torch.empty((M, site.K), dtype=torch.int8, device=device)
            self.xs[site.name] = torch.empty(M, dtype=torch.float32, device=device)
        for lin in w.linears:
            self.out[lin.name] = torch.empty((M, lin.N), dtype=torch.bfloat16, device=device)
            K = w.site(lin.site).K
            need = sq.gemm_workspace_size(M, lin.N, K, 0)
            self.ws[lin.name] = (torch.empty(need, dtype=torch.uint8, device=device)
                                 if need else None)

    def __call__(self, x: Dict[str, torch.Tensor], stream=None) -> Dict[str, torch.Tensor]:
        w = self.prep.workload
        for site in w.sites:
            src = next((l.source for l in w.linears if l.site == site.name and l.source), None)
            xin = self.out[src] if src else x[site.name]
            st = self.prep.sites[site.name]
            sq.norm_smooth_quant_per_token(xin, st.norm, st.gamma_folded, st.beta_folded, w.eps,
                                           self.xq[site.name], self.xs[site.name], stream=stream)
            for lin in w.linears_of(site.name):
                L = self.prep.linears[lin.name]
                sq.w8a8_gemm_dequant(self.xq[site.name], L.Wq, self.xs[site.name], L.w_scale,
                                     "bf16_relu" if lin.relu else "bf16", out=self.out[lin.name],
                                     workspace=self.ws[lin.name], stream=stream)
        return self.out

    def kernel_launches(self) -> int:
        """Kernels one forward launches (norm-quant per site, GEMM per Linear,
        plus the split-K reduction where the plan splits K)."""
        w = self.prep.workload
        n = len(w.sites)
        for lin in w.linears:
            n += 2 if self.ws[lin.name] is not None else 1
        return n
