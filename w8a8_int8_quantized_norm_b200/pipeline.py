"""A SmoothQuant W8A8 block run through the C ABI: offline preparation
(calibration, smoothing factors, fold, weight quantisation) and the runtime
forward (norm + per-token quant, INT8 GEMM + dequant epilogue).

Which Linears are smoothed follows "SmoothQuant, in depth" -- "Where the scales
go in a decoder block": projections fed by a norm share one s folded into that
norm; o_proj / down_proj style inputs (no norm in front) are not smoothed but
still quantised per token.  A Linear with no norm in front that *is* smoothed
gets its 1/s as a per-channel multiplier (the fold with gamma = 1).

Every arithmetic step runs in libsq.so; this module only sequences the calls
and owns the device buffers (allocated once, reused by every call).
"""
from __future__ import annotations

from typing import Callable, Dict, Optional

import torch

from . import sq
from .synthetic import Workload

# timer(kind, algorithmic_units, fn): a caller hook around every library call;
# kind names the kernel family ("gemm:<linear>" for a GEMM call), units are its
# algorithmic bytes (row kernels) or integer ops (the GEMM).
Timer = Optional[Callable[[str, float, Callable[[], None]], None]]


def _run(timer: Timer, kind: str, units: float, fn: Callable[[], None]) -> None:
    if timer is None:
        fn()
    else:
        timer(kind, units, fn)


GRANULARITIES = ("per_token", "per_tensor_dynamic", "per_tensor_static")
FORMATS = ("int8", "fp8")


class Block:
    """Device state of one workload for M tokens per forward.

    ``prepare`` runs the offline rows (calibration, smoothing factors + fold,
    weight smoothing + quantisation); ``forward`` the runtime rows (fused norm
    + per-token quantisation, INT8 GEMM with the dequant epilogue).  An optional
    ``timer`` hook brackets every library call (the benchmark records CUDA
    events there).

    ``granularity`` (see "SmoothQuant, in depth" -- "Granularity: O1, O2, O3"):
    ``per_token`` is the serving-stack scheme (per-token dynamic activation
    scales, per-output-channel weight scales); ``per_tensor_dynamic`` (O2) and
    ``per_tensor_static`` (O3) use one weight scale per matrix and one
    activation scale per tensor -- the tensor's own max |y| (O2), or the max
    over the calibration tokens through the folded norm, fixed in ``prepare``
    (O3; a site without calibration tokens, i.e. an unsmoothed Linear input,
    falls back to its own max).

    ``fmt`` = ``"fp8"`` runs the same smoothing with FP8 (e4m3) codes and the
    kind::f8f6f4 GEMM (per-token scales only; "LLM.int8() and SmoothQuant" --
    "example . what you get": FP8 W8A8 on FP8-capable GPUs keeps the
    smoothing).  Code tensors are then uint8 holding e4m3 bytes."""

    def __init__(self, w: Workload, M: int, device, granularity: str = "per_token",
                 fmt: str = "int8", shared: Optional["Block"] = None):
        """``shared``: a Block of the same layer shapes whose prepared state
        (smoothing factors, folded norm parameters, INT8 weights and their
        scales) this one reads instead of holding its own -- one set of
        weights serving several token counts, as a decode step beside a
        prefill step does.  Only the per-token buffers are allocated here."""
        if granularity not in GRANULARITIES:
            raise ValueError("granularity must be one of %s" % (GRANULARITIES,))
        if fmt not in FORMATS:
            raise ValueError("fmt must be one of %s" % (FORMATS,))
        if fmt == "fp8" and granularity != "per_token":
            raise ValueError("FP8 runs with per-token scales")
        self.w = w
        self.M = M
        self.granularity = granularity
        self.fmt = fmt
        code_dtype = torch.uint8 if fmt == "fp8" else torch.int8
        dev = torch.device(device)
        f32 = dict(dtype=torch.float32, device=dev)
        self.act_max: Dict[str, torch.Tensor] = {}
        self.s: Dict[str, Optional[torch.Tensor]] = {}
        self.gamma_f: Dict[str, Optional[torch.Tensor]] = {}
        self.beta_f: Dict[str, Optional[torch.Tensor]] = {}
        self.has_beta: Dict[str, bool] = {}
        for site in w.sites:
            self.s[site.name] = None
            self.gamma_f[site.name] = None
            self.beta_f[site.name] = None
            if site.smoothed:
                self.act_max[site.name] = torch.zeros(site.K, **f32)
                self.s[site.name] = torch.empty(site.K, **f32)
                self.gamma_f[site.name] = torch.empty(site.K, **f32)
        self.Wq: Dict[str, torch.Tensor] = {}
        self.w_scale: Dict[str, torch.Tensor] = {}
        self.out: Dict[str, torch.Tensor] = {}
        self.ws: Dict[str, Optional[torch.Tensor]] = {}
        if shared is not None:
            same = ([(s.name, s.K, s.norm, s.smoothed) for s in shared.w.sites]
                    == [(s.name, s.K, s.norm, s.smoothed) for s in w.sites]
                    and [(l.name, l.site, l.N) for l in shared.w.linears]
                    == [(l.name, l.site, l.N) for l in w.linears])
            if not same or shared.granularity != granularity or shared.fmt != fmt:
                raise ValueError("a shared Block must have the same layers, granularity "
                                 "and format")
            # the dicts themselves are shared: what the other Block's prepare
            # writes is what this one's forward reads
            self.act_max, self.s = shared.act_max, shared.s
            self.gamma_f, self.beta_f = shared.gamma_f, shared.beta_f
            self.Wq, self.w_scale = shared.Wq, shared.w_scale
        for lin in w.linears:
            K = w.site(lin.site).K
            if shared is None:
                self.Wq[lin.name] = torch.empty((lin.N, K), dtype=code_dtype, device=dev)
                self.w_scale[lin.name] = torch.empty(lin.N, **f32)
            self.out[lin.name] = torch.empty((M, lin.N), dtype=torch.bfloat16, device=dev)
            need = sq.gemm_workspace_size(M, lin.N, K, 0)
            self.ws[lin.name] = torch.empty(need, dtype=torch.uint8, device=dev) if need else None
        self.xq: Dict[str, torch.Tensor] = {}
        self.xs: Dict[str, torch.Tensor] = {}
        self.x_absmax: Dict[str, torch.Tensor] = {}  # per-tensor modes: max |y| per site
        self.static: Dict[str, bool] = {}            # O3: the site's max is calibrated
        for site in w.sites:
            self.xq[site.name] = torch.empty((M, site.K), dtype=code_dtype, device=dev)
            self.xs[site.name] = torch.empty(M, **f32)
            self.x_absmax[site.name] = torch.zeros(1, **f32)
            self.static[site.name] = (granularity == "per_tensor_static" and site.smoothed
                                      and site.calibrated)
        self.w_absmax: Dict[str, torch.Tensor] = {l.name: torch.zeros(1, **f32)
                                                  for l in w.linears}
        if shared is not None:
            self.w_absmax = shared.w_absmax
            for site in w.sites:  # O3's static maxima are prepared state too
                if self.static[site.name]:
                    self.x_absmax[site.name] = shared.x_absmax[site.name]
        # A Linear whose bf16 output is the whole input of a later per-token
        # site (no norm, no multiplier: fc1 -> ReLU -> fc2) reduces each
        # output row's max |out| in its GEMM epilogue, so that site's
        # quantisation reads the row once with its max already known.  Only
        # on prefill tiles (the decode plan keeps its own tiles).
        self._side = None  # second stream of `step`, created on first use
        self.rowmax: Dict[str, torch.Tensor] = {}  # source Linear -> [M] row maxima
        # per-tensor variants keep SiLU(gate) * up in bf16 (its tensor-wide max)
        self.h: Dict[str, torch.Tensor] = {
            site.name: torch.empty((M, site.K), dtype=torch.bfloat16, device=dev)
            for site in w.sites if site.act == "silu_mul" and granularity != "per_token"}
        if granularity == "per_token" and fmt == "int8":
            for lin in w.linears:
                site = w.site(lin.site)
                if (lin.source and not site.act and site.norm == sq.NORM_NONE
                        and not site.smoothed):
                    src = next(l for l in w.linears if l.name == lin.source)
                    K_src = w.site(src.site).K
                    if sq.gemm_plan(M, src.N, K_src).kernel != 2:
                        self.rowmax[src.name] = torch.empty(M, **f32)

    # -- offline rows -------------------------------------------------------
    def prepare(self, x_cal: Dict[str, torch.Tensor], W: Dict[str, torch.Tensor],
                gamma: Dict[str, Optional[torch.Tensor]], beta: Dict[str, Optional[torch.Tensor]],
                stream=None, timer: Timer = None) -> "Block":
        for site in self.w.sites:
            self._site_scales(site, x_cal, W, gamma, beta, stream, timer)
        for lin in self.w.linears:
            self._weight_quant(lin, W, stream, timer)
        return self

    def _calibrate(self, site, x_cal, gamma, beta, stream, timer):
        g, b = gamma.get(site.name), beta.get(site.name)
        am = self.act_max[site.name]
        xc = x_cal[site.name]
        am.zero_()
        _run(timer, "calibrate", xc.numel() * xc.element_size() + 4 * site.K,
             lambda: sq.calibrate_absmax(xc, site.norm, g, b, self.w.eps, act_max=am,
                                         stream=stream))

    def _site_weights(self, site, W):
        return [W[l.name] for l in self.w.linears_of(site.name)]

    def _site_scales(self, site, x_cal, W, gamma, beta, stream, timer, calibrated=False,
                     w_max_done=False):
        """Smoothing factors and the folded norm of one site (calibration
        first unless `calibrated`; the weight column maxima, already in
        s, when `w_max_done`), then O3's static max."""
        w = self.w
        g, b = gamma.get(site.name), beta.get(site.name)
        if site.smoothed:
            if b is not None and self.beta_f[site.name] is None:
                self.beta_f[site.name] = torch.empty_like(self.gamma_f[site.name])
            if not calibrated:
                self._calibrate(site, x_cal, gamma, beta, stream, timer)
            am = self.act_max[site.name]
            Ws = self._site_weights(site, W)
            if w_max_done:
                sq.smooth_scales_from_maxima(am, self.s[site.name], w.alpha, w.clamp_eps, g, b,
                                             s=self.s[site.name],
                                             gamma_folded=self.gamma_f[site.name],
                                             beta_folded=self.beta_f[site.name], stream=stream)
            else:
                _run(timer, "smooth_scales",
                     sum(t.numel() * t.element_size() for t in Ws) + 16 * site.K,
                     lambda: sq.compute_smooth_scales(am, Ws, w.alpha, w.clamp_eps, g, b,
                                                      s=self.s[site.name],
                                                      gamma_folded=self.gamma_f[site.name],
                                                      beta_folded=self.beta_f[site.name],
                                                      stream=stream))
        else:
            self.gamma_f[site.name], self.beta_f[site.name] = g, b
        if self.static[site.name]:
            # O3: the static max |y| of the calibration tokens through the folded norm
            xc = x_cal[site.name]
            am = self.x_absmax[site.name]
            am.zero_()
            _run(timer, "static_absmax", xc.numel() * xc.element_size(),
                 lambda: sq.norm_smooth_absmax(xc, site.norm, self.gamma_f[site.name],
                                               self.beta_f[site.name], w.eps, absmax=am,
                                               stream=stream))

    def _weight_quant(self, lin, W, stream, timer):
        Wl = W[lin.name]
        units = Wl.numel() * (Wl.element_size() + 1) + 4 * lin.N
        if self.fmt == "fp8":
            _run(timer, "weight_quant", units,
                 lambda: sq.smooth_quantize_weights_fp8(Wl, self.s[lin.site],
                                                        Wq8=self.Wq[lin.name],
                                                        w_scale=self.w_scale[lin.name],
                                                        stream=stream))
        elif self.granularity != "per_token":  # one more read of W for the matrix-wide max
            _run(timer, "weight_quant", units + Wl.numel() * Wl.element_size(),
                 lambda: sq.smooth_quantize_weights_per_tensor(
                     Wl, self.s[lin.site], Wq=self.Wq[lin.name],
                     w_scale=self.w_scale[lin.name], w_absmax=self.w_absmax[lin.name],
                     stream=stream))
        else:
            _run(timer, "weight_quant", units,
                 lambda: sq.smooth_quantize_weights(Wl, self.s[lin.site], Wq=self.Wq[lin.name],
                                                    w_scale=self.w_scale[lin.name],
                                                    stream=stream))

    # -- runtime rows -------------------------------------------------------
    def forward(self, x: Dict[str, torch.Tensor], stream=None, timer: Timer = None
                ) -> Dict[str, torch.Tensor]:
        for site in self.w.sites:
            self._quantize_site(site, x, stream, timer)
            self._gemms(site, stream, timer)
        return self.out

    def _source(self, site):
        return next((l.source for l in self.w.linears if l.site == site.name and l.source), None)

    def _quantize_site(self, site, x, stream, timer):
        w = self.w
        src = self._source(site)
        xin = self.out[src] if src else x[site.name]
        fused_act = site.act == "silu_mul" and site.name not in self.h
        if site.act == "silu_mul":
            # the down projection's input, SiLU(gate) * up of the merged
            # projection's output: per-token codes in the same pass; the
            # per-tensor variants store h and quantise it as a tensor
            h = self.h.get(site.name)
            gu = xin
            _run(timer, "silu_mul_quant",
                 gu.numel() * gu.element_size() + self.M * site.K * (1 + 2 * (h is not None))
                 + 4 * self.M,
                 lambda: sq.silu_mul_quant_per_token(gu, self.xq[site.name], self.xs[site.name],
                                                     h_out=h, stream=stream,
                                                     fp8=self.fmt == "fp8"))
            if h is not None:
                xin = h
        nparam = (self.gamma_f[site.name] is not None) + (self.beta_f[site.name] is not None)
        units = xin.numel() * (xin.element_size() + 1) + 4 * self.M + 4 * site.K * nparam
        gf, bf = self.gamma_f[site.name], self.beta_f[site.name]
        if fused_act:
            return
        if self.fmt == "fp8":
            _run(timer, "norm_quant", units,
                 lambda: sq.norm_smooth_quant_per_token_fp8(xin, site.norm, gf, bf, w.eps,
                                                            self.xq[site.name],
                                                            self.xs[site.name], stream=stream))
        elif src in self.rowmax:
            am = self.rowmax[src]
            _run(timer, "norm_quant", units,
                 lambda: sq.quant_per_token_given_absmax(xin, am, self.xq[site.name],
                                                         self.xs[site.name], stream=stream))
        elif self.granularity == "per_token":
            _run(timer, "norm_quant", units,
                 lambda: sq.norm_smooth_quant_per_token(xin, site.norm, gf, bf, w.eps,
                                                        self.xq[site.name],
                                                        self.xs[site.name], stream=stream))
        else:
            am = self.x_absmax[site.name]
            if not self.static[site.name]:  # O2: this tensor's own max first
                am.zero_()
                _run(timer, "absmax", xin.numel() * xin.element_size() + 4 * site.K * nparam,
                     lambda: sq.norm_smooth_absmax(xin, site.norm, gf, bf, w.eps, absmax=am,
                                                   stream=stream))
            _run(timer, "norm_quant", units,
                 lambda: sq.norm_smooth_quant_per_tensor(xin, site.norm, am, gf, bf, w.eps,
                                                         self.xq[site.name],
                                                         self.xs[site.name], stream=stream))

    def _gemms(self, site, stream, timer):
        for lin in self.w.linears_of(site.name):
            def gemm(lin=lin, site=site):
                if self.fmt == "fp8":
                    sq.fp8_gemm_dequant(self.xq[site.name], self.Wq[lin.name],
                                        self.xs[site.name], self.w_scale[lin.name],
                                        "bf16_relu" if lin.relu else "bf16",
                                        out=self.out[lin.name], workspace=self.ws[lin.name],
                                        whole_k=self.ws[lin.name] is None, stream=stream)
                    return
                if lin.name in self.rowmax:
                    sq.w8a8_gemm_dequant_rowmax(
                        self.xq[site.name], self.Wq[lin.name], self.xs[site.name],
                        self.w_scale[lin.name], "bf16_relu" if lin.relu else "bf16",
                        out=self.out[lin.name], row_absmax=self.rowmax[lin.name],
                        stream=stream)
                    return
                sq.w8a8_gemm_dequant(self.xq[site.name], self.Wq[lin.name],
                                     self.xs[site.name], self.w_scale[lin.name],
                                     "bf16_relu" if lin.relu else "bf16",
                                     out=self.out[lin.name], workspace=self.ws[lin.name],
                                     stream=stream)
            _run(timer, "gemm:" + lin.name, 2.0 * self.M * lin.N * site.K, gemm)

    # -- the whole step, independent work on two streams ----------------------
    def step(self, x_cal, W, gamma, beta, x) -> Dict[str, torch.Tensor]:
        """``prepare`` then ``forward`` (the same kernels, the same results),
        with work that does not depend on each other run concurrently on a
        second stream: calibration beside the weight column maxima, and the
        weight quantisation beside the quantisation of the block's input
        sites.  Both streams join the current one before the GEMMs and at the
        end, so the step is ordered like one stream to its caller (and can be
        captured in a CUDA graph)."""
        main = torch.cuda.current_stream()
        side = self._scales_two_streams(x_cal, W, gamma, beta)
        w = self.w
        # weights on the side stream, the input sites' codes on this one
        side.wait_stream(main)
        with torch.cuda.stream(side):
            for lin in w.linears:
                self._weight_quant(lin, W, None, None)
        inputs = [site for site in w.sites if self._source(site) is None]
        for site in inputs:
            self._quantize_site(site, x, None, None)
        main.wait_stream(side)
        for site in w.sites:
            if site in inputs:
                self._gemms(site, None, None)
            else:
                self._quantize_site(site, x, None, None)
                self._gemms(site, None, None)
        return self.out

    def _scales_two_streams(self, x_cal, W, gamma, beta):
        """Calibration on a second stream beside the weight column maxima on
        the current one, joined; then the smoothing factors and the fold.
        Returns the second stream."""
        main = torch.cuda.current_stream()
        if self._side is None:
            self._side = torch.cuda.Stream()
        side = self._side
        smoothed = [site for site in self.w.sites if site.smoothed]
        side.wait_stream(main)
        with torch.cuda.stream(side):
            for site in smoothed:
                self._calibrate(site, x_cal, gamma, beta, None, None)
        for site in smoothed:
            sq.weight_column_max(self._site_weights(site, W), w_max=self.s[site.name])
        main.wait_stream(side)
        for site in self.w.sites:
            self._site_scales(site, x_cal, W, gamma, beta, None, None, calibrated=True,
                              w_max_done=True)
        return side

    def prepare_two_streams(self, x_cal, W, gamma, beta) -> "Block":
        """``prepare`` with the calibration running beside the weight column
        maxima on a second stream (joined before the smoothing factors); the
        same kernels and the same results, ordered like one stream to the
        caller."""
        self._scales_two_streams(x_cal, W, gamma, beta)
        for lin in self.w.linears:
            self._weight_quant(lin, W, None, None)
        return self

    # -- launch accounting ---------------------------------------------------
    def prepare_launches(self) -> int:
        """Kernels of this library one ``prepare`` launches: per smoothed site
        calibration + one column-max per Linear reading it + the finalise
        kernel; one weight-quantisation kernel per Linear."""
        n = 0
        for site in self.w.sites:
            if site.smoothed:
                n += 2 + len(self.w.linears_of(site.name))
            if self.static[site.name]:
                n += 1  # the static max over the calibration tokens
        per_tensor = self.granularity != "per_token"
        return n + len(self.w.linears) * (2 if per_tensor else 1)

    def forward_launches(self) -> int:
        """Kernels one ``forward`` launches: norm-quant per site, and per Linear
        the kernels of its GEMM plan (the main kernel, plus the split-K
        reduction or stream-K fix-up where the plan has one)."""
        n = len(self.w.sites)
        n += sum(1 for site in self.w.sites if site.name in self.h)  # h, then its codes
        if self.granularity != "per_token":
            n += sum(1 for site in self.w.sites if not self.static[site.name])  # O2 max pass
        for lin in self.w.linears:
            if lin.name in self.rowmax or self.fmt == "fp8":
                n += 1  # one kernel (FP8: whole-K tiles; row max: the zeroing is a memset)
            else:
                n += sq.gemm_plan(self.M, lin.N, self.w.site(lin.site).K).launches
        return n

    # -- CUDA graph ----------------------------------------------------------
    def capture(self, x_cal, W, gamma, beta, x, timer: Timer = None, warmup: int = 1,
                overlap: bool = True):
        """Records one whole step into a CUDA graph and returns it;
        ``graph.replay()`` reruns every kernel of the step on the current
        stream with no host work per kernel.  With ``overlap`` the step is
        ``step`` (independent work on a second stream, joined inside the
        graph); otherwise ``prepare`` then ``forward`` in one stream, with the
        ``timer`` hooks captured too (e.g. CUDA event records, which then time
        each call inside every replay).  The step's tensors must stay where
        they are between replays (the graph holds their addresses)."""
        overlap = overlap and timer is None
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):  # first use of each kernel outside the capture
            for _ in range(warmup):
                if overlap:
                    self.step(x_cal, W, gamma, beta, x)
                else:
                    self.prepare(x_cal, W, gamma, beta)
                    self.forward(x)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            if overlap:
                self.step(x_cal, W, gamma, beta, x)
            else:
                self.prepare(x_cal, W, gamma, beta, timer=timer)
                self.forward(x, timer=timer)
        return graph


def capture_graph(fn, warmup: int = 1):
    """Records ``fn`` (a sequence of library calls on the current stream,
    possibly forking to others and joining back) into a CUDA graph after
    ``warmup`` runs outside the capture (the first use of each kernel sets
    its launch attributes)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(warmup):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    return graph


def capture_forward(blk: Block, x, warmup: int = 1):
    """The runtime rows of one step (norm + per-token quantisation, GEMMs with
    the dequant epilogue, for every Linear) as one CUDA graph."""
    return capture_graph(lambda: blk.forward(x), warmup)


def capture_prepare(blk: Block, x_cal, W, gamma, beta, warmup: int = 1):
    """The offline rows (calibration, smoothing factors and fold, weight
    smoothing and quantisation) as one CUDA graph, calibration beside the
    weight column maxima."""
    return capture_graph(lambda: blk.prepare_two_streams(x_cal, W, gamma, beta), warmup)


# Thin functional wrappers (used by tests and the smoke check).

def prepare(w: Workload, x_cal, W, gamma, beta, M: Optional[int] = None, device="cuda",
            stream=None, granularity: str = "per_token", fmt: str = "int8") -> Block:
    return Block(w, w.M if M is None else M, device, granularity, fmt).prepare(
        x_cal, W, gamma, beta, stream)
