"""Seeded synthetic inputs for the W8A8 linear workloads.

This module only draws random numbers and arranges them into the shapes of the
workloads; it holds none of the SmoothQuant arithmetic, so both the CUDA path
and the CPU oracle can be fed from it without sharing any of the method.

Value laws (the pages describe activations with a few persistent outlier
channels that are tens of times larger than the rest in every token):

* activations ``X`` ~ N(0, 1), and every token's value in an outlier channel
  j is multiplied by a per-channel factor c_j that is fixed for the workload;
* weights ``W`` ~ N(0, 0.02), nn.Linear layout ``[N_out, K_in]``;
* RMSNorm / LayerNorm ``gamma`` ~ U[0.5, 1.5]; LayerNorm ``beta`` ~ N(0, 0.1);
* the calibration batch follows the activation law (same outlier channels and
  factors) from its own random stream.

Every tensor comes from its own substream of ``SeedSequence(seed)``, so any
one of them can be regenerated alone.  bf16 tensors are generated in fp32 and
rounded to bf16 by torch; they are returned as ``uint16`` bit patterns (the
oracle's bf16 convention) and can be viewed as ``torch.bfloat16``.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, List, Optional, Tuple

import numpy as np

NORM_NONE, NORM_RMS, NORM_LAYER = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class OutlierLaw:
    """Which activation channels are outliers and by how much."""
    channels: Optional[Tuple[int, ...]] = None  # fixed channel ids, or None = random
    count: int = 0                              # number of random channels
    fraction: float = 0.0                       # or a fraction of K (rounded)
    factor: Optional[float] = None              # fixed multiplier ...
    factor_range: Optional[Tuple[float, float]] = None  # ... or U[lo, hi] per channel

    def pick(self, K: int, rng: np.random.Generator) -> Tuple[np.ndarray, np.ndarray]:
        if self.channels is not None:
            ch = np.array(self.channels, dtype=np.int64)
        else:
            n = self.count if self.count else max(1, int(round(self.fraction * K)))
            ch = np.sort(rng.choice(K, size=n, replace=False)).astype(np.int64)
        if self.factor_range is not None:
            lo, hi = self.factor_range
            c = rng.uniform(lo, hi, size=ch.shape[0]).astype(np.float32)
        else:
            c = np.full(ch.shape[0], self.factor, dtype=np.float32)
        return ch, c


@dataclasses.dataclass(frozen=True)
class Site:
    """An activation tensor feeding one or more Linears.

    ``norm`` is the norm in front of it (``NORM_NONE`` when the Linear reads the
    tensor directly).  ``smoothed`` says whether the Linears that read it are
    smoothed (their s folded into the norm, or applied as a per-channel
    multiplier when there is no norm)."""
    name: str
    K: int
    norm: int
    smoothed: bool
    calibrated: bool = True  # smoothed sites need a calibration batch
    # how a site fed by a Linear's output is formed from it: "" = the output
    # itself; "silu_mul" = SiLU(first half) * second half (gate, up), K wide
    act: str = ""


@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    site: str        # activation site it reads
    N: int
    relu: bool = False
    source: Optional[str] = None  # Linear whose output forms this Linear's site, if any


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int                       # tokens per step
    M_cal: int                   # calibration tokens
    dtype: str                   # "f32" or "bf16" activations and weights
    alpha: float
    sites: Tuple[Site, ...]
    linears: Tuple[Linear, ...]
    outliers: OutlierLaw
    eps: float = 1e-5            # norm epsilon
    clamp_eps: float = 1e-5      # epsilon of the smoothing-factor clamps

    def site(self, name: str) -> Site:
        return next(s for s in self.sites if s.name == name)

    def linears_of(self, site: str) -> List[Linear]:
        return [l for l in self.linears if l.site == site]

    def gemm_ops(self, M: Optional[int] = None) -> int:
        M = self.M if M is None else M
        return sum(2 * M * l.N * self.site(l.site).K for l in self.linears)


def _llama_block(M: int, name: str) -> Workload:
    return Workload(
        name=name, M=M, M_cal=512, dtype="bf16", alpha=0.8,
        sites=(Site("attn_norm", 8192, NORM_RMS, True),
               Site("attn_out", 8192, NORM_NONE, False, calibrated=False),
               Site("mlp_norm", 8192, NORM_RMS, True),
               Site("mlp_act", 28672, NORM_NONE, False, calibrated=False, act="silu_mul")),
        linears=(Linear("qkv", "attn_norm", 10240),
                 Linear("o_proj", "attn_out", 8192),
                 Linear("gate_up", "mlp_norm", 57344),
                 Linear("down", "mlp_act", 8192, source="gate_up")),
        outliers=OutlierLaw(fraction=0.001, factor=50.0))


WORKLOADS: Dict[str, Workload] = {}


def _register(w: Workload) -> Workload:
    WORKLOADS[w.name] = w
    return w


# A single smoothed linear with no norm in front: its 1/s is a per-channel
# multiplier on the input (the fold with gamma = 1).
SMALL = _register(Workload(
    name="smoothed-linear-16x64x64", M=16, M_cal=64, dtype="f32", alpha=0.5,
    sites=(Site("x", 64, NORM_NONE, True),),
    linears=(Linear("fc", "x", 64),),
    outliers=OutlierLaw(channels=(5, 41), factor=40.0)))

# OPT-style prefill: RMSNorm -> fused QKV 4096 -> 12288 on 2048 tokens.
OPT_QKV = _register(Workload(
    name="opt-prefill-rmsnorm-qkv-2048x4096x12288", M=2048, M_cal=512, dtype="bf16", alpha=0.5,
    sites=(Site("attn_norm", 4096, NORM_RMS, True),),
    linears=(Linear("qkv", "attn_norm", 12288),),
    outliers=OutlierLaw(count=8, factor_range=(20.0, 100.0))))

# OPT-66B-width MLP: LayerNorm -> fc1 -> ReLU -> per-token requant -> fc2.
OPT66B_MLP = _register(Workload(
    name="opt66b-mlp-layernorm-fc1-relu-fc2-4096x9216x36864", M=4096, M_cal=512, dtype="bf16",
    alpha=0.5,
    sites=(Site("ffn_norm", 9216, NORM_LAYER, True),
           Site("fc1_act", 36864, NORM_NONE, False, calibrated=False)),
    linears=(Linear("fc1", "ffn_norm", 36864, relu=True),
             Linear("fc2", "fc1_act", 9216, source="fc1")),
    outliers=OutlierLaw(fraction=0.001, factor=60.0)))

# Llama-style decoder block, hidden 8192, 8 sequences x 2048 tokens prefill.
LLAMA_BLOCK = _register(_llama_block(16384, "llama-block-8192-prefill-16384tok"))

# Decode sweep on the same block weights: M tokens per step.
for _m in (1, 8, 32, 128):
    _register(_llama_block(_m, "llama-block-8192-decode-m%d" % _m))


# --------------------------------------------------------------------------
# generation
# --------------------------------------------------------------------------

def _stream(seed: int, *path: str) -> np.random.Generator:
    """Independent substream for one named tensor of one workload."""
    key = [zlib.crc32(p.encode()) for p in path]
    return np.random.default_rng(np.random.SeedSequence([seed, *key]))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 data to bf16 storage (torch's cast) and return the bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    return to_bf16_bits(a) if dtype == "bf16" else np.ascontiguousarray(a, dtype=np.float32)


def outlier_channels(w: Workload, site: str, seed: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """(channel ids, per-channel factors) of the site's outlier channels."""
    return w.outliers.pick(w.site(site).K, _stream(seed, _family(w), site, "outlier-channels"))


def _family(w: Workload) -> str:
    # decode workloads draw their weights and norm parameters from the prefill
    # block they belong to, so every M shares one set of weights
    return LLAMA_BLOCK.name if w.name.startswith("llama-block-8192") else w.name


def activations(w: Workload, site: str, rows: int, stream: str, seed: int = 0,
                row_offset: int = 0) -> np.ndarray:
    """``rows`` tokens of the activation law for ``site`` ([rows, K])."""
    K = w.site(site).K
    ch, c = outlier_channels(w, site, seed)
    rng = _stream(seed, w.name, site, stream)
    if row_offset:
        rng.standard_normal((row_offset, K), dtype=np.float32)  # skip ahead
    x = rng.standard_normal((rows, K), dtype=np.float32)
    x[:, ch] *= c[None, :]
    return _store(x, w.dtype)


def weight(w: Workload, lin: Linear, seed: int = 0) -> np.ndarray:
    K = w.site(lin.site).K
    rng = _stream(seed, _family(w), lin.name, "weight")
    a = rng.standard_normal((lin.N, K), dtype=np.float32)
    a *= np.float32(0.02)
    return _store(a, w.dtype)


def norm_params(w: Workload, site: str, seed: int = 0):
    """(gamma, beta) fp32 for the site's norm; None where the norm has none."""
    s = w.site(site)
    if s.norm == NORM_NONE:
        return None, None
    K = s.K
    gamma = _stream(seed, _family(w), site, "gamma").uniform(0.5, 1.5, K).astype(np.float32)
    beta = None
    if s.norm == NORM_LAYER:
        beta = (_stream(seed, _family(w), site, "beta").standard_normal(K, dtype=np.float32)
                * np.float32(0.1))
    return gamma, beta


@dataclasses.dataclass
class Inputs:
    workload: Workload
    x: Dict[str, np.ndarray]           # runtime activations per site (sites fed by a
                                       # Linear's output are absent)
    x_cal: Dict[str, np.ndarray]       # calibration batch per smoothed site
    W: Dict[str, np.ndarray]           # weights per Linear
    gamma: Dict[str, Optional[np.ndarray]]
    beta: Dict[str, Optional[np.ndarray]]


def make_inputs(w: Workload, seed: int = 0, rows: Optional[int] = None,
                weights: bool = True, token_seed: Optional[int] = None) -> Inputs:
    """All inputs of one workload.  ``rows`` limits the runtime token count
    (a prefix of the full token stream).  ``token_seed`` (default ``seed``)
    draws the runtime tokens alone: data-parallel replicas share weights, norm
    parameters and the calibration batch and differ only in their tokens."""
    M = w.M if rows is None else rows
    ts = seed if token_seed is None else token_seed
    fed = {l.site for l in w.linears if l.source is not None}
    x, xc, Ws, g, b = {}, {}, {}, {}, {}
    for s in w.sites:
        if s.name not in fed:
            x[s.name] = activations(w, s.name, M, "x", ts)
        if s.smoothed and s.calibrated:
            xc[s.name] = activations(_cal_workload(w), s.name, w.M_cal, "x_cal", seed)
        g[s.name], b[s.name] = norm_params(w, s.name, seed)
    if weights:
        for l in w.linears:
            Ws[l.name] = weight(w, l, seed)
    return Inputs(w, x, xc, Ws, g, b)


def _cal_workload(w: Workload) -> Workload:
    # the calibration batch belongs to the weights' family so every decode M
    # calibrates on the same tokens as the prefill block
    return WORKLOADS[_family(w)]
