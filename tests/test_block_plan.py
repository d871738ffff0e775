"""Host-side choices of the block (no GPU): which sites take the row-max
epilogue, the SiLU(gate)*up pass or a stored h, and how many kernels a step
launches.  Blocks are built on the CPU device (no kernel runs)."""
import pytest

from w8a8_int8_quantized_norm_b200 import pipeline, sq
from w8a8_int8_quantized_norm_b200 import synthetic as S


def test_relu_gemm_feeding_a_per_token_site_reduces_row_maxima():
    blk = pipeline.Block(S.OPT66B_MLP, 256, "cpu")
    assert set(blk.rowmax) == {"fc1"} and blk.h == {}
    # decode tiles keep their own plan: no row-max epilogue
    assert pipeline.Block(S.OPT66B_MLP, 64, "cpu").rowmax == {}
    # neither per-tensor scales nor FP8 codes use it
    assert pipeline.Block(S.OPT66B_MLP, 256, "cpu", "per_tensor_dynamic").rowmax == {}
    assert pipeline.Block(S.OPT66B_MLP, 256, "cpu", fmt="fp8").rowmax == {}


def test_silu_mul_site_is_fused_or_stored():
    w = S.WORKLOADS["llama-block-8192-decode-m8"]
    assert pipeline.Block(w, 8, "cpu").h == {}                  # fused INT8 pass
    assert pipeline.Block(w, 8, "cpu", fmt="fp8").h == {}       # fused FP8 pass
    assert set(pipeline.Block(w, 8, "cpu", "per_tensor_static").h) == {"mlp_act"}


def test_bad_format_and_granularity_are_refused():
    with pytest.raises(ValueError):
        pipeline.Block(S.SMALL, 16, "cpu", fmt="int4")
    with pytest.raises(ValueError):
        pipeline.Block(S.SMALL, 16, "cpu", "per_tensor_dynamic", fmt="fp8")


def _plan_launches(M, w):
    return sum(sq.gemm_plan(M, l.N, w.site(l.site).K).launches for l in w.linears)


def test_forward_launch_counts():
    # OPT-66B prefill: two row passes (norm + quant, given-max requant), two GEMMs
    # (fc1 with the row-max epilogue: one kernel, the zeroing is a memset)
    w = S.OPT66B_MLP
    assert pipeline.Block(w, 256, "cpu").forward_launches() == 2 + 1 + \
        sq.gemm_plan(256, 9216, 36864).launches
    # Llama decode, INT8: four sites, the GEMMs' plans (stream-K fix-ups included)
    w = S.WORKLOADS["llama-block-8192-decode-m8"]
    assert pipeline.Block(w, 8, "cpu").forward_launches() == 4 + _plan_launches(8, w)
    # FP8: whole-K tiles (one kernel per GEMM), the SiLU*up site in one pass
    assert pipeline.Block(w, 8, "cpu", fmt="fp8").forward_launches() == 4 + 4
    # O2: one max pass per site, plus the stored-h pass
    assert pipeline.Block(w, 8, "cpu", "per_tensor_dynamic").forward_launches() == \
        4 + 4 + 1 + _plan_launches(8, w)
