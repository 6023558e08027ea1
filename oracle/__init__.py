"""CPU oracle for the Averis mean-residual split NVFP4 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It is a plain, slow, obviously correct
restatement of what the method computes, written from

  * "The Curse and Blessing of Mean Bias in FP4-Quantized LLM Training"
    (Cao, Huang et al.), as reviewed on the Lighthouse blog page
    "Averis：FP4 训练不稳定的元凶是一个秩一均值偏差" -- section 二 2.1
    (column mean mu_X = (1/l) 1^T X), section 二 "Averis 方法" (the forward
    and backward split equations), section 三 3.1 (E2M1 NVFP4, stochastic
    rounding by default);
  * the arXiv abstract page of the same paper (mean-residual splitting using
    only reductions and elementwise subtractions before FP4 quantization);
  * the gist.science technical summary, section 2 "Il Metodo Proposto:
    Averis" (X_R = X - 1 mu_X^T, mean and residual quantized separately).

The pages fix the algebra of the split and the number format's name only.
Every finer numeric rule (block size 16, E4M3 block scales, FP32 tensor
scale, the fixed reduction order, the Philox stream mapping, the scale
layout) is a stated reading; each function says which one it follows.

It shares no code with the CUDA path: no kernels, headers, tables or
helpers.  Floating point that the contract fixes to fp32 is done in numpy
float32 (single IEEE operations, round to nearest even, no contraction);
reference products are fp64.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, brute force, published known-answer vectors or
invariants, except the end-to-end overhead figure, which the pages quote on
unstated hardware and which therefore has no oracle ("parity unpinned").
"""

from .philox import philox4x32_10, random_bits16
from .nvfp4 import (
    E2M1_GRID,
    e2m1_rne,
    e2m1_sr,
    e2m1_value,
    e4m3_rne_satfinite,
    e4m3_value,
    nvfp4_quantize,
    nvfp4_dequantize,
    scale_offset,
    swizzle_scales,
    unswizzle_scales,
    pack_codes,
    unpack_codes,
    NVFP4,
)
from .averis import (
    TAGS,
    column_mean,
    mean_residual_split,
    column_mean_and_residual_amax,
    averis_split_quant,
    vanilla_quant,
    quant_weight,
    bias_row,
    gemm_reference,
    averis_linear_reference,
    vanilla_linear_reference,
    padded_tokens,
    transpose_padded,
    averis_split_quant_t,
    vanilla_quant_t,
    wgrad_reference,
    averis_wgrad_reference,
    vanilla_wgrad_reference,
    MOE_ALIGN,
    moe_offsets,
    moe_split_quant,
    moe_quant_weights,
    moe_linear_reference,
)
from . import stats

__all__ = [
    "philox4x32_10", "random_bits16",
    "E2M1_GRID", "e2m1_rne", "e2m1_sr", "e2m1_value", "e4m3_rne_satfinite",
    "e4m3_value", "nvfp4_quantize", "nvfp4_dequantize", "scale_offset",
    "swizzle_scales", "unswizzle_scales", "pack_codes", "unpack_codes", "NVFP4",
    "TAGS", "column_mean", "mean_residual_split", "column_mean_and_residual_amax",
    "averis_split_quant", "vanilla_quant", "quant_weight", "bias_row",
    "gemm_reference", "averis_linear_reference", "vanilla_linear_reference",
    "stats",
]
