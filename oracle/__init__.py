"""CPU oracle for the W4A8 routed-expert MoE layer.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, float64 numpy
restatement of what the layer computes.  It exists to check the CUDA path and
is not part of it: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` may import it.  The CUDA library never
calls it and shares no code with it (the only common module is the seeded
input generator ``workloads``, which holds no arithmetic of the method).

Sources.  The method is described by five web pages about 4-bit-weight /
8-bit-activation versions of the GLM-5.3 MoE model:

* "GLM-5.3-W4A8" model card (zh): routed experts in INT4 with group size 128,
  activations FP8 with per-token dynamic scales (intro; table "differences from
  the other 4-bit releases"); symmetric INT4 per group, packed as
  compressed-tensors ``pack-quantized`` uint4b8 in int32 words, 8 weights per
  word (section "quantisation method"; note on the ~370B parameter display);
  the expert GEMM converts INT4 to FP8 in the kernel and never dequantises to
  BF16 (intro; "quantisation method").
* "GLM-5.3-W4AFP8" model card (PhalaCloud): INT4 group-128 experts, FP8
  activations; dequantisation audit (section "Verification").
* "GLM-5.3 EVAL_DETAILS" (zh), section 1: expert-weight reconstruction error
  (naive RTN 0.124, RTN with the per-group MSE clip search 0.103).
* "GLM-5.3-Channel-INT4-w4a8" (hygon): the per-channel INT4 weight /
  per-token INT8 activation variant (quantisation table: RTN, static,
  per-channel INT4 experts; dynamic per-token INT8 activations).
* "From 755GB to 395GB" (Bitdeer AI blog): 256 routed experts per MoE layer,
  3 projections per expert.
* The non-expert layers, the shared expert among them, keep FP8 E4M3 weights
  with 128 x 128 block scales (GLM-5.3-W4A8 model card, intro and
  "quantisation method"); ``shared.py`` is that expert.

Steps the pages leave open are fixed by the plainest reading; each function's
docstring states the reading it takes.  Where a float decides an integer (an
INT4 value, an FP8 code, a bf16 scale) the oracle takes that decision in the
precision the kernels use (IEEE float32 division, correctly rounded), emulated
here as float64 arithmetic rounded to float32, which is exact for one
division (53 >= 2*24 + 2).

Parity pins: every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_*.py`` against a library routine, a closed form, an
invariant or brute force on tiny inputs.  The end-to-end values at full size
have no pin beyond those of their parts.
"""
from .numerics import (bf16_bits_to_f64, f64_to_bf16_bits, bf16_round, f32_round,
                       e4m3_decode, e4m3_encode, E4M3_MAX)
from .quant import (rtn_quantize_int4, mse_clip_quantize_int4, mse_clip_candidates,
                    MSE_ERR_REL_BOUND, CLIP_RATIOS, pack_uint4b8,
                    unpack_uint4b8, dequantize_int4, quant_act_fp8_per_token,
                    quant_act_int8_per_token, rtn_quantize_int4_channel)
from .moe import route_topk, permute_by_expert, moe_forward, expert_forward, ExpertStore
from .shared import (quant_fp8_block, dequant_fp8_block, quant_act_fp8_group,
                     dequant_act_fp8_group, shared_expert_forward)

__all__ = ["bf16_bits_to_f64", "f64_to_bf16_bits", "bf16_round", "f32_round",
           "e4m3_decode", "e4m3_encode", "E4M3_MAX", "rtn_quantize_int4",
           "mse_clip_quantize_int4", "mse_clip_candidates", "MSE_ERR_REL_BOUND", "CLIP_RATIOS",
           "pack_uint4b8", "unpack_uint4b8", "dequantize_int4",
           "quant_act_fp8_per_token", "quant_act_int8_per_token", "route_topk", "permute_by_expert",
           "moe_forward", "expert_forward", "ExpertStore", "rtn_quantize_int4_channel", "quant_fp8_block",
           "dequant_fp8_block", "quant_act_fp8_group", "dequant_act_fp8_group",
           "shared_expert_forward"]
