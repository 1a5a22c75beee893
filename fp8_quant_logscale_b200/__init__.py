"""B200 (sm_100a) FP8 in-context-learning attention layer.

Steps, each a hand-written CUDA kernel behind the C ABI in include/sdm_fp8.h:
fused LogScale/GatedLogScale query scaling, FP8 e4m3 quantisation with
context-derived per-head scales, tcgen05 FP8 flash attention, and split-KV
cached prediction over a resident FP8 K/V cache; plus the normal-precision
(fp16 tcgen05) attention that the precision rule keeps for the final layer and
short contexts.
"""
from .binding import (FP8Cache, OffloadedFP8Cache, SdmError, cached_attention, cached_attention_offload,
                      fp8_attention, fp8_eligible, fp8_quantize_context, gqa_prefill, icl_attention, icl_attention_f16,
                      icl_layer, lib, new_workspace, qscale_fused, sync_status, workspace_size)

__all__ = ["FP8Cache", "OffloadedFP8Cache", "SdmError", "cached_attention", "cached_attention_offload",
           "fp8_attention", "fp8_eligible", "fp8_quantize_context", "gqa_prefill",
           "icl_attention", "icl_attention_f16", "icl_layer", "lib", "new_workspace", "qscale_fused", "sync_status",
           "workspace_size"]
