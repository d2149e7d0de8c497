"""fp64 CPU oracle of the routed MoE layer -- TEST INFRASTRUCTURE ONLY.

Imported by the tests, by the smoke check and by the bench's CPU-baseline leg,
never by the library.  It shares no code with the CUDA path.
"""
from .moe_oracle import (router_logits, topk_gates, counts_offsets, permutation, route,
                         dispatch, combine, combine_bwd, dispatch_bwd, experts_fwd, experts_bwd,
                         swiglu_bwd, silu, layer_fwd, layer_bwd, rel_fro, load_stats)
from .mx import bf16_round, tf32_round, mx_quantize, mx_quantize_dequantize, e4m3_round, e4m3_encode, e4m3_decode

__all__ = ["router_logits", "topk_gates", "counts_offsets", "permutation", "route", "dispatch",
           "combine", "combine_bwd", "dispatch_bwd", "experts_fwd", "experts_bwd", "swiglu_bwd",
           "silu", "bf16_round", "tf32_round", "load_stats", "layer_fwd", "layer_bwd", "rel_fro", "mx_quantize", "mx_quantize_dequantize",
           "e4m3_round", "e4m3_encode", "e4m3_decode"]
