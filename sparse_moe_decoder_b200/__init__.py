"""B200-native sparse MoE feed-forward path of the ZONOS2 decoder (libzmoe + thin binding)."""
from .zmoe import (ZMOE_BF16, ZMOE_F32, ZmoeError, lib, zmoe_combine, zmoe_decode_stack, zmoe_delay_shear, zmoe_delay_unshear,
                   zmoe_embed_sum_rmsnorm, zmoe_get_device_errors, zmoe_grouped_swiglu,
                   zmoe_grouped_swiglu_workspace_size, zmoe_grouped_swiglu_f16h, zmoe_moe_layer, zmoe_moe_layer_f16h, zmoe_moe_layer_w8a8, zmoe_prepare_w_down_f16, zmoe_moe_layer_fp8, zmoe_moe_layer_workspace_size, zmoe_output_heads, zmoe_permute, zmoe_speaker_prefix,
                   zmoe_permute_workspace_size, zmoe_rmsnorm, zmoe_route, zmoe_version)
from .layer import DecodeStack, MoELayerRunner, MoEWeights

__all__ = [
    "ZMOE_BF16", "ZMOE_F32", "ZmoeError", "lib", "zmoe_combine", "zmoe_decode_stack", "zmoe_delay_shear", "zmoe_delay_unshear",
    "zmoe_embed_sum_rmsnorm", "zmoe_get_device_errors", "zmoe_grouped_swiglu", "zmoe_grouped_swiglu_workspace_size", "zmoe_grouped_swiglu_f16h", "zmoe_moe_layer_f16h", "zmoe_moe_layer_w8a8", "zmoe_prepare_w_down_f16",
    "zmoe_moe_layer", "zmoe_moe_layer_fp8", "zmoe_moe_layer_workspace_size", "zmoe_output_heads", "zmoe_speaker_prefix", "zmoe_permute", "zmoe_permute_workspace_size", "zmoe_rmsnorm", "zmoe_route", "zmoe_version",
    "DecodeStack", "MoELayerRunner", "MoEWeights",
]
