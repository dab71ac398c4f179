"""B200-native (sm_100a) denoise path for block text diffusion.

The compute lives in libdg.so (CUDA kernels behind the C ABI in include/dg.h); this package
is its thin Python binding.  Build with `python -m block_text_diffusion_dg_b200.build`.
"""
from .api import (DiffusionModel, Sampler, canvas_attention, e4m3_pitch, generate, make_config,
                  moe_ffn, moe_ffn_e4m3, moe_ffn_nvfp4, moe_workspace, quantize_e4m3,
                  quantize_experts, quantize_head, quantize_nvfp4, workspace_bytes)

__all__ = ["DiffusionModel", "Sampler", "canvas_attention", "e4m3_pitch", "generate",
           "make_config", "moe_ffn", "moe_ffn_e4m3", "moe_ffn_nvfp4", "moe_workspace",
           "quantize_e4m3", "quantize_experts", "quantize_head", "quantize_nvfp4",
           "workspace_bytes"]
