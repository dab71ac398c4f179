"""ctypes declarations of libdg's C ABI (include/dg.h).  Marshalling only."""
import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")

DG_OK = 0
DG_ERR = {-1: "DG_ERR_INVALID_ARG", -2: "DG_ERR_CAPACITY", -3: "DG_ERR_CUDA",
          -4: "DG_ERR_TIMEOUT", -5: "DG_ERR_UNSUPPORTED"}
DTYPE_BF16, DTYPE_FP32, DTYPE_BF16_E4M3, DTYPE_BF16_NVFP4 = 0, 1, 2, 3
STATE_DONE, STATE_STOP_STEP, STATE_WOULD_STOP, STATE_STEPS_RUN, STATE_LOCKED, STATE_ERROR = range(6)
STATE_WORDS = 16
KERNEL_KINDS = dict(expert_gate_up=0, expert_down=1, attention=2, lm_head=3, qkv=4,
                    o_proj=5, sampler=6, router=8, qkv_finalize=9, attn_combine=10,
                    residual_norm=11, router_topk=12, route=13, gather=14, combine_norm=15,
                    embed=16, quant_h=17)


class Config(C.Structure):
    _fields_ = [
        ("n_layers", C.c_int32), ("d_model", C.c_int32), ("n_heads", C.c_int32),
        ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("n_experts", C.c_int32),
        ("top_k", C.c_int32), ("expert_hidden", C.c_int32), ("shared_hidden", C.c_int32),
        ("vocab", C.c_int32), ("canvas", C.c_int32), ("kv_capacity", C.c_int32),
        ("dtype", C.c_int32), ("eps", C.c_float), ("rope_theta", C.c_float),
        ("tau", C.c_double), ("h_bound", C.c_double), ("max_steps", C.c_int32),
        ("fixed_steps", C.c_int32), ("prefill_chunk", C.c_int32),
        ("lock_rule", C.c_int32), ("entropy_lock", C.c_double), ("sticky_locks", C.c_int32),
        ("temperature", C.c_float), ("commit_reuse_kv", C.c_int32), ("batch", C.c_int32),
        ("lm_head_e4m3", C.c_int32),
    ]


class LayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in
                ("attn_norm", "wqkv", "wo", "ffn_norm", "wr", "w_gu", "w_d", "ws_gu", "ws_d",
                 "w_gu_scale", "w_d_scale", "ws_gu_scale", "ws_d_scale",
                 "w_gu_sf", "w_d_sf", "ws_gu_sf", "ws_d_sf")]


class Weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("final_norm", C.c_void_p),
                ("layers", C.POINTER(LayerWeights)), ("head_codes", C.c_void_p),
                ("head_scale", C.c_void_p)]


_P = C.c_void_p
_I = C.c_int32
_SZ = C.c_size_t
_PROTOS = {
    "dg_workspace_bytes": (C.c_int, [C.POINTER(Config), C.POINTER(_SZ), C.POINTER(_SZ)]),
    "dg_create": (C.c_int, [C.POINTER(Config), C.POINTER(Weights), _P, _P, _P, C.POINTER(_P)]),
    "dg_destroy": (None, [_P]),
    "dg_kv_length": (C.c_int32, [_P]),
    "dg_kv_truncate": (C.c_int, [_P, _I]),
    "dg_kv_append": (C.c_int, [_P, _P, _I, _P]),
    "dg_canvas_init": (C.c_int, [_P, C.c_uint64, C.c_uint32, _P]),
    "dg_reset_block": (C.c_int, [_P, _P]),
    "dg_denoise_step": (C.c_int, [_P, C.c_uint32, _P]),
    "dg_sample_update": (C.c_int, [_P, C.c_uint32, _P]),
    "dg_commit_block": (C.c_int, [_P, _P, _P, _P]),
    "dg_get_buffers": (C.c_int, [_P, C.POINTER(_P), C.POINTER(_P), C.POINTER(_P), C.POINTER(_P),
                                 C.POINTER(_P)]),
    "dg_check_device_status": (C.c_int, [_P, _P]),
    "dg_sampler_workspace_bytes": (C.c_int, [_I, _I, C.POINTER(_SZ)]),
    "dg_sampler_reset": (C.c_int, [_I, _I, _P, _P, _P]),
    "dg_sampler_step": (C.c_int, [_P, _I, _I, _I, C.c_uint64, C.c_uint32, C.c_uint32, C.c_double,
                                  C.c_double, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "dg_sampler_step_static": (C.c_int, [_P, _I, _I, _I, C.c_uint64, C.c_uint32, C.c_uint32,
                                         C.c_double, C.c_double, _I, _I, _P, _P, _P, _P, _P, _P]),
    "dg_attention_workspace_bytes": (C.c_int, [_I, _I, _I, _I, C.POINTER(_SZ)]),
    "dg_canvas_attention": (C.c_int, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, C.c_float, _P,
                                      _SZ, _P]),
    "dg_moe_workspace_bytes": (C.c_int, [_I, _I, _I, _I, _I, _I, C.POINTER(_SZ)]),
    "dg_moe_ffn": (C.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                             _P, _SZ, _P]),
    "dg_moe_ffn_e4m3": (C.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I,
                                  _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "dg_quantize_e4m3": (C.c_int, [_P, _I, _I, C.c_int64, _P, C.c_int64, _P, _P]),
    "dg_quantize_nvfp4": (C.c_int, [_P, _I, _I, C.c_int64, _P, C.c_int64, _P, _P, _P]),
    "dg_moe_ffn_nvfp4": (C.c_int, [_P] * 19 + [_I] * 6 + [_P, _SZ, _P]),
    "dg_debug_logits": (C.c_int, [_P, _P, _P]),
    "dg_debug_layer": (C.c_int, [_P, _I, _P, _P, _I, _I, _P]),
    "dg_debug_hidden": (C.c_int, [_P, C.POINTER(_P)]),
    "dg_debug_layer_part": (C.c_int, [_P, _I, _I, _P, _P, _I, _I, _P]),
    "dg_debug_tensors": (C.c_int, [_P, C.POINTER(_P), C.POINTER(_P), C.POINTER(_P)]),
    "dg_debug_routing": (C.c_int, [_P, C.POINTER(_P), C.POINTER(_P), C.POINTER(_P)]),
    "dg_launch_count": (C.c_uint64, []),
    "dg_profile_kernel": (C.c_int, [_I, _I]),
    "dg_profile_read": (C.c_int32, [C.POINTER(C.c_float), _I]),
    "dg_last_error": (C.c_char_p, []),
    "dg_version": (C.c_char_p, []),
}

_lib = None


def lib():
    """Load libdg.so (raises if it has not been built: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdg.so not found at {LIB_PATH}; build it with "
                               "`python -m block_text_diffusion_dg_b200.build`")
        h = C.CDLL(LIB_PATH)
        for name, (res, args) in _PROTOS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def check(rc, what):
    if rc != DG_OK:
        msg = lib().dg_last_error().decode(errors="replace")
        raise RuntimeError(f"{what}: {DG_ERR.get(rc, rc)}: {msg}")
