"""The C-ABI library loads, exports every declared entry point, and checks arguments on the host.

No call here needs a GPU: only workspace sizing and argument validation, which run before any
CUDA call.
"""
import ctypes as C
import os
import re

import pytest

from block_text_diffusion_dg_b200 import build as dg_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    dg_build.build()
    from block_text_diffusion_dg_b200 import _lib
    return _lib


def _declared():
    src = open(os.path.join(ROOT, "include", "dg.h")).read()
    return sorted(set(re.findall(r"^DG_API\s+[\w\s\*]*?\b(dg_\w+)\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 20
    h = C.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(h, n), n
    assert set(names) == set(L._PROTOS), "binding and header disagree"


def _cfg(L, shape, **kw):
    from block_text_diffusion_dg_b200.api import make_config
    from dg_synth import SHAPES
    return make_config(SHAPES[shape], kv_capacity=kw.pop("kv_capacity", 8192), **kw)


@pytest.mark.parametrize("shape", ["tiny_fp32", "small_bf16", "a4b"])
def test_workspace_sizes(L, shape):
    from block_text_diffusion_dg_b200.api import workspace_bytes
    cfg = _cfg(L, shape, kv_capacity=5376)
    kv, sc = workspace_bytes(cfg)
    esz = 4 if shape == "tiny_fp32" else 2
    assert kv == 2 * cfg.n_layers * cfg.n_kv_heads * 5376 * cfg.head_dim * esz
    assert sc > cfg.canvas * cfg.d_model * 4 and sc % 256 == 0


def test_bad_configs_are_rejected(L):
    lib = L.lib()
    kv, sc = C.c_size_t(), C.c_size_t()
    for field, value, code in [("n_heads", 3, -1), ("top_k", 9, -5), ("canvas", 300, -5),
                               ("kv_capacity", 1001, -1), ("head_dim", 64, -5), ("vocab", 1000, -5),
                               ("dtype", 7, -1), ("d_model", 0, -1)]:
        cfg = _cfg(L, "small_bf16")
        setattr(cfg, field, value)
        rc = lib.dg_workspace_bytes(C.byref(cfg), C.byref(kv), C.byref(sc))
        assert rc == code, (field, rc, lib.dg_last_error())
        assert lib.dg_last_error()


def test_create_rejects_null_buffers(L):
    lib = L.lib()
    cfg = _cfg(L, "small_bf16")
    w = L.Weights()
    out = C.c_void_p()
    assert lib.dg_create(C.byref(cfg), C.byref(w), None, None, None, C.byref(out)) == -1


def test_loop_entry_points_reject_a_null_context(L):
    lib = L.lib()
    assert lib.dg_reset_block(None, None) == -1
    assert lib.dg_canvas_init(None, 0, 0, None) == -1
    assert lib.dg_denoise_step(None, 1, None) == -1
    assert lib.dg_sample_update(None, 1, None) == -1
    assert lib.dg_commit_block(None, None, None, None) == -1


def test_standalone_shape_checks(L):
    lib = L.lib()
    n = C.c_size_t()
    # a 16-byte partial and a 4-byte piece length per (row, 8192-column segment), at least
    assert lib.dg_sampler_workspace_bytes(256, 262144, C.byref(n)) == 0 and n.value >= 256 * 32 * 20
    assert lib.dg_sampler_workspace_bytes(256, 1001, C.byref(n)) == -1
    assert lib.dg_sampler_workspace_bytes(2000, 1024, C.byref(n)) == -1
    assert lib.dg_attention_workspace_bytes(16, 8, 256, 4352, C.byref(n)) == 0
    assert lib.dg_attention_workspace_bytes(16, 8, 200, 4352, C.byref(n)) == -1
    assert lib.dg_moe_workspace_bytes(256, 2816, 128, 8, 704, 2112, C.byref(n)) == 0
    assert lib.dg_moe_workspace_bytes(256, 2816, 128, 9, 704, 2112, C.byref(n)) == -1
    assert lib.dg_moe_workspace_bytes(256, 2800, 128, 8, 704, 2112, C.byref(n)) == -1
    # null pointers are caught before any device work
    assert lib.dg_canvas_attention(None, None, None, None, 16, 8, 256, 256, 4352, 4352, -1, 0.1,
                                   None, 0, None) == -1
    assert lib.dg_sampler_step(None, 0, 256, 262144, 0, 0, 1, 0.9, 0.005, 48, 0, None, None, None,
                               None, None, None, None) == -1


def test_e4m3_config_and_workspace(L):
    from block_text_diffusion_dg_b200.api import make_config, workspace_bytes
    from dg_synth import SHAPES
    c16 = make_config(SHAPES["a4b"], kv_capacity=5376)
    c8 = make_config(SHAPES["a4b"], kv_capacity=5376, experts="e4m3")
    assert c8.dtype == L.DTYPE_BF16_E4M3 and c16.dtype == L.DTYPE_BF16
    kv16, sc16 = workspace_bytes(c16)
    kv8, sc8 = workspace_bytes(c8)
    assert kv8 == kv16  # the KV cache stays bf16
    # x_perm shrinks to one byte per code at the 128-byte pitch; the e4m3 buffers are added
    assert sc8 != sc16 and sc8 % 256 == 0
    with pytest.raises(ValueError):
        make_config(SHAPES["tiny_fp32"], kv_capacity=512, experts="e4m3")
    with pytest.raises(ValueError):
        make_config(SHAPES["small_bf16"], kv_capacity=512, experts="int4")
    from block_text_diffusion_dg_b200 import e4m3_pitch
    assert [e4m3_pitch(c) for c in (16, 128, 129, 704, 2112, 2816)] == [128, 128, 256, 768, 2176,
                                                                       2816]


def test_quantiser_argument_checks(L):
    lib = L.lib()
    a = 1 << 20  # a 16-byte aligned address that is never dereferenced: checks run first
    assert lib.dg_quantize_e4m3(None, 4, 64, 64, a, 64, a, None) == -1
    assert lib.dg_quantize_e4m3(a, 4, 24, 24, a, 32, a, None) == -1      # cols % 16
    assert lib.dg_quantize_e4m3(a, 4, 64, 60, a, 64, a, None) == -1      # ld_in < cols
    assert lib.dg_quantize_e4m3(a, 4, 64, 64, a, 48, a, None) == -1      # ld_codes < cols
    assert lib.dg_quantize_e4m3(a, 4, 64, 64, a, 72, a, None) == -1      # ld_codes % 16
    assert lib.dg_quantize_e4m3(a + 8, 4, 64, 64, a, 64, a, None) == -1  # misaligned input
    assert lib.dg_quantize_e4m3(a, 4, 64, 64, a + 4, 64, a, None) == -1  # misaligned codes
    assert "ld_codes" in lib.dg_last_error().decode() or "misaligned" in lib.dg_last_error().decode()
    assert lib.dg_quantize_e4m3(a, 0, 64, 64, a, 64, a, None) == 0       # nothing to do


def test_e4m3_moe_requires_scales(L):
    lib = L.lib()
    n = C.c_size_t()
    assert lib.dg_moe_workspace_bytes(256, 2816, 128, 8, 704, 2112, C.byref(n)) == 0
    a = 1 << 20
    rc = lib.dg_moe_ffn_e4m3(a, None, a, a, None, a, a, a, a, a, a, a, None, None, None, 256, 2816,
                             128, 8, 704, 2112, a, n.value, None)
    assert rc == -1 and "scales" in lib.dg_last_error().decode()


def test_e4m3_create_requires_scales(L):
    lib = L.lib()
    cfg = _cfg(L, "small_bf16", experts="e4m3", kv_capacity=1024)
    a = 1 << 20
    layers = (L.LayerWeights * cfg.n_layers)()
    for lw in layers:
        for name in ("attn_norm", "wqkv", "wo", "ffn_norm", "wr", "w_gu", "w_d", "ws_gu", "ws_d",
                     "w_gu_scale", "w_d_scale", "ws_gu_scale", "ws_d_scale"):
            setattr(lw, name, a)
    layers[1].ws_d_scale = None
    w = L.Weights(embed=a, final_norm=a, layers=layers)
    out = C.c_void_p()
    assert lib.dg_create(C.byref(cfg), C.byref(w), a, a, None, C.byref(out)) == -1
    assert "e4m3 expert scales" in lib.dg_last_error().decode()


def test_sampler_variant_config(L):
    from block_text_diffusion_dg_b200.api import make_config, workspace_bytes
    from dg_synth import SHAPES
    cfg = make_config(SHAPES["small_bf16"], kv_capacity=1024, lock_rule="entropy_bound",
                      entropy_lock=0.1, sticky=True)
    assert (cfg.lock_rule, cfg.entropy_lock, cfg.sticky_locks) == (1, 0.1, 1)
    workspace_bytes(cfg)
    for field, value in (("entropy_lock", -1.0), ("lock_rule", 2), ("sticky_locks", 3)):
        bad = make_config(SHAPES["small_bf16"], kv_capacity=1024)
        setattr(bad, field, value)
        with pytest.raises(RuntimeError, match="INVALID_ARG"):
            workspace_bytes(bad)
    with pytest.raises(ValueError):
        make_config(SHAPES["small_bf16"], kv_capacity=1024, lock_rule="top_p")
