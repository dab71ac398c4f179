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
