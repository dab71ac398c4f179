"""Parity of the NVFP4 expert format: the quantiser, the MoE operator and the model layers.

Codes, block scales and row scales are integer / binary32 decisions taken from identical bf16
inputs, so they are compared exactly (+0 and -0 count as one code).  The MoE and the layers are
compared against the oracle's NVFP4 MoE, which quantises the same bf16 weights itself.
"""
import numpy as np
import pytest
import torch

from dg_synth import SHAPES, model_weights, moe_inputs, scaled_rows, uniform_ids
from oracle import model as om
from oracle.moe import moe_ffn_nvfp4 as o_moe4
from oracle.quant import encode_e2m1, encode_e4m3, quantize_nvfp4_rows
from tests._helpers import check_layer_parts, np64, npf32, rel_close, weights_to_np

pytestmark = pytest.mark.gpu


def _unpack_codes(codes, cols):
    """[rows, pitch] bytes -> [rows, cols] e2m1 codes (low nibble = even column)."""
    b = np.asarray(codes, dtype=np.uint8)[:, :cols // 2]
    out = np.empty((b.shape[0], cols), dtype=np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def _block_scales(atoms, rows, cols):
    """[tiles, 4 ceil(cols / 256), 512] atoms -> [rows, cols / 16] scale codes."""
    a = np.asarray(atoms, dtype=np.uint8)
    out = np.empty((rows, cols // 16), dtype=np.uint8)
    r = np.arange(rows)
    for blk in range(cols // 16):
        g, b = blk // 4, blk % 4
        out[:, blk] = a[r // 128, g, (r % 128 % 32) * 16 + (r % 128 // 32) * 4 + b]
    return out


def _same_e2m1(got, ref_values):
    ref = encode_e2m1(ref_values)
    zero = (ref & 0x7) == 0
    return bool(np.array_equal(got[~zero], ref[~zero]) and np.all((got[zero] & 0x7) == 0))


@pytest.mark.parametrize("rows,cols", [(1, 64), (3, 192), (130, 704), (300, 2816)])
def test_nvfp4_quantiser_bit_exact(rows, cols):
    from block_text_diffusion_dg_b200 import quantize_nvfp4
    x = scaled_rows(rows, cols, seed=rows * 7 + cols)
    codes, sf, g = quantize_nvfp4(x.cuda())
    torch.cuda.synchronize()
    q, sb, g_ref = quantize_nvfp4_rows(npf32(x))
    assert np.array_equal(g.cpu().numpy().view(np.uint32), g_ref.view(np.uint32))
    assert _same_e2m1(_unpack_codes(codes.cpu().numpy(), cols), q)
    assert np.array_equal(_block_scales(sf.cpu().numpy(), rows, cols), encode_e4m3(sb))
    assert not codes.cpu().numpy()[:, cols // 2:].any()


def _case4(t, d, e, k, h, hs, seed):
    from block_text_diffusion_dg_b200 import moe_ffn_nvfp4, quantize_nvfp4
    m = moe_inputs(t, d, e, h, hs, seed=seed)
    dev = {kk: (None if v is None else v.cuda()) for kk, v in m.items()}
    q = {n: (None if dev[n] is None else quantize_nvfp4(dev[n])) for n in
         ("w_gu", "w_d", "ws_gu", "ws_d")}
    ids = torch.empty(t, k, dtype=torch.int32, device="cuda")
    rl = torch.empty(t, e, dtype=torch.float32, device="cuda")
    y = moe_ffn_nvfp4(dev["x"], dev["wr"], q["w_gu"], q["w_d"], k, q["ws_gu"], q["ws_d"], ids=ids,
                      router_logits=rl)
    torch.cuda.synchronize()
    shared = None if hs == 0 else (npf32(m["ws_gu"]), npf32(m["ws_d"]))
    y_ref, info = o_moe4(np64(m["x"]), npf32(m["wr"]), npf32(m["w_gu"]), npf32(m["w_d"]), k, shared)
    srt = -np.sort(-info["router_logits"], axis=1)
    gap = srt[:, k - 1] - srt[:, k] if k < e else np.full(t, np.inf)
    g_ids = ids.cpu().numpy()
    assert np.array_equal(g_ids[gap > 1e-3], info["ids"][gap > 1e-3])
    same = np.all(g_ids == info["ids"], axis=1)
    # 4-bit h: a code step on either side of a bf16 rounding difference moves an element by up
    # to a third, so the elementwise bound is wider than the bf16 one
    ok, worst, nrel = rel_close(y.cpu().numpy()[same], y_ref[same], 6e-2)
    assert ok, (worst, nrel)
    assert nrel < 2e-2, nrel
    return same.mean()


@pytest.mark.parametrize("t,d,e,k,h,hs", [
    (64, 256, 8, 2, 128, 0),
    (256, 512, 8, 2, 256, 384),
    (200, 512, 16, 4, 192, 256),
    (1100, 512, 16, 4, 128, 320),
])
def test_moe_nvfp4_small(t, d, e, k, h, hs):
    assert _case4(t, d, e, k, h, hs, seed=t + d + 2) > 0.95


def test_moe_nvfp4_full_size():
    assert _case4(256, 2816, 128, 8, 704, 2112, seed=0) > 0.95


def _to_cuda(w):
    def cv(t):
        return None if t is None else t.cuda()
    return dict(embed=cv(w["embed"]), final_norm=cv(w["final_norm"]),
                layers=[{k: cv(v) for k, v in lw.items()} for lw in w["layers"]])


def test_small_model_with_nvfp4_experts():
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config, quantize_experts
    shape = SHAPES["small_bf16"]
    w = model_weights("small_bf16", seed=9, norm_jitter=0.1)
    prompt = uniform_ids(shape["prompt"], shape["vocab"], seed=10)
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=2, experts="nvfp4")
    m = DiffusionModel(cfg, quantize_experts(_to_cuda(w), fmt="nvfp4"))
    s = SHAPES["small_bf16"]
    ocfg = om.ModelConfig(**{kk: s[kk] for kk in (
        "n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "n_experts", "top_k",
        "expert_hidden", "shared_hidden", "vocab", "canvas", "storage")}, experts="nvfp4")
    ow = weights_to_np(w)
    ocache = om.causal_encode(ocfg, ow, prompt.numpy(), om.KVCache())
    m.kv_append(prompt.cuda())
    m.canvas_init(3, 0)
    m.denoise_step(1)
    m.sample_update(1)
    torch.cuda.synchronize()
    from oracle import sampler as osmp
    canvas0 = osmp.canvas_init(3, 0, 256, shape["vocab"])
    x = np.asarray(ow["embed"], dtype=np.float64)[canvas0]
    pos = shape["prompt"] + np.arange(256)
    for l in range(cfg.n_layers):
        att, moe, frac = check_layer_parts(m, ocfg, ow["layers"][l], x, pos, ocache.k[l],
                                           ocache.v[l], l, shape["top_k"], rtol=6e-2)
        assert att[0], ("attention half", l, att)
        assert moe[0] and moe[2] < 2e-2, ("moe half", l, moe)
        assert frac > 0.95, frac
        x, _, _, _ = om.layer_forward(ocfg, ow["layers"][l], x, pos, ocache.k[l], ocache.v[l],
                                      causal=False)
    ids, st = m.commit_block()
    torch.cuda.synchronize()
    m.check_device_status()
