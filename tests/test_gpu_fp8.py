"""Parity of the e4m3 (FP8) expert format: the quantiser, the MoE operator and the model layers.

The quantiser's codes are integer decisions taken from identical bf16 inputs in binary32 on both
sides, so they are compared bit-exactly (+0 and -0 count as the same code).  The MoE and the
layers are compared against the oracle's fp8 MoE, which quantises the same bf16 weights itself.
"""
import numpy as np
import pytest
import torch

from dg_synth import SHAPES, model_weights, moe_inputs, scaled_rows, uniform_ids
from oracle import model as om
from oracle import sampler as osmp
from oracle.moe import moe_ffn_fp8 as o_moe8
from oracle.quant import encode_e4m3, quantize_matrix, quantize_rows
from tests._helpers import check_layer_parts, np64, npf32, rel_close, weights_to_np

pytestmark = pytest.mark.gpu
RTOL = 2e-2


def _same_codes(got, ref_values):
    ref = encode_e4m3(ref_values)
    got = np.asarray(got, dtype=np.uint8)
    zero = (ref & 0x7F) == 0
    return bool(np.array_equal(got[~zero], ref[~zero]) and np.all((got[zero] & 0x7F) == 0))


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 48), (37, 704), (300, 2816), (9, 4096)])
def test_quantiser_bit_exact(rows, cols):
    from block_text_diffusion_dg_b200 import quantize_e4m3
    x = scaled_rows(rows, cols, seed=rows * 131 + cols)
    codes, scales = quantize_e4m3(x.cuda())
    packed, _ = quantize_e4m3(x.cuda(), pitch=cols)
    torch.cuda.synchronize()
    q, s = quantize_rows(npf32(x))
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), s.view(np.uint32))
    c = codes.cpu().numpy()
    assert c.shape[1] == (cols + 127) // 128 * 128 and not c[:, cols:].any()
    assert _same_codes(c[:, :cols], q)
    assert np.array_equal(packed.cpu().numpy(), c[:, :cols])


def test_quantiser_rejects_bad_shapes():
    from block_text_diffusion_dg_b200 import quantize_e4m3
    with pytest.raises(RuntimeError, match="INVALID_ARG"):
        quantize_e4m3(torch.zeros(4, 24, dtype=torch.bfloat16, device="cuda"))


def _quantised(dev):
    from block_text_diffusion_dg_b200 import quantize_e4m3
    q = {}
    for name in ("w_gu", "w_d", "ws_gu", "ws_d"):
        if dev[name] is None:
            q[name] = q[name + "_scale"] = None
        else:
            q[name], q[name + "_scale"] = quantize_e4m3(dev[name])
    return q


def _case8(t, d, e, k, h, hs, seed):
    from block_text_diffusion_dg_b200 import moe_ffn_e4m3
    m = moe_inputs(t, d, e, h, hs, seed=seed)
    dev = {kk: (None if v is None else v.cuda()) for kk, v in m.items()}
    q = _quantised(dev)
    ids = torch.empty(t, k, dtype=torch.int32, device="cuda")
    wts = torch.empty(t, k, dtype=torch.float32, device="cuda")
    rl = torch.empty(t, e, dtype=torch.float32, device="cuda")
    y = moe_ffn_e4m3(dev["x"], dev["wr"], q["w_gu"], q["w_gu_scale"], q["w_d"], q["w_d_scale"], k,
                     q["ws_gu"], q["ws_gu_scale"], q["ws_d"], q["ws_d_scale"], ids=ids, weights=wts,
                     router_logits=rl)
    torch.cuda.synchronize()
    # the weights the kernels read are the oracle's quantisation of the same bf16 weights
    gq, gs = quantize_matrix(npf32(m["w_gu"][e - 1]))
    assert _same_codes(q["w_gu"][e - 1, :, :d].cpu().numpy(), gq)
    assert np.array_equal(q["w_gu_scale"][e - 1].cpu().numpy(), gs)
    shared = None if hs == 0 else (npf32(m["ws_gu"]), npf32(m["ws_d"]))
    y_ref, info = o_moe8(np64(m["x"]), npf32(m["wr"]), npf32(m["w_gu"]), npf32(m["w_d"]), k, shared)
    g_logits = rl.cpu().numpy().astype(np.float64)
    ok, worst, _ = rel_close(g_logits, info["router_logits"], 1e-4)
    assert ok, worst
    srt = -np.sort(-info["router_logits"], axis=1)
    gap = srt[:, k - 1] - srt[:, k] if k < e else np.full(t, np.inf)
    g_ids = ids.cpu().numpy()
    assert np.array_equal(g_ids[gap > 1e-3], info["ids"][gap > 1e-3])
    same = np.all(g_ids == info["ids"], axis=1)
    ok, worst, nrel = rel_close(y.cpu().numpy()[same], y_ref[same], RTOL)
    assert ok, (worst, nrel)
    assert nrel < 1e-2, nrel
    return same.mean()


@pytest.mark.parametrize("t,d,e,k,h,hs", [
    (64, 256, 8, 2, 128, 0),         # tiny, no shared expert
    (256, 512, 8, 2, 256, 384),      # the small test model's MoE
    (200, 512, 16, 4, 192, 256),     # ragged tokens; h = 192: the last 128-wide K slab half empty
    (1100, 512, 16, 4, 128, 320),    # 256-token chunks; hs = 320 ragged
    (2048, 256, 128, 8, 64, 0),      # a long pass: 16 384 routed slots, one half-empty K slab
])
def test_moe_e4m3_small(t, d, e, k, h, hs):
    assert _case8(t, d, e, k, h, hs, seed=t + d + 1) > 0.95


def test_moe_e4m3_full_size():
    # 256 tokens, d 2816, 128 experts top-8 (SiLU-GLU 704) + shared expert 2112
    assert _case8(256, 2816, 128, 8, 704, 2112, seed=0) > 0.95


def _to_cuda(w):
    def cv(t):
        return None if t is None else t.cuda()
    return dict(embed=cv(w["embed"]), final_norm=cv(w["final_norm"]),
                layers=[{k: cv(v) for k, v in lw.items()} for lw in w["layers"]])


def test_small_model_with_e4m3_experts():
    """The small bf16 model with FP8 experts: prefill, a denoise step checked layer by layer
    (teacher-forced halves against the oracle's fp8 MoE), the LM head, sampler, a commit."""
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config, quantize_experts
    shape = SHAPES["small_bf16"]
    w = model_weights("small_bf16", seed=5, norm_jitter=0.1)
    prompt = uniform_ids(shape["prompt"], shape["vocab"], seed=6)
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=2, experts="e4m3")
    wq = quantize_experts(_to_cuda(w))
    assert wq["layers"][0]["w_gu"].dtype == torch.uint8
    m = DiffusionModel(cfg, wq)
    s = SHAPES["small_bf16"]
    ocfg = om.ModelConfig(**{kk: s[kk] for kk in (
        "n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "n_experts", "top_k",
        "expert_hidden", "shared_hidden", "vocab", "canvas", "storage")}, experts="fp8")
    ow = weights_to_np(w)
    ocache = om.causal_encode(ocfg, ow, prompt.numpy(), om.KVCache())
    m.kv_append(prompt.cuda())
    m.canvas_init(3, 0)
    m.denoise_step(1)
    logits = m.debug_logits()
    m.sample_update(1)
    bufs = m.buffers()
    torch.cuda.synchronize()
    ref_logits = om.lm_head(ocfg, ow, np64(m.debug_hidden()))
    assert np.max(np.abs(np64(logits) - ref_logits)) < 3e-2
    conf, ent, amax = osmp.row_stats(np64(logits))
    assert np.array_equal(bufs["argmax"].cpu().numpy(), amax)
    canvas0 = osmp.canvas_init(3, 0, 256, shape["vocab"])
    x = np.asarray(ow["embed"], dtype=np.float64)[canvas0]
    pos = shape["prompt"] + np.arange(256)
    for l in range(cfg.n_layers):
        att, moe, frac = check_layer_parts(m, ocfg, ow["layers"][l], x, pos, ocache.k[l],
                                           ocache.v[l], l, shape["top_k"])
        assert att[0] and att[2] < 5e-3, ("attention half", l, att)
        assert moe[0] and moe[2] < 1e-2, ("moe half", l, moe)
        assert frac > 0.98, frac
        x, _, _, _ = om.layer_forward(ocfg, ow["layers"][l], x, pos, ocache.k[l], ocache.v[l],
                                      causal=False)
    m.denoise_step(2)
    m.sample_update(2)
    ids, st = m.commit_block()
    torch.cuda.synchronize()
    assert st.cpu().tolist()[:2] == [1, 2] and m.kv_length == shape["prompt"] + 256
    m.check_device_status()


def test_e4m3_model_rejects_missing_scales():
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config, quantize_experts
    shape = SHAPES["small_bf16"]
    w = quantize_experts(_to_cuda(model_weights("small_bf16", seed=7)))
    w["layers"][1]["w_d_scale"] = None
    cfg = make_config(shape, kv_capacity=512, experts="e4m3")
    with pytest.raises(RuntimeError, match="scales"):
        DiffusionModel(cfg, w)


# ---- the LM head on e4m3 operands (dg_config.lm_head_e4m3) ----------------------------------------

@pytest.mark.parametrize("batch", [1, 2])
def test_e4m3_lm_head_small_model(batch):
    """The e4m3 head's logits (dg_debug_logits: the same MMA core and scaling as the fused
    statistics) against the oracle's lm_head_fp8 on the GPU's own final hidden state; the fused
    statistics and the sampler on the GPU's logits; one and two sequences."""
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config, quantize_head
    shape = SHAPES["small_bf16"]
    v, t = shape["vocab"], shape["canvas"]
    w = model_weights("small_bf16", seed=31, norm_jitter=0.1)
    wc = quantize_head(_to_cuda(w))
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=2, head="e4m3", batch=batch)
    m = DiffusionModel(cfg, wc)
    prompts = torch.stack([uniform_ids(96, v, seed=32 + b) for b in range(batch)])
    m.kv_append(prompts.cuda())
    m.canvas_init(7, 0)
    m.denoise_step(1)
    logits = np64(m.debug_logits())
    m.sample_update(1)
    bufs = m.buffers()
    torch.cuda.synchronize()
    x_final = np64(m.debug_hidden())
    ocfg = om.ModelConfig(**{k: shape[k] for k in (
        "n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "n_experts", "top_k",
        "expert_hidden", "shared_hidden", "vocab", "canvas", "storage")}, head="fp8")
    ow = weights_to_np(w)
    ref = om.lm_head(ocfg, ow, x_final)
    err = np.max(np.abs(logits - ref))
    assert err < 3e-2, err
    # the quantisation acts: the bf16 head differs by more than the comparison's noise
    ref16 = om.lm_head(om.ModelConfig(**{**ocfg.__dict__, "head": "bf16"}), ow, x_final)
    assert np.max(np.abs(ref16 - ref)) > 5 * err
    conf, ent, amax = osmp.row_stats(logits)
    assert np.array_equal(bufs["argmax"].cpu().numpy(), amax)
    assert np.max(np.abs(bufs["entropy"].cpu().numpy() - ent)) < 1e-5
    g_canvas = bufs["canvas"].cpu().numpy().reshape(batch, t)
    for b in range(batch):
        rows = slice(b * t, (b + 1) * t)
        nxt, _ = osmp.sample_update(conf[rows], amax[rows], 7 + b, 0, 1, v)
        clear = np.abs(conf[rows] - 0.9) > 1e-4
        assert np.array_equal(g_canvas[b][clear], nxt[clear])
    m.commit_block()
    m.check_device_status()
    m.close()


def test_e4m3_lm_head_full_vocabulary():
    """One decoder layer of the full model's shapes with the 262,144-entry tied head in e4m3: the
    head's codes bit-exact for sampled vocabulary rows, the logits of sampled (row, vocabulary)
    entries against the oracle (tokens quantised from the GPU's own final hidden state), the
    fused statistics of all 256 rows on the GPU's logits."""
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config, quantize_head
    shape = dict(SHAPES["a4b"], n_layers=1)
    v, d = shape["vocab"], shape["d_model"]
    w = model_weights(shape, seed=41, device="cuda")
    wc = quantize_head(w)
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=1, head="e4m3")
    m = DiffusionModel(cfg, wc)
    m.kv_append(uniform_ids(128, v, seed=42).cuda())
    m.canvas_init(43, 0)
    m.denoise_step(1)
    logits = m.debug_logits()
    m.sample_update(1)
    bufs = m.buffers()
    torch.cuda.synchronize()
    rng = np.random.default_rng(44)
    vrows = np.sort(rng.choice(v, 2048, replace=False))
    emb = npf32(w["embed"][torch.from_numpy(vrows).cuda()])
    eq, es = quantize_rows(emb)
    codes = wc["head_codes"][torch.from_numpy(vrows).cuda()].cpu().numpy()[:, :d]
    assert _same_codes(codes, eq)
    assert np.array_equal(wc["head_scale"][torch.from_numpy(vrows).cuda()].cpu().numpy(), es)
    x_final = np64(m.debug_hidden())
    rows = np.arange(0, 256, 17)
    xf = om.rmsnorm(x_final[rows], npf32(w["final_norm"]), 1e-6)
    from oracle.numerics import round_bf16
    ref = om.lm_head_fp8(round_bf16(xf).astype(np.float64), emb)
    got = np64(logits[torch.from_numpy(rows).cuda()][:, torch.from_numpy(vrows).cuda()])
    assert np.max(np.abs(got - ref)) < 3e-2
    conf, ent, amax = osmp.row_stats(np64(logits))
    assert np.array_equal(bufs["argmax"].cpu().numpy(), amax)
    assert np.max(np.abs(bufs["entropy"].cpu().numpy() - ent)) < 1e-5
    m.check_device_status()
    m.close()
