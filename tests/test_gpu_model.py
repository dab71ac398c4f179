"""End-to-end parity of the model context: prefill, denoise steps, sampler, commit.

Two models: the all-fp32 two-layer model (1e-4 tolerance, every step compared) and a small
bf16 model with the production kernels' tile shapes (2e-2 tolerance, teacher-forced layers,
LM-head statistics on identical logits, ragged prefill chunk, two committed blocks).
"""
import numpy as np
import pytest
import torch

from dg_synth import SHAPES, model_weights, uniform_ids
from oracle import model as om
from oracle import sampler as osmp
from oracle.numerics import round_bf16
from tests._helpers import (check_layer_parts, kv_tokens_close, np64, rel_close, router_gaps,
                            weights_to_np)

pytestmark = pytest.mark.gpu


def _ocfg(shape, **kw):
    s = SHAPES[shape]
    return om.ModelConfig(**{k: s[k] for k in ("n_layers", "d_model", "n_heads", "n_kv_heads",
                                               "head_dim", "n_experts", "top_k", "expert_hidden",
                                               "shared_hidden", "vocab", "canvas", "storage")}, **kw)


def _to_cuda(w):
    def cv(t):
        return None if t is None else t.cuda()
    return dict(embed=cv(w["embed"]), final_norm=cv(w["final_norm"]),
                layers=[{k: cv(v) for k, v in lw.items()} for lw in w["layers"]])


def _kv_views(m, cfg):
    """K [L, Hkv, cap, hd] and V^T [L, Hkv, hd, cap] views of the context's cache."""
    dt = torch.float32 if cfg.dtype == 1 else torch.bfloat16
    kv = m.kv.view(dt)
    half = kv.numel() // 2
    shp = (cfg.n_layers, cfg.n_kv_heads, cfg.kv_capacity, cfg.head_dim)
    return kv[:half].view(shp), kv[half:].view(cfg.n_layers, cfg.n_kv_heads, cfg.head_dim,
                                               cfg.kv_capacity)


def _argmax_guarded(logits_ref, got, margin):
    srt = -np.sort(-logits_ref, axis=1)[:, :2]
    clear = (srt[:, 0] - srt[:, 1]) > margin
    ref = np.argmax(logits_ref, axis=1)
    return np.array_equal(got[clear], ref[clear]), clear.mean()


def test_tiny_fp32_end_to_end():
    """2-layer fp32 model, 128-token prompt, one canvas, 16 fixed steps, seed 0."""
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config
    shape = SHAPES["tiny_fp32"]
    w = model_weights("tiny_fp32", seed=0)
    prompt = uniform_ids(shape["prompt"], shape["vocab"], seed=0)
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=16)
    m = DiffusionModel(cfg, _to_cuda(w))
    ocfg, ow = _ocfg("tiny_fp32"), weights_to_np(w)
    _, blocks, ocache = om.decode(ocfg, ow, prompt.numpy(), 1, seed=0, fixed_steps=16)
    ref_steps = blocks[0]["steps"]
    m.kv_append(prompt.cuda())
    k_gpu, vt_gpu = _kv_views(m, cfg)
    torch.cuda.synchronize()
    for l in range(cfg.n_layers):
        ok, worst, _ = rel_close(np64(k_gpu[l, :, :128]), ocache.k[l][:, :128], 1e-4)
        assert ok, ("prefill K", l, worst)
        ok, worst, _ = rel_close(np64(vt_gpu[l, :, :, :128]).transpose(0, 2, 1), ocache.v[l][:, :128], 1e-4)
        assert ok, ("prefill V", l, worst)
    m.canvas_init(0, 0)
    bufs = m.buffers()
    torch.cuda.synchronize()
    assert np.array_equal(bufs["canvas"].cpu().numpy(), ref_steps[0]["canvas_in"])
    for t in range(1, 17):
        m.denoise_step(t)
        if t == 16:
            logits = m.debug_logits()
        m.sample_update(t)
        torch.cuda.synchronize()
        r = ref_steps[t - 1]
        assert np.array_equal(bufs["canvas"].cpu().numpy(), r["canvas_out"]), t
        assert np.max(np.abs(bufs["entropy"].cpu().numpy() - r["entropy"])) < 1e-5, t
        ok, frac = _argmax_guarded(
            om.denoise_logits(ocfg, ow, r["canvas_in"], _cache_prefix(ocache, 128)),
            bufs["argmax"].cpu().numpy(), 1e-4) if t in (1, 16) else (True, 1.0)
        assert ok and frac > 0.9, t
    ref_logits = om.denoise_logits(ocfg, ow, ref_steps[15]["canvas_in"], _cache_prefix(ocache, 128))
    ok, worst, _ = rel_close(np64(logits), ref_logits, 1e-4)
    assert ok, worst
    ids, st = m.commit_block()
    torch.cuda.synchronize()
    assert st.cpu().tolist()[:4] == [1, 16, 0, 16]
    assert np.array_equal(ids.cpu().numpy(), bufs["argmax"].cpu().numpy())
    assert m.kv_length == 128 + 256


def _cache_prefix(cache, n):
    c = om.KVCache()
    c.k = [k[:, :n] for k in cache.k]
    c.v = [v[:, :n] for v in cache.v]
    return c


def test_small_bf16_prefill_denoise_commit():
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config
    shape = SHAPES["small_bf16"]
    k_top = shape["top_k"]
    w = model_weights("small_bf16", seed=1, norm_jitter=0.1)
    prompt = uniform_ids(shape["prompt"], shape["vocab"], seed=2)  # 320 = 256 + ragged 64
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=3)
    m = DiffusionModel(cfg, _to_cuda(w))
    ocfg, ow = _ocfg("small_bf16"), weights_to_np(w)
    ocache = om.causal_encode(ocfg, ow, prompt.numpy(), om.KVCache())
    gaps = router_gaps(ocfg, ow, prompt.numpy(), np.arange(320), om.KVCache())
    m.kv_append(prompt.cuda())
    assert m.kv_length == 320
    k_gpu, vt_gpu = _kv_views(m, cfg)
    torch.cuda.synchronize()
    for l in range(cfg.n_layers):
        ok, bad, _ = kv_tokens_close(np64(k_gpu[l, :, :320]), ocache.k[l], gaps, l, 2e-2)
        assert ok, ("prefill K", l, bad)
        ok, bad, _ = kv_tokens_close(np64(vt_gpu[l, :, :, :320]).transpose(0, 2, 1), ocache.v[l],
                                      gaps, l, 2e-2)
        assert ok, ("prefill V", l, bad)
    # one denoise step
    m.canvas_init(11, 0)
    m.denoise_step(1)
    logits = m.debug_logits()
    m.sample_update(1)
    bufs = m.buffers()
    torch.cuda.synchronize()
    x_final = np64(m.debug_hidden())
    canvas0 = osmp.canvas_init(11, 0, 256, shape["vocab"])
    # the LM head on the GPU's own final hidden state
    ref_logits = om.lm_head(ocfg, ow, x_final)
    err = np.max(np.abs(np64(logits) - ref_logits))
    assert err < 3e-2, err
    # statistics and argmax of the fused LM head equal the oracle's on the GPU's own logits
    conf, ent, amax = osmp.row_stats(np64(logits))
    assert np.array_equal(bufs["argmax"].cpu().numpy(), amax)
    assert np.max(np.abs(bufs["entropy"].cpu().numpy() - ent)) < 1e-5
    nxt, _ = osmp.sample_update(conf, amax, 11, 0, 1, shape["vocab"])
    assert np.array_equal(bufs["canvas"].cpu().numpy(), nxt)
    # teacher-forced layers, half by half from identical inputs (see check_layer_parts)
    x = np.asarray(ow["embed"], dtype=np.float64)[canvas0]
    pos = 320 + np.arange(256)
    for l in range(cfg.n_layers):
        att, moe, frac = check_layer_parts(m, ocfg, ow["layers"][l], x, pos, ocache.k[l],
                                           ocache.v[l], l, k_top)
        assert att[0] and att[2] < 5e-3, ("attention half", l, att)
        assert moe[0] and moe[2] < 5e-3, ("moe half", l, moe)
        assert frac > 0.98, frac
        x, _, _, _ = om.layer_forward(ocfg, ow["layers"][l], x, pos, ocache.k[l], ocache.v[l],
                                      causal=False)
    # finish the block, commit it, check the committed K slots against a teacher-forced commit
    for t in (2, 3):
        m.denoise_step(t)
        m.sample_update(t)
    ids, st = m.commit_block()
    torch.cuda.synchronize()
    ids_np = ids.cpu().numpy()
    assert st.cpu().tolist()[:2] == [1, 3]
    assert m.kv_length == 320 + 256
    gaps = router_gaps(ocfg, ow, ids_np, 320 + np.arange(256), ocache)
    om.causal_encode(ocfg, ow, ids_np, ocache)
    k_gpu, vt_gpu = _kv_views(m, cfg)
    for l in range(cfg.n_layers):
        ok, bad, _ = kv_tokens_close(np64(k_gpu[l, :, 320:576]), ocache.k[l][:, 320:576], gaps, l,
                                      2e-2)
        assert ok, ("commit K", l, bad)
        ok, bad, _ = kv_tokens_close(np64(vt_gpu[l, :, :, 320:576]).transpose(0, 2, 1),
                                      ocache.v[l][:, 320:576], gaps, l, 2e-2)
        assert ok, ("commit V", l, bad)
    # second block runs against the longer history
    m.canvas_init(11, 1)
    for t in (1, 2, 3):
        m.denoise_step(t)
        m.sample_update(t)
    ids2, st2 = m.commit_block()
    torch.cuda.synchronize()
    assert st2.cpu().tolist()[:2] == [1, 3] and m.kv_length == 320 + 512
    m.check_device_status()


def test_small_bf16_prefill_in_large_chunks():
    """The prompt encoded in 512-token passes (the last one ragged) gives the cache the oracle's
    chunk-invariant causal encode gives, and a denoise step on top of it (query buffer sized for
    the larger pass) matches the oracle layer by layer."""
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config
    shape = SHAPES["small_bf16"]
    w = model_weights("small_bf16", seed=3, norm_jitter=0.1)
    prompt = uniform_ids(640, shape["vocab"], seed=4)  # 512 + ragged 128
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=2, prefill_chunk=512)
    m = DiffusionModel(cfg, _to_cuda(w))
    ocfg, ow = _ocfg("small_bf16"), weights_to_np(w)
    ocache = om.causal_encode(ocfg, ow, prompt.numpy(), om.KVCache())
    gaps = router_gaps(ocfg, ow, prompt.numpy(), np.arange(640), om.KVCache())
    m.kv_append(prompt.cuda())
    assert m.kv_length == 640
    k_gpu, vt_gpu = _kv_views(m, cfg)
    torch.cuda.synchronize()
    for l in range(cfg.n_layers):
        ok, bad, _ = kv_tokens_close(np64(k_gpu[l, :, :640]), ocache.k[l], gaps, l, 2e-2)
        assert ok, ("prefill K", l, bad)
        ok, bad, _ = kv_tokens_close(np64(vt_gpu[l, :, :, :640]).transpose(0, 2, 1), ocache.v[l],
                                      gaps, l, 2e-2)
        assert ok, ("prefill V", l, bad)
    m.canvas_init(5, 0)
    m.denoise_step(1)
    m.sample_update(1)
    torch.cuda.synchronize()
    canvas0 = osmp.canvas_init(5, 0, 256, shape["vocab"])
    x = np.asarray(ow["embed"], dtype=np.float64)[canvas0]
    att, moe, frac = check_layer_parts(m, ocfg, ow["layers"][0], x, 640 + np.arange(256),
                                       ocache.k[0], ocache.v[0], 0, shape["top_k"])
    assert att[0] and att[2] < 5e-3, ("attention half", att)
    assert moe[0] and moe[2] < 5e-3, ("moe half", moe)
    m.check_device_status()
