"""Small-batch canvases: B sequences decoded in lockstep by one context (dg_config.batch).

The pages say the method's advantage is strongest at small-to-medium batch on one accelerator
(aitoday.skyai.vn, serving paragraph); B canvases per step share every weight stream of the
denoise forward.  The oracle's reading (oracle.model.decode_batch): each sequence is the
single-sequence decode of its own prompt with Philox key seed + b, and lockstep changes nothing
because a stopped canvas is frozen.  Checked here:

  * a two-layer bf16 model with 3 sequences (ragged 320-token prompts): every sequence's prefill
    K/V against the oracle (router near-ties excused as in the single-sequence tests), each canvas
    the Philox stream of its own key, the LM-head statistics of all 768 rows on the GPU's logits,
    each sequence's lock / re-noise decisions, both halves of layer 0 teacher-forced over the 768
    batched tokens against the oracle per sequence, and the committed blocks' K/V;
  * the adaptive stop per sequence: a model whose attention and expert outputs are zero, with the
    final-norm weights ramped so that sequences 1 and 2 stop at step 3 and sequences 0 and 3 at
    step 4: the stopped canvases stay frozen while the others run, and every step after the last
    stop is a no-op.
"""
import numpy as np
import pytest
import torch

from dg_synth import SHAPES, model_weights, uniform_ids
from oracle import model as om
from oracle import sampler as osmp
from oracle.philox import uniform_ids as uniform_ids_np
from tests._helpers import (NEAR_TIE, kv_tokens_close, np64, rel_close, router_gaps,
                            weights_to_np)

pytestmark = pytest.mark.gpu
RTOL = 2e-2


def _to_cuda(w):
    def cv(t):
        return None if t is None else t.cuda()
    return dict(embed=cv(w["embed"]), final_norm=cv(w["final_norm"]),
                layers=[{k: cv(v) for k, v in lw.items()} for lw in w["layers"]])


def _ocfg(shape, **kw):
    return om.ModelConfig(**{k: shape[k] for k in (
        "n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "n_experts", "top_k",
        "expert_hidden", "shared_hidden", "vocab", "canvas", "storage")}, **kw)


def _kv(m, cfg, nb):
    """K [B, L, Hkv, cap, hd] and V^T [B, L, Hkv, hd, cap] of a batched context."""
    kv = m.kv.view(torch.bfloat16)
    half = kv.numel() // 2
    k = kv[:half].view(nb, cfg.n_layers, cfg.n_kv_heads, cfg.kv_capacity, cfg.head_dim)
    vt = kv[half:].view(nb, cfg.n_layers, cfg.n_kv_heads, cfg.head_dim, cfg.kv_capacity)
    return k, vt


def test_batched_decode_matches_each_sequence():
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config
    shape = SHAPES["small_bf16"]
    nb, t, v, k_top = 3, shape["canvas"], shape["vocab"], shape["top_k"]
    wt = model_weights("small_bf16", seed=71, norm_jitter=0.1)
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=2, batch=nb)
    m = DiffusionModel(cfg, _to_cuda(wt))
    prompts = torch.stack([uniform_ids(320, v, seed=72 + b) for b in range(nb)])
    m.kv_append(prompts.cuda())
    assert m.kv_length == 320
    ocfg, ow = _ocfg(shape), weights_to_np(wt)
    k_gpu, vt_gpu = _kv(m, cfg, nb)
    torch.cuda.synchronize()
    caches = []
    for b in range(nb):
        ids = prompts[b].numpy()
        cache = om.causal_encode(ocfg, ow, ids, om.KVCache())
        gaps = router_gaps(ocfg, ow, ids, np.arange(320), om.KVCache())
        for l in range(cfg.n_layers):
            ok, bad, _ = kv_tokens_close(np64(k_gpu[b, l, :, :320]), cache.k[l], gaps, l, RTOL)
            assert ok, ("prefill K", b, l, bad)
            ok, bad, _ = kv_tokens_close(np64(vt_gpu[b, l, :, :, :320]).transpose(0, 2, 1),
                                         cache.v[l], gaps, l, RTOL)
            assert ok, ("prefill V", b, l, bad)
        caches.append(cache)
    seed = 74
    m.canvas_init(seed, 0)
    bufs = m.buffers()
    torch.cuda.synchronize()
    canvas0 = bufs["canvas"].cpu().numpy().astype(np.int64).reshape(nb, t)
    for b in range(nb):
        assert np.array_equal(canvas0[b], osmp.canvas_init(seed + b, 0, t, v)), b
    m.denoise_step(1)
    logits = np64(m.debug_logits())
    m.sample_update(1)
    torch.cuda.synchronize()
    conf, ent, amax = osmp.row_stats(logits)
    assert np.array_equal(bufs["argmax"].cpu().numpy(), amax)
    assert np.max(np.abs(bufs["entropy"].cpu().numpy() - ent)) < 1e-5
    g_canvas = bufs["canvas"].cpu().numpy().astype(np.int64).reshape(nb, t)
    for b in range(nb):
        rows = slice(b * t, (b + 1) * t)
        nxt, _ = osmp.sample_update(conf[rows], amax[rows], seed + b, 0, 1, v)
        clear = np.abs(conf[rows] - 0.9) > 1e-4
        assert np.array_equal(g_canvas[b][clear], nxt[clear]), b
    st = bufs["state"].cpu().numpy()
    assert st.shape == (nb, 16) and np.all(st[:, 3] == 1) and np.all(st[:, 0] == 0)
    # layer 0 teacher-forced over the 768 batched tokens, half by half, per sequence
    pos = 320 + np.arange(t)
    x_in = np.concatenate([np.asarray(ow["embed"], dtype=np.float64)[canvas0[b]] for b in range(nb)])
    x1_gpu = m.debug_layer_part(0, 0, torch.from_numpy(x_in.astype(np.float32)).cuda(), False)
    x1 = np64(x1_gpu)
    x2_gpu = m.debug_layer_part(0, 1, x1_gpu.contiguous(), False)
    ids_g, _, _ = m.debug_routing(n=nb * t)
    torch.cuda.synchronize()
    x2 = np64(x2_gpu)
    ids_g = ids_g.cpu().numpy()
    for b in range(nb):
        rows = slice(b * t, (b + 1) * t)
        ref1, _, _, _ = om.attention_block(ocfg, ow["layers"][0], x_in[rows], pos,
                                           caches[b].k[0], caches[b].v[0], causal=False)
        ok, worst, nrel = rel_close(x1[rows], ref1, RTOL)
        assert ok and nrel < 5e-3, ("attention half", b, worst, nrel)
        ref2, info = om.moe_block(ocfg, ow["layers"][0], x1[rows])
        match = np.all(np.sort(ids_g[rows], 1) == np.sort(info["moe"]["ids"], 1), axis=1)
        srt = -np.sort(-info["moe"]["router_logits"], axis=1)
        gap = srt[:, k_top - 1] - srt[:, k_top]
        assert np.all(gap[~match] < NEAR_TIE), ("routing away from a near-tie", b)
        ok, worst, nrel = rel_close(x2[rows][match], ref2[match], RTOL)
        assert ok and nrel < 5e-3, ("moe half", b, worst, nrel)
    # finish the block, commit every sequence, check the committed K/V per sequence
    m.denoise_step(2)
    m.sample_update(2)
    ids, states = m.commit_block()
    torch.cuda.synchronize()
    assert m.kv_length == 320 + t
    assert states.shape == (nb, 16) and np.all(states.cpu().numpy()[:, :2] == [1, 2])
    ids_np = ids.cpu().numpy().reshape(nb, t)
    k_gpu, vt_gpu = _kv(m, cfg, nb)
    for b in range(nb):
        gaps = router_gaps(ocfg, ow, ids_np[b], 320 + np.arange(t), caches[b])
        om.causal_encode(ocfg, ow, ids_np[b], caches[b])
        for l in range(cfg.n_layers):
            ok, bad, _ = kv_tokens_close(np64(k_gpu[b, l, :, 320:320 + t]), caches[b].k[l][:, 320:],
                                         gaps, l, RTOL)
            assert ok, ("commit K", b, l, bad)
    # the next block runs on the longer caches
    m.canvas_init(seed, 1)
    m.denoise_step(1)
    m.sample_update(1)
    m.check_device_status()
    m.close()


def test_batched_adaptive_stop_freezes_stopped_canvases():
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config
    shape = SHAPES["small_bf16"]
    nb, t, v, tau = 4, shape["canvas"], shape["vocab"], 0.9
    wc = model_weights("small_bf16", seed=61)
    for lw in wc["layers"]:  # attention and MoE contribute nothing: x stays the embedding
        for key in ("wo", "w_d", "ws_d"):
            lw[key] = torch.zeros_like(lw[key])
    w = _to_cuda(wc)
    base = w["final_norm"].clone()
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=0, max_steps=48, tau=tau, batch=nb)
    m = DiffusionModel(cfg, w)
    m.kv_append(torch.stack([uniform_ids(64, v, seed=80 + b) for b in range(nb)]).cuda())
    seed = 66
    m.canvas_init(seed, 0)
    bufs = m.buffers()
    torch.cuda.synchronize()
    prev = [None] * nb
    stopped = [0] * nb
    scale = {1: 0.9, 2: 1.22}
    for step in range(1, 6):
        w["final_norm"].copy_(base * scale.get(step, 8.0))
        before = bufs["canvas"].cpu().numpy().reshape(nb, t).copy()
        m.denoise_step(step)
        logits = np64(m.debug_logits()) if step <= 4 else None
        m.sample_update(step)
        torch.cuda.synchronize()
        g_canvas = bufs["canvas"].cpu().numpy().reshape(nb, t)
        g_amax = bufs["argmax"].cpu().numpy().reshape(nb, t)
        st = bufs["state"].cpu().numpy()
        for b in range(nb):
            if stopped[b]:  # frozen: nothing of this canvas moves
                assert np.array_equal(g_canvas[b], before[b]) and st[b, 1] == stopped[b], (step, b)
                continue
            rows = slice(b * t, (b + 1) * t)
            conf, ent, amax = osmp.row_stats(logits[rows])
            assert np.all(np.abs(conf - tau) > 1e-4) and abs(ent.mean() - 0.005) > 5e-5
            nxt, lock = osmp.sample_update(conf, amax, seed + b, 0, step, v, tau=tau)
            assert np.array_equal(g_amax[b], amax) and np.array_equal(g_canvas[b], nxt), (step, b)
            stop = osmp.would_stop(step, ent.mean(), amax, prev[b])
            assert bool(st[b, 0]) == stop and st[b, 3] == step and st[b, 4] == lock.sum(), (step, b)
            if stop:
                stopped[b] = step
            prev[b] = amax
        if step == 1:  # the re-noised positions take their own key's Philox draw
            for b in range(nb):
                exp = uniform_ids_np(seed + b, 0, 1, np.arange(t), osmp.TAG_RENOISE, v)
                assert np.array_equal(g_canvas[b], exp)
    assert stopped == [4, 3, 3, 4], stopped
    ids, states = m.commit_block()
    torch.cuda.synchronize()
    s = states.cpu().numpy()
    assert np.array_equal(s[:, 0], [1, 1, 1, 1]) and np.array_equal(s[:, 1], [4, 3, 3, 4])
    assert np.array_equal(ids.cpu().numpy().reshape(nb, t), np.stack(prev))
    m.check_device_status()
    m.close()
