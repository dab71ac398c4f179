"""Sampler variants in the model: entropy-bound locking and sticky locks.

Each step's lock decisions, next canvas and the committed block are compared with the oracle's
sampler (oracle/sampler.py) applied to the GPU's own logits of that step, so the comparison is
of the integer decisions given identical logits; positions whose entropy lies within 1e-4 of the
bound may decide either way and are excluded.
"""
import numpy as np
import pytest
import torch

from dg_synth import SHAPES, model_weights, uniform_ids
from oracle import sampler as osmp
from tests._helpers import np64

pytestmark = pytest.mark.gpu


def _to_cuda(w):
    def cv(t):
        return None if t is None else t.cuda()
    return dict(embed=cv(w["embed"]), final_norm=cv(w["final_norm"]),
                layers=[{k: cv(v) for k, v in lw.items()} for lw in w["layers"]])


def _model(w, prompt, **kw):
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config
    cfg = make_config(SHAPES["small_bf16"], kv_capacity=1024, fixed_steps=3, **kw)
    m = DiffusionModel(cfg, w)
    m.kv_append(prompt.cuda())
    return m


@pytest.mark.parametrize("sticky", [True, False])
def test_entropy_bound_locks_match_the_oracle(sticky):
    shape = SHAPES["small_bf16"]
    v = shape["vocab"]
    # larger weights than the other tests so that the canvas entropies spread out
    w = _to_cuda(model_weights("small_bf16", seed=11, std=0.08))
    prompt = uniform_ids(64, v, seed=12)
    seed = 13
    # probe: the step-1 entropies fix a bound that splits the canvas
    probe = _model(w, prompt)
    probe.canvas_init(seed, 0)
    probe.denoise_step(1)
    ent1 = osmp.row_stats(np64(probe.debug_logits()))[1]
    probe.close()
    bound = float(np.median(ent1))
    m = _model(w, prompt, lock_rule="entropy_bound", entropy_lock=bound, sticky=sticky)
    m.canvas_init(seed, 0)
    bufs = m.buffers()
    torch.cuda.synchronize()
    canvas = bufs["canvas"].cpu().numpy().astype(np.int64)
    locked = None
    n_locked_seen = []
    for t in (1, 2, 3):
        m.denoise_step(t)
        logits = np64(m.debug_logits())
        m.sample_update(t)
        torch.cuda.synchronize()
        conf, ent, amax = osmp.row_stats(logits)
        nxt, lock = osmp.sample_update(conf, amax, seed, 0, t, v, entropy=ent,
                                       rule="entropy_bound", entropy_bound=bound, sticky=sticky,
                                       prev_canvas=canvas, prev_locked=locked)
        clear = np.abs(ent - bound) > 1e-4
        if sticky and locked is not None:
            clear |= locked  # kept positions do not depend on this step's entropy
        g_canvas = bufs["canvas"].cpu().numpy().astype(np.int64)
        assert np.array_equal(g_canvas[clear], nxt[clear]), t
        assert np.array_equal(bufs["argmax"].cpu().numpy(), amax)
        # the device counts the locked positions of the step
        g_locked = int(bufs["state"].cpu().numpy()[4])
        assert abs(g_locked - int(lock.sum())) <= int((~clear).sum()), (t, g_locked, lock.sum())
        n_locked_seen.append(int(lock.sum()))
        # carry the GPU's own canvas and the oracle's mask (equal to the GPU's where clear)
        canvas, locked = g_canvas, lock
    assert 0 < n_locked_seen[0] < shape["canvas"]  # the bound splits the canvas
    if sticky:
        assert n_locked_seen[2] >= n_locked_seen[0]  # locks persist
    ids, st = m.commit_block()
    torch.cuda.synchronize()
    want = np.where(locked, canvas, amax)
    assert np.array_equal(ids.cpu().numpy()[clear], want[clear])
    m.check_device_status()
    m.close()


@pytest.mark.parametrize("shape_name,temp", [("small_bf16", 0.7), ("tiny_fp32", 1.6)])
def test_temperature_statistics_match_the_oracle(shape_name, temp):
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config
    shape = SHAPES[shape_name]
    v = shape["vocab"]
    w = _to_cuda(model_weights(shape_name, seed=21, std=0.08))
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=2, temperature=temp)
    m = DiffusionModel(cfg, w)
    m.kv_append(uniform_ids(64, v, seed=22).cuda())
    m.canvas_init(23, 0)
    m.denoise_step(1)
    logits = np64(m.debug_logits())
    m.sample_update(1)
    bufs = m.buffers()
    torch.cuda.synchronize()
    conf, ent, amax = osmp.row_stats(logits, temperature=temp)
    assert np.array_equal(bufs["argmax"].cpu().numpy(), amax)
    assert np.max(np.abs(bufs["entropy"].cpu().numpy() - ent)) < 1e-5
    assert np.max(np.abs(bufs["conf"].cpu().numpy() - conf)) < 1e-5
    # the temperature changes the statistics: at T = 1 they differ
    _, ent1, _ = osmp.row_stats(logits)
    assert np.max(np.abs(ent1 - ent)) > 1e-3
    clear = np.abs(conf - 0.9) > 1e-4
    nxt, _ = osmp.sample_update(conf, amax, 23, 0, 1, v)
    assert np.array_equal(bufs["canvas"].cpu().numpy()[clear], nxt[clear])
    m.check_device_status()
    m.close()


def test_commit_reusing_canvas_kv():
    """commit_reuse_kv: the commit keeps the K/V the last denoise step wrote for the canvas (the
    bidirectional forward of that step's input canvas) and only advances the cache length; the
    slots match the oracle's commit_reusing_canvas_kv, token by token (routing near-ties
    excused as in the prefill checks), and the next block runs on the longer cache."""
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config
    from oracle import model as om
    from tests._helpers import kv_tokens_close, router_gaps, weights_to_np
    shape = SHAPES["small_bf16"]
    v = shape["vocab"]
    wt = model_weights("small_bf16", seed=41, norm_jitter=0.1)
    cfg = make_config(shape, kv_capacity=1024, fixed_steps=2, commit="reuse_kv")
    m = DiffusionModel(cfg, _to_cuda(wt))
    prompt = uniform_ids(128, v, seed=42)
    m.kv_append(prompt.cuda())
    m.canvas_init(43, 0)
    m.denoise_step(1)
    m.sample_update(1)
    bufs = m.buffers()
    torch.cuda.synchronize()
    canvas_in_2 = bufs["canvas"].cpu().numpy().astype(np.int64)
    m.denoise_step(2)
    m.sample_update(2)
    kv = m.kv.view(torch.bfloat16)
    half = kv.numel() // 2
    k_all = kv[:half].view(cfg.n_layers, cfg.n_kv_heads, cfg.kv_capacity, cfg.head_dim)
    vt_all = kv[half:].view(cfg.n_layers, cfg.n_kv_heads, cfg.head_dim, cfg.kv_capacity)
    k_before = k_all[:, :, 128:384].clone()
    v_before = vt_all[:, :, :, 128:384].clone()
    ids, st = m.commit_block()
    torch.cuda.synchronize()
    assert m.kv_length == 384 and st.cpu().tolist()[:2] == [1, 2]
    assert np.array_equal(ids.cpu().numpy(), bufs["argmax"].cpu().numpy())
    # nothing was re-encoded: the slots hold exactly what step 2 wrote
    assert torch.equal(k_all[:, :, 128:384], k_before)
    assert torch.equal(vt_all[:, :, :, 128:384], v_before)
    ocfg = om.ModelConfig(**{k: shape[k] for k in (
        "n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "n_experts", "top_k",
        "expert_hidden", "shared_hidden", "vocab", "canvas", "storage")})
    ow = weights_to_np(wt)
    ocache = om.causal_encode(ocfg, ow, prompt.numpy(), om.KVCache())
    gaps = router_gaps(ocfg, ow, canvas_in_2, 128 + np.arange(256), ocache, causal=False)
    om.commit_reusing_canvas_kv(ocfg, ow, canvas_in_2, ocache)
    for l in range(cfg.n_layers):
        ok, bad, _ = kv_tokens_close(np64(k_before[l]), ocache.k[l][:, 128:], gaps, l, 2e-2)
        assert ok, ("reused K", l, bad)
        ok, bad, _ = kv_tokens_close(np64(v_before[l]).transpose(0, 2, 1), ocache.v[l][:, 128:],
                                     gaps, l, 2e-2)
        assert ok, ("reused V", l, bad)
    m.canvas_init(43, 1)
    m.denoise_step(1)
    m.sample_update(1)
    m.check_device_status()
    m.close()
