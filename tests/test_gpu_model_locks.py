"""The model's own sampler (the LM head's vocabulary-tile statistics merged by the sampler kernel):
confidence locks and the adaptive stop, compared with the oracle's sampler on the GPU's logits.

Random-init models at N(0, 0.02) never reach a confidence of 0.9, so the end-to-end tests only
see re-noised positions.  Here the lock path is driven two ways ([canvas] step 3, [course] table
2.1: confident tokens stay, uncertain ones are re-randomised, at most 48 steps, stop once the mean
entropy is below 0.005 and the argmax is identical on two consecutive steps):

  * the lock threshold is set to the median step-1 confidence of a real two-layer model, so about
    half the canvas locks at every step;
  * a model whose attention and expert output projections are zero keeps each canvas token's own
    embedding as its final hidden state, so its tied LM head ranks the input token first; scaling
    the final-norm weights between steps moves the confidence from below the threshold (step 1),
    through a mixed canvas (steps 2-3) to certainty (step 4 on), which makes the adaptive stop fall
    at step 5 by construction (step 4 locks everything but its argmax differs from step 3's, whose
    canvas was partly re-noised; step 5 sees the same canvas again); dg_reset_block then restarts
    the stopped block, which stops again at step 2.

Every step's next canvas, argmax and device state words are compared with oracle/sampler.py on the
logits the GPU produced for that step (dg_debug_logits: the same MMA core as the fused head).
Positions whose confidence lies within 1e-4 of the threshold may lock either way.
"""
import numpy as np
import pytest
import torch

from dg_synth import SHAPES, model_weights, uniform_ids
from oracle import sampler as osmp
from oracle.philox import uniform_ids as uniform_ids_np
from tests._helpers import np64

pytestmark = pytest.mark.gpu

GUARD = 1e-4  # confidence guard band around the lock threshold


def _to_cuda(w):
    def cv(t):
        return None if t is None else t.cuda()
    return dict(embed=cv(w["embed"]), final_norm=cv(w["final_norm"]),
                layers=[{k: cv(v) for k, v in lw.items()} for lw in w["layers"]])


def _model(w, prompt, **kw):
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config
    cfg = make_config(SHAPES["small_bf16"], kv_capacity=1024, **kw)
    m = DiffusionModel(cfg, w)
    m.kv_append(prompt.cuda())
    return m


def _check_step(m, t, seed, block, tau):
    """Run step t; compare with the oracle sampler on this step's GPU logits.  Returns
    (canvas_out, argmax, n_locked, mean entropy)."""
    v = SHAPES["small_bf16"]["vocab"]
    m.denoise_step(t)
    logits = np64(m.debug_logits())
    m.sample_update(t)
    bufs = m.buffers()
    torch.cuda.synchronize()
    conf, ent, amax = osmp.row_stats(logits)
    nxt, lock = osmp.sample_update(conf, amax, seed, block, t, v, tau=tau)
    clear = np.abs(conf - tau) > GUARD
    g_canvas = bufs["canvas"].cpu().numpy().astype(np.int64)
    assert np.array_equal(bufs["argmax"].cpu().numpy(), amax), t
    assert np.array_equal(g_canvas[clear], nxt[clear]), t
    # inside the guard band the id is one of the two candidates: the argmax or the Philox draw
    noise = uniform_ids_np(seed, block, t, np.arange(len(conf)), osmp.TAG_RENOISE, v)
    inside = ~clear
    assert np.all((g_canvas[inside] == amax[inside]) | (g_canvas[inside] == noise[inside])), t
    assert np.max(np.abs(bufs["entropy"].cpu().numpy() - ent)) < 1e-5, t
    st = bufs["state"].cpu().numpy()
    assert abs(int(st[4]) - int(lock.sum())) <= int((~clear).sum()), (t, st[4], lock.sum())
    return g_canvas, amax, int(lock.sum()), float(ent.mean()), st


def test_confidence_locks_in_the_model():
    shape = SHAPES["small_bf16"]
    w = _to_cuda(model_weights("small_bf16", seed=21, norm_jitter=0.1))
    prompt = uniform_ids(96, shape["vocab"], seed=22)
    seed = 23
    probe = _model(w, prompt, fixed_steps=3)
    probe.canvas_init(seed, 0)
    probe.denoise_step(1)
    conf1 = osmp.row_stats(np64(probe.debug_logits()))[0]
    probe.close()
    tau = float(np.median(conf1))
    m = _model(w, prompt, fixed_steps=3, tau=tau)
    m.canvas_init(seed, 0)
    torch.cuda.synchronize()
    canvas = m.buffers()["canvas"].cpu().numpy()
    prev = None
    for t in (1, 2, 3):
        canvas, amax, n_locked, _, st = _check_step(m, t, seed, 0, tau)
        assert 0 < n_locked < shape["canvas"], (t, n_locked)  # the threshold splits the canvas
        prev = amax
    ids, st = m.commit_block()
    torch.cuda.synchronize()
    assert st.cpu().tolist()[:4] == [1, 3, 0, 3]
    assert np.array_equal(ids.cpu().numpy(), prev)
    m.check_device_status()
    m.close()


def test_adaptive_stop_in_the_model():
    shape = SHAPES["small_bf16"]
    wc = model_weights("small_bf16", seed=31)
    for lw in wc["layers"]:  # attention and MoE contribute nothing: x stays the embedding
        for key in ("wo", "w_d", "ws_d"):
            lw[key] = torch.zeros_like(lw[key])
    w = _to_cuda(wc)
    base_norm = w["final_norm"].clone()
    prompt = uniform_ids(64, shape["vocab"], seed=32)
    seed, block, tau = 33, 0, 0.9
    m = _model(w, prompt, fixed_steps=0, max_steps=48, tau=tau)
    m.canvas_init(seed, block)
    torch.cuda.synchronize()
    canvas = m.buffers()["canvas"].cpu().numpy()
    prev = None
    scale = {1: 0.9, 2: 1.1, 3: 1.1}
    history = []
    for t in range(1, 7):
        w["final_norm"].copy_(base_norm * scale.get(t, 8.0))
        if t <= 5:
            canvas_in = canvas
            canvas, amax, n_locked, h_mean, st = _check_step(m, t, seed, block, tau)
            assert abs(h_mean - 0.005) > 5e-5, (t, h_mean)  # no stop decision inside the guard
            oracle_stop = t >= 2 and h_mean < 0.005 and np.array_equal(amax, prev)
            history.append((t, n_locked, h_mean, oracle_stop))
            assert bool(st[0]) == oracle_stop, (t, history)
            if t == 1:
                assert n_locked == 0
            elif t in (2, 3):
                assert 0 < n_locked < shape["canvas"], history
            else:
                assert n_locked == shape["canvas"], history
                assert np.array_equal(amax, canvas_in)  # the input token ranks first
            prev = amax
        else:  # the block is done: later steps are no-ops on the device
            before = {k: v.clone() for k, v in m.buffers().items()}
            m.denoise_step(t)
            m.sample_update(t)
            torch.cuda.synchronize()
            for k, v in m.buffers().items():
                assert torch.equal(v, before[k]), k
    assert [h[3] for h in history] == [False, False, False, False, True], history
    st = m.buffers()["state"].cpu().tolist()
    assert st[:4] == [1, 5, 5, 5]
    stopped_argmax = prev
    # dg_reset_block: the stopped block runs again from step 1 on its current canvas (the step-5
    # argmax); with every position certain it stops at step 2, the earliest step allowed
    m.reset_block()
    torch.cuda.synchronize()
    assert m.buffers()["state"].cpu().tolist()[:6] == [0] * 6
    prev = None
    for t in (1, 2):
        canvas, amax, n_locked, h_mean, st = _check_step(m, t, seed, block, tau)
        assert n_locked == shape["canvas"] and np.array_equal(amax, stopped_argmax)
        assert st[:4].tolist() == ([0, 0, 0, 1] if t == 1 else [1, 2, 2, 2])
    ids, st = m.commit_block()
    torch.cuda.synchronize()
    assert st.cpu().tolist()[:4] == [1, 2, 2, 2]
    assert np.array_equal(ids.cpu().numpy(), stopped_argmax)
    m.check_device_status()
    m.close()
