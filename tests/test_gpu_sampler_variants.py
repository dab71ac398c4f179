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
