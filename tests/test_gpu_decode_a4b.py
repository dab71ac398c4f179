"""Parity of the full-size decode model in the configuration the benchmark times.

30 layers, d 2816, 16/8 heads x 128, 128 experts top-8 x 704 + shared 2112, V 262144, bf16,
random init (the benchmark's rank-0 weights), a 4,096-token prompt prefilled, then one canvas.
The oracle cannot run the whole model, so the checks are sampled: the Philox canvas bit-exact,
the fused LM-head statistics against the oracle on the GPU's own logits for every row, the logits
of sampled rows against the oracle's LM head on the GPU's final hidden state, the first and last
layers teacher-forced against the GPU's own KV cache, and a full 16-step block plus its commit.
"""
import numpy as np
import pytest
import torch

from dg_synth import SHAPES, model_weights, uniform_ids
from oracle import model as om
from oracle import sampler as osmp
from tests._helpers import check_layer_parts, np64, npf32, rel_close

pytestmark = pytest.mark.gpu

PROMPT = 4096


def _ocfg(s):
    return om.ModelConfig(**{k: s[k] for k in ("n_layers", "d_model", "n_heads", "n_kv_heads",
                                               "head_dim", "n_experts", "top_k", "expert_hidden",
                                               "shared_hidden", "vocab", "canvas", "storage")})


@pytest.fixture(scope="module")
def model():
    from block_text_diffusion_dg_b200 import DiffusionModel, make_config
    s = SHAPES["a4b"]
    dev = torch.device("cuda", 0)
    w = model_weights("a4b", seed=1000, device=dev)
    cfg = make_config(s, kv_capacity=PROMPT + 4 * 256 + 256, fixed_steps=16)
    m = DiffusionModel(cfg, w, device=dev)
    m.kv_append(uniform_ids(PROMPT, s["vocab"], seed=0).to(dev))
    yield m, w, cfg
    m.close()


def _layer_np(w, l):
    return {k: (None if v is None else npf32(v)) for k, v in w["layers"][l].items()}


def _cache_np(m, cfg, l, n):
    kv = m.kv.view(torch.bfloat16)
    half = kv.numel() // 2
    k = kv[:half].view(cfg.n_layers, cfg.n_kv_heads, cfg.kv_capacity, cfg.head_dim)[l, :, :n]
    vt = kv[half:].view(cfg.n_layers, cfg.n_kv_heads, cfg.head_dim, cfg.kv_capacity)[l, :, :, :n]
    return np64(k), np64(vt).transpose(0, 2, 1)


def test_denoise_step_sampled(model):
    m, w, cfg = model
    s = SHAPES["a4b"]
    ocfg = _ocfg(s)
    m.canvas_init(0, 0)
    bufs = m.buffers()
    torch.cuda.synchronize()
    canvas0 = osmp.canvas_init(0, 0, 256, s["vocab"])
    assert np.array_equal(bufs["canvas"].cpu().numpy(), canvas0)
    m.denoise_step(1)
    logits = m.debug_logits()
    m.sample_update(1)
    torch.cuda.synchronize()
    x_final = np64(m.debug_hidden())
    g_logits = np64(logits)
    # fused statistics == oracle statistics on the same logits, every row
    conf, ent, amax = osmp.row_stats(g_logits)
    assert np.array_equal(bufs["argmax"].cpu().numpy(), amax)
    assert np.max(np.abs(bufs["entropy"].cpu().numpy() - ent)) < 1e-5
    nxt, _ = osmp.sample_update(conf, amax, 0, 0, 1, s["vocab"])
    assert np.array_equal(bufs["canvas"].cpu().numpy(), nxt)
    # LM head on sampled rows of the GPU's final hidden state
    rows = np.array([0, 1, 77, 128, 200, 255])
    emb = npf32(w["embed"])
    ref = om.lm_head(ocfg, dict(embed=emb, final_norm=npf32(w["final_norm"])), x_final[rows])
    err = np.max(np.abs(g_logits[rows] - ref))
    assert err < 3e-2, err
    del emb
    # first and last layers teacher-forced, half by half, against the GPU's own prompt cache
    k_top = s["top_k"]
    pos = PROMPT + np.arange(256)
    rng = np.random.default_rng(7)
    inputs = {0: np64(w["embed"][torch.from_numpy(canvas0).to(w["embed"].device)]),
              s["n_layers"] - 1: rng.standard_normal((256, s["d_model"])).astype(np.float32).astype(np.float64)}
    for l, x_in in inputs.items():
        ck, cv = _cache_np(m, cfg, l, PROMPT)
        att, moe, frac = check_layer_parts(m, ocfg, _layer_np(w, l), x_in, pos, ck, cv, l, k_top)
        assert att[0] and att[2] < 5e-3, ("attention half", l, att)
        assert moe[0] and moe[2] < 5e-3, ("moe half", l, moe)
        assert frac > 0.98, frac


def test_full_block_and_commit(model):
    m, w, cfg = model
    s = SHAPES["a4b"]
    m.canvas_init(3, 0)
    for t in range(1, 17):
        m.denoise_step(t)
        m.sample_update(t)
    bufs = m.buffers()
    torch.cuda.synchronize()
    argmax = bufs["argmax"].cpu().numpy().copy()
    canvas = bufs["canvas"].cpu().numpy().copy()
    # random weights never lock (conf << 0.9): the canvas after step 16 is the Philox stream
    conf = bufs["conf"].cpu().numpy()
    assert conf.max() < 0.9
    from oracle.philox import uniform_ids as o_ids
    assert np.array_equal(canvas, o_ids(3, 0, 16, np.arange(256), 1, s["vocab"]))
    ids, st = m.commit_block()
    torch.cuda.synchronize()
    assert st.cpu().tolist()[:4] == [1, 16, 0, 16]
    assert np.array_equal(ids.cpu().numpy(), argmax)
    assert m.kv_length == PROMPT + 256
    # layer-0 K of the committed block depends only on the committed ids: teacher-forced check
    ocfg = _ocfg(s)
    x_in = np.asarray(npf32(w["embed"][ids.long()]), dtype=np.float64)
    ck, cv = _cache_np(m, cfg, 0, PROMPT)
    _, k_ref, _, _ = om.layer_forward(ocfg, _layer_np(w, 0), x_in, PROMPT + np.arange(256), ck, cv,
                                      causal=True)
    k_gpu, _ = _cache_np(m, cfg, 0, PROMPT + 256)
    ok, worst, nrel = rel_close(k_gpu[:, PROMPT:], k_ref, 2e-2)
    assert ok and nrel < 1e-2, (worst, nrel)
    m.check_device_status()
