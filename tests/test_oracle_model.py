"""Pins for the oracle's decoder pieces and the block-autoregressive decode loop."""
import numpy as np
import pytest

from oracle import model as om
from oracle import sampler as smp


def _cfg(**kw):
    base = dict(n_layers=2, d_model=32, n_heads=4, n_kv_heads=2, head_dim=8, n_experts=4, top_k=2,
                expert_hidden=16, shared_hidden=24, vocab=512, canvas=16, storage="fp32")
    base.update(kw)
    return om.ModelConfig(**base)


def _weights(cfg, seed=0, zero_blocks=False, std=0.02):
    rng = np.random.default_rng(seed)
    n = (lambda *s: np.zeros(s)) if zero_blocks else (lambda *s: rng.standard_normal(s) * std)
    d, hd = cfg.d_model, cfg.head_dim
    layers = []
    for _ in range(cfg.n_layers):
        layers.append(dict(
            attn_norm=1 + rng.standard_normal(d) * 0.1, ffn_norm=1 + rng.standard_normal(d) * 0.1,
            wqkv=n((cfg.n_heads + 2 * cfg.n_kv_heads) * hd, d), wo=n(d, cfg.n_heads * hd),
            wr=n(cfg.n_experts, d), w_gu=n(cfg.n_experts, 2 * cfg.expert_hidden, d),
            w_d=n(cfg.n_experts, d, cfg.expert_hidden),
            ws_gu=n(2 * cfg.shared_hidden, d) if cfg.shared_hidden else None,
            ws_d=n(d, cfg.shared_hidden) if cfg.shared_hidden else None))
    return dict(embed=rng.standard_normal((cfg.vocab, d)) * std, layers=layers,
                final_norm=np.ones(d))


def test_rmsnorm_closed_form():
    x = np.full((1, 10), -3.0)
    w = np.linspace(0.5, 2, 10)
    out = om.rmsnorm(x, w, 1e-6)
    assert np.allclose(out, -3.0 / np.sqrt(9.0 + 1e-6) * w, rtol=1e-15)


def test_rope_is_complex_rotation():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, 5, 16))
    pos = np.array([0, 1, 7, 100, 4095])
    out = om.rope(x, pos, 10000.0)
    z = x[..., :8] + 1j * x[..., 8:]
    ang = pos[:, None] * 10000.0 ** (-np.arange(8) / 8.0)
    ref = z * np.exp(1j * ang)[None]
    assert np.allclose(out[..., :8], ref.real, atol=1e-12) and np.allclose(out[..., 8:], ref.imag, atol=1e-12)
    assert np.allclose(out[:, 0], x[:, 0])  # position 0 is the identity


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal((1, 1, 32)), rng.standard_normal((1, 1, 32))
    s = [float((om.rope(q, [p + 5], 1e4) * om.rope(k, [p], 1e4)).sum()) for p in (0, 17, 300)]
    assert np.allclose(s, s[0], rtol=1e-10)


def test_causal_encode_is_chunk_invariant():
    cfg = _cfg()
    w = _weights(cfg)
    ids = np.random.default_rng(2).integers(0, cfg.vocab, 37)
    c1 = om.causal_encode(cfg, w, ids, om.KVCache())
    c2 = om.causal_encode(cfg, w, ids[:20], om.KVCache())
    om.causal_encode(cfg, w, ids[20:], c2)
    assert c1.length == c2.length == 37
    for l in range(cfg.n_layers):
        assert np.allclose(c1.k[l], c2.k[l], atol=1e-6) and np.allclose(c1.v[l], c2.v[l], atol=1e-6)


def test_denoise_leaves_cache_untouched_and_uses_it():
    cfg = _cfg()
    w = _weights(cfg, std=0.2)
    cache = om.causal_encode(cfg, w, np.arange(10), om.KVCache())
    canvas = np.arange(cfg.canvas) + 3
    l1 = om.denoise_logits(cfg, w, canvas, cache)
    assert cache.length == 10
    cache_b = om.causal_encode(cfg, w, np.arange(10) + 1, om.KVCache())
    l2 = om.denoise_logits(cfg, w, canvas, cache_b)
    assert np.abs(l1 - l2).max() > 1e-6  # the history matters


def test_zero_blocks_model_returns_input_token():
    # with every projection zero the residual stream is the embedding, and the tied head ranks
    # each token's own embedding first; with tau = 0 every position locks, so the canvas never moves
    cfg = _cfg(tau=0.0)
    w = _weights(cfg, zero_blocks=True)
    w["embed"] = np.random.default_rng(3).standard_normal((cfg.vocab, cfg.d_model)) * 0.02
    ids, blocks, cache = om.decode(cfg, w, np.arange(5), 2, seed=9, fixed_steps=3)
    for b in range(2):
        init = smp.canvas_init(9, b, cfg.canvas, cfg.vocab)
        assert np.array_equal(blocks[b]["committed"], init)
        for st in blocks[b]["steps"]:
            assert np.array_equal(st["amax"], init) and st["locked"].all()
    assert cache.length == 5 + 2 * cfg.canvas and len(ids) == 2 * cfg.canvas


def test_never_locking_canvas_is_the_philox_stream():
    cfg = _cfg(tau=1.5)
    w = _weights(cfg)
    _, blocks, _ = om.decode(cfg, w, np.arange(4), 1, seed=123, fixed_steps=4)
    from oracle.philox import uniform_ids
    for st in blocks[0]["steps"]:
        exp = uniform_ids(123, 0, st["step"], np.arange(cfg.canvas), 1, cfg.vocab)
        assert np.array_equal(st["canvas_out"], exp)


def test_bf16_storage_points_are_rounded():
    cfg = _cfg(storage="bf16")
    w = _weights(cfg)
    cache = om.causal_encode(cfg, w, np.arange(8), om.KVCache())
    _, infos = om.denoise_logits(cfg, w, np.arange(cfg.canvas), cache, keep_info=True)
    from oracle.numerics import round_bf16
    for key in ("xn", "q", "k", "v", "o", "xn2"):
        a = infos[0][key]
        assert np.array_equal(a, round_bf16(a)), key
    assert np.array_equal(cache.k[0], round_bf16(cache.k[0]))


def test_reuse_kv_commit_equals_reencode_when_tokens_only_see_themselves():
    # zero blocks: every layer's K/V of a token depend on its own embedding and position only, so
    # the bidirectional K/V of a canvas equal the causal K/V of the same ids; with tau = 0 the
    # canvas never moves (the committed ids are the last step's input canvas)
    cfg = _cfg(tau=0.0)
    w = _weights(cfg, zero_blocks=True)
    w["embed"] = np.random.default_rng(3).standard_normal((cfg.vocab, cfg.d_model)) * 0.02
    ids_a, _, cache_a = om.decode(cfg, w, np.arange(5), 2, seed=9, fixed_steps=3)
    ids_b, _, cache_b = om.decode(cfg, w, np.arange(5), 2, seed=9, fixed_steps=3,
                                  commit="reuse_kv")
    assert np.array_equal(ids_a, ids_b) and cache_a.length == cache_b.length
    for l in range(cfg.n_layers):
        assert np.array_equal(cache_a.k[l], cache_b.k[l]) and np.array_equal(cache_a.v[l], cache_b.v[l])


def test_reuse_kv_commit_keeps_the_last_step_canvas_kv():
    cfg = _cfg()
    w = _weights(cfg, std=0.2)
    ids, blocks, cache = om.decode(cfg, w, np.arange(6), 1, seed=4, fixed_steps=2,
                                   commit="reuse_kv")
    canvas_in = blocks[0]["steps"][1]["canvas_in"]
    assert not np.array_equal(canvas_in, ids)  # nothing locked: the canvas is not the block
    prompt_cache = om.causal_encode(cfg, w, np.arange(6), om.KVCache())
    _, kv_last, _ = om.forward_tokens(cfg, w, canvas_in, 6 + np.arange(cfg.canvas), prompt_cache,
                                      causal=False)
    reenc = om.causal_encode(cfg, w, ids, om.causal_encode(cfg, w, np.arange(6), om.KVCache()))
    for l in range(cfg.n_layers):
        assert np.array_equal(cache.k[l][:, :6], prompt_cache.k[l])
        assert np.array_equal(cache.k[l][:, 6:], kv_last[l][0])
        assert np.array_equal(cache.v[l][:, 6:], kv_last[l][1])
        assert not np.allclose(cache.k[l][:, 6:], reenc.k[l][:, 6:])  # not the re-encode
    with pytest.raises(ValueError):
        om.decode(cfg, w, np.arange(6), 1, seed=4, fixed_steps=2, commit="other")


def test_decode_batch_is_independent_sequences():
    cfg = _cfg()
    w = _weights(cfg, std=0.2)
    prompts = np.random.default_rng(7).integers(0, cfg.vocab, (3, 6))
    res = om.decode_batch(cfg, w, prompts, 1, seed=40, fixed_steps=2)
    assert len(res) == 3
    for b in range(3):
        ids, blocks, _ = om.decode(cfg, w, prompts[b], 1, seed=40 + b, fixed_steps=2)
        assert np.array_equal(res[b][0], ids)
        assert np.array_equal(blocks[0]["steps"][0]["canvas_in"],
                              smp.canvas_init(40 + b, 0, cfg.canvas, cfg.vocab))
    # different keys give different canvases
    assert not np.array_equal(res[0][1][0]["steps"][0]["canvas_in"], res[1][1][0]["steps"][0]["canvas_in"])
