"""Pins for the oracle's decoder wiring (oracle/model.py) against an independent restatement.

The oracle composes its pinned leaves (RMSNorm, RoPE, attention, router, experts) into a decoder
layer, the causal encode, the denoise forward and the LM head.  A mistake in that composition (a
wrong softmax scale, RoPE applied to V, swapped K/V slices of the fused projection, a wrong
grouped-query head map, a dropped final norm, a causal mask off by one) would leave every leaf pin
green.  These tests restate the decoder a second time with torch.nn.functional in float64, written
from the same readings of the pages ([canvas] steps 1-4, [uniform] and [arch] on the pages'
decoder: causal prefill into a KV cache, bidirectional denoise over [cache | canvas], a top-k
routed MoE FFN, the tied LM head), and compare:

  * RMSNorm through F.rms_norm, RoPE as a complex rotation (torch.polar), attention through
    F.scaled_dot_product_attention with enable_gqa and an explicit boolean causal mask, the
    router through softmax + torch.topk, experts with F.silu, the LM head through F.linear;
  * two hand-worked cases whose values are written out with scalar math: a one-head, two-token
    attention layer in which the 1/sqrt(hd) scale and the RoPE rotation are visible, and a
    two-channel LM head with a non-unit final norm;
  * planted mistakes: each test of the last group rewrites one line of the oracle's source (on the
    CPU, in this process only) and checks that the restatement then disagrees.
"""
import inspect
import math
import textwrap

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as oatt
from oracle import model as om
from oracle import moe as omoe

F64 = torch.float64


def _cfg(**kw):
    base = dict(n_layers=2, d_model=32, n_heads=4, n_kv_heads=2, head_dim=8, n_experts=4, top_k=2,
                expert_hidden=16, shared_hidden=24, vocab=64, canvas=7, storage="fp32")
    base.update(kw)
    return om.ModelConfig(**base)


def _weights(cfg, seed=0, std=0.25):
    # larger than the model's N(0, 0.02) init so that attention is peaked and routing decided
    # by clear margins: a wrong scale or head map then changes the output by far more than the
    # fp32 storage rounding of the oracle
    rng = np.random.default_rng(seed)
    d, hd = cfg.d_model, cfg.head_dim

    def n(*s):
        return rng.standard_normal(s) * std

    layers = []
    for _ in range(cfg.n_layers):
        layers.append(dict(
            attn_norm=1 + rng.standard_normal(d) * 0.2, ffn_norm=1 + rng.standard_normal(d) * 0.2,
            wqkv=n((cfg.n_heads + 2 * cfg.n_kv_heads) * hd, d), wo=n(d, cfg.n_heads * hd) * 0.5,
            wr=n(cfg.n_experts, d) * 4, w_gu=n(cfg.n_experts, 2 * cfg.expert_hidden, d),
            w_d=n(cfg.n_experts, d, cfg.expert_hidden) * 0.5,
            ws_gu=n(2 * cfg.shared_hidden, d) if cfg.shared_hidden else None,
            ws_d=n(d, cfg.shared_hidden) * 0.5 if cfg.shared_hidden else None))
    return dict(embed=rng.standard_normal((cfg.vocab, d)), layers=layers,
                final_norm=1 + rng.standard_normal(d) * 0.3)


# ---- the independent restatement (torch.nn.functional, float64) ----------------------------

def _t(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float64), dtype=F64)


def t_rope(x, pos, theta):
    """x [H, T, hd]: channel i and channel i + hd/2 form the complex number rotated by
    pos * theta^(-2i/hd)."""
    half = x.shape[-1] // 2
    freq = theta ** (-2.0 * torch.arange(half, dtype=F64) / x.shape[-1])
    ang = _t(pos)[:, None] * freq[None, :]
    z = torch.complex(x[..., :half], x[..., half:]) * torch.polar(torch.ones_like(ang), ang)
    return torch.cat([z.real, z.imag], dim=-1)


def t_attention_half(cfg, lw, x, pos, ck, cv, causal):
    """x [T, d]; ck, cv [Hkv, P, hd]; returns (x + O-projection, k, v)."""
    t, d = x.shape
    hq, hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    xn = F.rms_norm(x, (d,), weight=_t(lw["attn_norm"]), eps=cfg.eps)
    wq, wk, wv = torch.split(_t(lw["wqkv"]), [hq * hd, hkv * hd, hkv * hd], dim=0)
    q = F.linear(xn, wq).view(t, hq, hd).transpose(0, 1)
    k = F.linear(xn, wk).view(t, hkv, hd).transpose(0, 1)
    v = F.linear(xn, wv).view(t, hkv, hd).transpose(0, 1)
    q, k = t_rope(q, pos, cfg.rope_theta), t_rope(k, pos, cfg.rope_theta)
    keys, vals = torch.cat([ck, k], dim=1), torch.cat([cv, v], dim=1)
    p = ck.shape[1]
    mask = None
    if causal:  # token i (absolute position p + i) sees keys 0 .. p + i
        mask = torch.ones(t, p + t, dtype=torch.bool).tril(diagonal=p)
    o = F.scaled_dot_product_attention(q[None], keys[None], vals[None], attn_mask=mask,
                                       enable_gqa=True)[0]
    o = o.transpose(0, 1).reshape(t, hq * hd)
    return x + F.linear(o, _t(lw["wo"])), k, v


def t_glu(x, w_gu, w_d):
    w_gu = _t(w_gu)
    return F.linear(F.silu(F.linear(x, w_gu[0::2])) * F.linear(x, w_gu[1::2]), _t(w_d))


def t_moe_half(cfg, lw, x1):
    d = x1.shape[1]
    xn = F.rms_norm(x1, (d,), weight=_t(lw["ffn_norm"]), eps=cfg.eps)
    probs = torch.softmax(F.linear(xn, _t(lw["wr"])), dim=-1)
    top_p, top_i = torch.topk(probs, cfg.top_k, dim=-1)
    gates = top_p / top_p.sum(dim=-1, keepdim=True)
    y = torch.zeros_like(x1)
    for tok in range(x1.shape[0]):
        for s in range(cfg.top_k):
            e = int(top_i[tok, s])
            y[tok] += gates[tok, s] * t_glu(xn[tok:tok + 1], lw["w_gu"][e], lw["w_d"][e])[0]
    if lw.get("ws_gu") is not None:
        y = y + t_glu(xn, lw["ws_gu"], lw["ws_d"])
    return x1 + y


def t_forward(cfg, w, ids, pos, cache, causal):
    """All layers over ids; cache = per-layer (k, v) lists or None; returns (x, new k/v)."""
    x = _t(w["embed"])[torch.as_tensor(np.asarray(ids))]
    new = []
    for l, lw in enumerate(w["layers"]):
        if cache is None:
            ck = torch.zeros(cfg.n_kv_heads, 0, cfg.head_dim, dtype=F64)
            cv = ck.clone()
        else:
            ck, cv = cache[l]
        x, k, v = t_attention_half(cfg, lw, x, pos, ck, cv, causal)
        x = t_moe_half(cfg, lw, x)
        new.append((k, v))
    return x, new


def t_lm_head(cfg, w, x):
    return F.linear(F.rms_norm(x, (x.shape[1],), weight=_t(w["final_norm"]), eps=cfg.eps),
                    _t(w["embed"]))


def _rel(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    if not (np.all(np.isfinite(a)) and np.all(np.isfinite(b))):
        return math.inf
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _compare_decoder(cfg, w, seed=0):
    """Oracle vs restatement: prompt K/V, a second (commit-like) causal chunk over the prompt's
    cache, and the denoise logits of a canvas over the longer cache.  Returns the worst
    max-abs-relative error over the compared tensors."""
    rng = np.random.default_rng(seed + 100)
    prompt = rng.integers(0, cfg.vocab, 9)
    block = rng.integers(0, cfg.vocab, 5)
    canvas = rng.integers(0, cfg.vocab, cfg.canvas)
    worst = 0.0
    cache = om.causal_encode(cfg, w, prompt, om.KVCache())
    _, tkv = t_forward(cfg, w, prompt, np.arange(9), None, causal=True)
    for l in range(cfg.n_layers):
        worst = max(worst, _rel(cache.k[l], tkv[l][0]), _rel(cache.v[l], tkv[l][1]))
    om.causal_encode(cfg, w, block, cache)
    _, tkv2 = t_forward(cfg, w, block, 9 + np.arange(5), tkv, causal=True)
    for l in range(cfg.n_layers):
        worst = max(worst, _rel(cache.k[l][:, 9:], tkv2[l][0]), _rel(cache.v[l][:, 9:], tkv2[l][1]))
    full = [(torch.cat([a[0], b[0]], 1), torch.cat([a[1], b[1]], 1)) for a, b in zip(tkv, tkv2)]
    logits = om.denoise_logits(cfg, w, canvas, cache)
    x, _ = t_forward(cfg, w, canvas, 14 + np.arange(cfg.canvas), full, causal=False)
    worst = max(worst, _rel(logits, t_lm_head(cfg, w, x)))
    return worst


# The oracle stores its intermediates in binary32 in this configuration, the restatement keeps
# float64: the two differ by a few binary32 roundings propagated through two layers.
TOL = 2e-5


@pytest.mark.parametrize("seed", [0, 1])
def test_decoder_matches_torch_restatement(seed):
    cfg = _cfg()
    w = _weights(cfg, seed=seed)
    assert _compare_decoder(cfg, w, seed) < TOL


def test_decoder_matches_restatement_without_shared_expert_mha():
    cfg = _cfg(n_heads=2, n_kv_heads=2, shared_hidden=0, top_k=1, n_layers=1)
    w = _weights(cfg, seed=5)
    assert _compare_decoder(cfg, w, 5) < TOL


def test_router_margins_are_clear():
    # the comparison assumes both sides pick the same experts: no top-k near-tie in the oracle
    cfg = _cfg()
    w = _weights(cfg, seed=0)
    ids = np.random.default_rng(100).integers(0, cfg.vocab, 9)
    _, _, infos = om.forward_tokens(cfg, w, ids, np.arange(9), om.KVCache(), causal=True,
                                    keep_info=True)
    for info in infos:
        srt = -np.sort(-info["moe"]["router_logits"], axis=1)
        assert np.min(srt[:, cfg.top_k - 1] - srt[:, cfg.top_k]) > 1e-4


# ---- hand-worked cases ----------------------------------------------------------------------

def _identity_layer(d, hd, hq=1, hkv=1):
    """q = k = v = normed x, O projection = identity, unit norms."""
    eye = np.eye(hd, d)
    return dict(attn_norm=np.ones(d), wqkv=np.concatenate([eye] * (hq + 2 * hkv)), wo=np.eye(d, hq * hd))


def test_hand_worked_attention_scale():
    """One head, hd = 4, two tokens at position 0 (RoPE is the identity there), no history.
    x0 = (2,0,0,0), x1 = (0,2,0,0) have rms 1, so with eps = 0 the normed rows equal x.  Scores:
    q0.k0 = 4, q0.k1 = 0, scaled by 1/sqrt(4) to (2, 0): p = 1/(1 + e^-2) on the own token.
    Output row 0 = x0 + (2p, 2(1-p), 0, 0); row 1 is the mirror image.  A scale of 1/hd would
    give p = 1/(1 + e^-1) instead."""
    cfg = _cfg(d_model=4, n_heads=1, n_kv_heads=1, head_dim=4, eps=0.0)
    x = np.array([[2.0, 0, 0, 0], [0, 2.0, 0, 0]])
    empty = np.zeros((1, 0, 4))
    x1, k, v, _ = om.attention_block(cfg, _identity_layer(4, 4), x, np.array([0, 0]), empty, empty,
                                     causal=False)
    p = 1.0 / (1.0 + math.exp(-2.0))
    want = np.array([[2 + 2 * p, 2 * (1 - p), 0, 0], [2 * (1 - p), 2 + 2 * p, 0, 0]])
    assert np.allclose(x1, want, rtol=1e-7, atol=1e-7)
    assert np.allclose(k[0], x) and np.allclose(v[0], x)
    # causal: token 0 sees only itself, token 1 both
    x1c, _, _, _ = om.attention_block(cfg, _identity_layer(4, 4), x, np.array([0, 0]), empty,
                                      empty, causal=True)
    assert np.allclose(x1c, [[4, 0, 0, 0], want[1]], rtol=1e-7, atol=1e-7)


def test_hand_worked_rope_rotation():
    """hd = d = 2, one head; tokens at positions 0 and 1, theta irrelevant (frequency theta^0 = 1).
    x0 = (1, 1), x1 = (1, -1) (rms 1, eps 0).  q = k = RoPE(x): token 1 is rotated by 1 radian,
    (a, b) -> (a cos 1 - b sin 1, b cos 1 + a sin 1); V is not rotated.  Scores scaled by
    1/sqrt(2)."""
    cfg = _cfg(d_model=2, n_heads=1, n_kv_heads=1, head_dim=2, eps=0.0)
    x = np.array([[1.0, 1.0], [1.0, -1.0]])
    c, s = math.cos(1.0), math.sin(1.0)
    r1 = (1.0 * c + 1.0 * s, -1.0 * c + 1.0 * s)
    keys = [(1.0, 1.0), r1]
    vals = [(1.0, 1.0), (1.0, -1.0)]
    want = []
    for qi, xi in zip(keys, x):  # q = k per token
        sc = [(qi[0] * kj[0] + qi[1] * kj[1]) / math.sqrt(2.0) for kj in keys]
        e = [math.exp(z - max(sc)) for z in sc]
        p = [z / sum(e) for z in e]
        want.append([xi[0] + p[0] * vals[0][0] + p[1] * vals[1][0],
                     xi[1] + p[0] * vals[0][1] + p[1] * vals[1][1]])
    empty = np.zeros((1, 0, 2))
    x1, k, v, _ = om.attention_block(cfg, _identity_layer(2, 2), x, np.array([0, 1]), empty, empty,
                                     causal=False)
    assert np.allclose(x1, want, rtol=1e-7, atol=1e-7)
    assert np.allclose(k[0], keys, atol=1e-7) and np.allclose(v[0], vals)


def test_hand_worked_lm_head():
    """x = (3, 4): rms = sqrt(12.5); final norm weights (2, 0.5); embeddings e0 = (1, 0),
    e1 = (0, 1), e2 = (1, 1): logits = (x / rms * w) . e_j."""
    cfg = _cfg(d_model=2, vocab=3, eps=0.0)
    w = dict(final_norm=np.array([2.0, 0.5]), embed=np.array([[1.0, 0], [0, 1.0], [1.0, 1.0]]))
    r = math.sqrt(12.5)
    a, b = 3 / r * 2.0, 4 / r * 0.5
    assert np.allclose(om.lm_head(cfg, w, np.array([[3.0, 4.0]])), [[a, b, a + b]], rtol=1e-7)


def test_hand_worked_gqa_head_map():
    """Two query heads share one KV head (Hq = 2, Hkv = 1); with a second KV head (Hq = 4,
    Hkv = 2), query heads 0, 1 read KV head 0 and query heads 2, 3 read KV head 1."""
    q = np.zeros((4, 1, 2))
    k = np.zeros((2, 2, 2))
    v = np.array([[[1.0, 0], [1.0, 0]], [[0, 1.0], [0, 1.0]]])  # kv head 0 -> (1,0), 1 -> (0,1)
    o = oatt.attention(q, k, v, 1.0)
    assert np.allclose(o[:, 0], [[1, 0], [1, 0], [0, 1], [0, 1]])


# ---- planted mistakes: the pins above must catch each one ------------------------------------

def _mutant(monkeypatch, module, name, old, new):
    """Replace module.name by a copy of its source with `old` replaced by `new` (CPU only)."""
    fn = getattr(module, name)
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) == 1, (name, old)
    ns = dict(fn.__globals__)
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    monkeypatch.setattr(module, name, ns[name])
    # modules that imported the function by name see the mutant too
    for mod in (om, omoe, oatt):
        if getattr(mod, name, None) is fn:
            monkeypatch.setattr(mod, name, ns[name])


MUTATIONS = [
    ("scale 1/hd", om, "attention_block", "1.0 / np.sqrt(hd)", "1.0 / hd"),
    ("RoPE on V", om, "attention_block", "v = round_storage(v, st)",
     "v = round_storage(rope(v, positions, cfg.rope_theta), st)"),
    ("K/V slices swapped", om, "attention_block",
     "k = qkv[:, hq * hd:(hq + hkv) * hd]", "k = qkv[:, (hq + hkv) * hd:]"),
    ("GQA head map j % Hkv", oatt, "attention", "g = j // group", "g = j % hkv"),
    ("causal mask off by one", oatt, "attention", "np.arange(n)[None, :] <=", "np.arange(n)[None, :] <"),
    ("final norm dropped", om, "lm_head", 'rmsnorm(x, weights["final_norm"], cfg.eps)', "x"),
    ("RoPE sign", om, "rope", "x1 * c - x2 * s", "x1 * c + x2 * s"),
    ("RoPE frequency", om, "rope", "-2.0 * np.arange(half", "-1.0 * np.arange(half"),
    ("attention residual dropped", om, "attention_block",
     "np.asarray(x, dtype=np.float64) + o @", "0.0 * np.asarray(x, dtype=np.float64) + o @"),
    ("attention norm weight dropped", om, "attention_block", 'rmsnorm(x, lw["attn_norm"], cfg.eps)',
     "rmsnorm(x, 1.0, cfg.eps)"),
    ("ffn norm takes the attention norm's weight", om, "moe_block", 'rmsnorm(x1, lw["ffn_norm"]',
     'rmsnorm(x1, lw["attn_norm"]'),
    ("router weights not renormalised", omoe, "router", "w = sel / sel.sum(axis=1, keepdims=True)",
     "w = sel"),
    ("gate and up swapped", omoe, "expert_glu", "g = xn @ w_gu[0::2].T", "g = xn @ w_gu[1::2].T"),
    ("shared expert dropped", omoe, "moe_ffn", "y = y + ys", "y = y"),
    ("cache ignored by denoise", om, "forward_tokens", "if cache.length:", "if False:"),
]


@pytest.mark.parametrize("label,module,name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, label, module, name, old, new):
    cfg = _cfg()
    w = _weights(cfg, seed=0)
    assert _compare_decoder(cfg, w, 0) < TOL  # sane before the mutation
    _mutant(monkeypatch, module, name, old, new)
    caught = _compare_decoder(cfg, w, 0) > 1e-3
    if label in ("scale 1/hd", "RoPE on V", "RoPE sign"):
        # these must also fail a hand-worked case
        try:
            test_hand_worked_attention_scale()
            test_hand_worked_rope_rotation()
            hand = False
        except AssertionError:
            hand = True
        caught = caught and hand
    if label == "final norm dropped":
        try:
            test_hand_worked_lm_head()
            hand = False
        except AssertionError:
            hand = True
        caught = caught and hand
    assert caught, label
