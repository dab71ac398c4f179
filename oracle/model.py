"""Decoder forward, denoise step, causal encode and the block-autoregressive decode loop.

The loop is the one the pages describe ([canvas] steps 1-4, [arch]): encode the
prompt causally into a KV cache; for each 256-token block fill a canvas with
uniform-random ids, run denoise steps (a full bidirectional forward over the
canvas against the cache, then the sampler and stop test), commit the argmax
block by encoding it causally into the cache like the prompt, and start the next
canvas conditioned on the longer history.

Model structure (the pages give only "Gemma 4 26B-A4B backbone, MoE, diffusion
head"; the plainest decoder reading is used):

    x      = E[ids]                                   tied embedding, no scale
    per layer:
      xn   = rnd(rmsnorm(x, w_attn))                  pre-norm, eps 1e-6
      q,k,v= xn Wqkv^T ; q,k = rope(q,k; absolute pos); rnd(q), rnd(k), rnd(v)
      o    = rnd(attention(q, [K_cache | k], [V_cache | v]))  no mask / causal
      x    = f32(x + o Wo^T)
      xn2  = rnd(rmsnorm(x, w_ffn))
      x    = f32(x + moe_ffn(xn2))
    logits = f32(rnd(rmsnorm(x, w_final)) E^T)        the LM ("diffusion") head

rnd() is the path's storage rounding (bf16 RNE, or fp32 for the all-fp32
configuration); f32() is rounding to binary32 for the fp32 residual stream and
logits.  RoPE is rotate-half: for i < hd/2, angle = pos * theta^(-2i/hd),
out_i = x_i cos - x_{i+hd/2} sin, out_{i+hd/2} = x_{i+hd/2} cos + x_i sin.
"""
from dataclasses import dataclass, field

import numpy as np

from . import sampler as smp
from .attention import attention
from .moe import moe_ffn, moe_ffn_fp8, moe_ffn_nvfp4
from .numerics import round_f32, round_storage
from .quant import quantize_rows


@dataclass
class ModelConfig:
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    expert_hidden: int
    shared_hidden: int
    vocab: int
    canvas: int = 256
    storage: str = "bf16"
    experts: str = "bf16"  # "fp8" / "nvfp4": quantised expert weights and activations (quant.py)
    head: str = "bf16"     # "fp8": the LM head on e4m3 operands (lm_head_fp8)
    eps: float = 1e-6
    rope_theta: float = 10000.0
    tau: float = smp.TAU
    h_bound: float = smp.H_BOUND
    max_steps: int = smp.MAX_STEPS


def rmsnorm(x, w, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * np.asarray(w, dtype=np.float64)


def rope(x, positions, theta):
    """x [H, T, hd] rotated at absolute positions [T] (rotate-half)."""
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    half = hd // 2
    inv = theta ** (-2.0 * np.arange(half, dtype=np.float64) / hd)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang)[None], np.sin(ang)[None]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


@dataclass
class KVCache:
    """Per-layer committed keys/values [Hkv, P, hd] (float64 holding stored values)."""
    k: list = field(default_factory=list)
    v: list = field(default_factory=list)

    @property
    def length(self):
        return 0 if not self.k else self.k[0].shape[1]


def attention_block(cfg, lw, x, positions, cache_k, cache_v, causal):
    """Attention half of a layer over new tokens x [T, d]: returns (x + O-projection, k, v, info).

    cache_k/v: [Hkv, P, hd] committed history.
    """
    st = cfg.storage
    t = x.shape[0]
    hq, hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    xn = round_storage(rmsnorm(x, lw["attn_norm"], cfg.eps), st)
    qkv = xn @ np.asarray(lw["wqkv"], dtype=np.float64).T
    q = qkv[:, :hq * hd].reshape(t, hq, hd).transpose(1, 0, 2)
    k = qkv[:, hq * hd:(hq + hkv) * hd].reshape(t, hkv, hd).transpose(1, 0, 2)
    v = qkv[:, (hq + hkv) * hd:].reshape(t, hkv, hd).transpose(1, 0, 2)
    q = round_storage(rope(q, positions, cfg.rope_theta), st)
    k = round_storage(rope(k, positions, cfg.rope_theta), st)
    v = round_storage(v, st)
    keys = np.concatenate([cache_k, k], axis=1)
    vals = np.concatenate([cache_v, v], axis=1)
    p = cache_k.shape[1]
    o = attention(q, keys, vals, 1.0 / np.sqrt(hd), causal_prefix=p if causal else None)
    o = round_storage(o.transpose(1, 0, 2).reshape(t, hq * hd), st)
    x1 = round_f32(np.asarray(x, dtype=np.float64) + o @ np.asarray(lw["wo"], dtype=np.float64).T)
    return x1, k, v, dict(xn=xn, q=q, k=k, v=v, o=o, x_attn=x1)


def moe_block(cfg, lw, x1):
    """MoE half of a layer: returns (x1 + MoE(rmsnorm(x1)), info)."""
    st = cfg.storage
    xn2 = round_storage(rmsnorm(x1, lw["ffn_norm"], cfg.eps), st)
    shared = (lw["ws_gu"], lw["ws_d"]) if lw.get("ws_gu") is not None else None
    if cfg.experts == "fp8":
        y, minfo = moe_ffn_fp8(xn2, lw["wr"], lw["w_gu"], lw["w_d"], cfg.top_k, shared)
    elif cfg.experts == "nvfp4":
        y, minfo = moe_ffn_nvfp4(xn2, lw["wr"], lw["w_gu"], lw["w_d"], cfg.top_k, shared)
    else:
        y, minfo = moe_ffn(xn2, lw["wr"], lw["w_gu"], lw["w_d"], cfg.top_k, st, shared)
    x2 = round_f32(np.asarray(x1, dtype=np.float64) + y)
    return x2, dict(xn2=xn2, moe=minfo)


def layer_forward(cfg, lw, x, positions, cache_k, cache_v, causal):
    """One decoder layer over new tokens x [T, d] (fp32 values).

    cache_k/v: [Hkv, P, hd] committed history.  Returns (x_out, k_new, v_new, info).
    """
    x1, k, v, info = attention_block(cfg, lw, x, positions, cache_k, cache_v, causal)
    x2, minfo = moe_block(cfg, lw, x1)
    info.update(minfo)
    return x2, k, v, info


def forward_tokens(cfg, weights, ids, positions, cache, causal, keep_info=False):
    """Run all layers over new tokens; returns (final hidden x [T, d], per-layer (k, v), infos)."""
    x = round_f32(np.asarray(weights["embed"], dtype=np.float64)[np.asarray(ids)])
    kv_new, infos = [], []
    for l, lw in enumerate(weights["layers"]):
        if cache.length:
            ck, cv = cache.k[l], cache.v[l]
        else:
            ck = np.zeros((cfg.n_kv_heads, 0, cfg.head_dim))
            cv = np.zeros((cfg.n_kv_heads, 0, cfg.head_dim))
        x, k, v, info = layer_forward(cfg, lw, x, positions, ck, cv, causal)
        kv_new.append((k, v))
        if keep_info:
            infos.append(info)
    return x, kv_new, infos


def lm_head(cfg, weights, x):
    """Final norm then the tied LM head; logits rounded to fp32 like the GPU's accumulators."""
    xf = round_storage(rmsnorm(x, weights["final_norm"], cfg.eps), cfg.storage)
    if cfg.head == "fp8":
        return lm_head_fp8(xf, weights["embed"])
    return round_f32(xf @ np.asarray(weights["embed"], dtype=np.float64).T)


def lm_head_fp8(xf, embed):
    """The tied LM head with e4m3 operands (the FP8 weight format applied to the head; [pl] lists
    FP8 weights, the pages give no scheme): the stored normed rows xf [T, d] and the embedding
    rows [V, d] are each quantised per row (quant.quantize_rows: scale = max|row| / 448, codes
    rounded to nearest even); the code products are summed and scaled by (token scale) x
    (vocabulary-row scale); logits rounded to fp32."""
    xq, xs = quantize_rows(xf)
    eq, es = quantize_rows(embed)
    acc = xq @ eq.T
    return round_f32(acc * np.asarray(xs, dtype=np.float64)[:, None]
                     * np.asarray(es, dtype=np.float64)[None, :])


def denoise_logits(cfg, weights, canvas, cache, keep_info=False):
    """One denoise forward: canvas [T] ids at positions P..P+T-1, no mask, cache untouched."""
    p = cache.length
    pos = p + np.arange(len(canvas))
    x, _, infos = forward_tokens(cfg, weights, canvas, pos, cache, causal=False, keep_info=keep_info)
    logits = lm_head(cfg, weights, x)
    return (logits, infos) if keep_info else logits


def _append(cache, kv_new):
    for l, (k, v) in enumerate(kv_new):
        if len(cache.k) <= l:
            cache.k.append(k)
            cache.v.append(v)
        else:
            cache.k[l] = np.concatenate([cache.k[l], k], axis=1)
            cache.v[l] = np.concatenate([cache.v[l], v], axis=1)
    return cache


def causal_encode(cfg, weights, ids, cache):
    """Prefill / commit: encode ids causally at positions P.. and append their K/V."""
    p = cache.length
    pos = p + np.arange(len(ids))
    _, kv_new, _ = forward_tokens(cfg, weights, ids, pos, cache, causal=True)
    return _append(cache, kv_new)


def commit_reusing_canvas_kv(cfg, weights, canvas_in, cache):
    """The commit variant that keeps the K/V the last denoise forward computed for the canvas:
    the bidirectional forward of that step's input canvas at positions P..P+T-1, appended as is
    (no causal re-encode of the committed ids).  The pages only say the block is committed to the
    cache ([canvas] step 4, [arch]); re-encoding is the default reading, this is its alternative."""
    p = cache.length
    pos = p + np.arange(len(canvas_in))
    _, kv_new, _ = forward_tokens(cfg, weights, canvas_in, pos, cache, causal=False)
    return _append(cache, kv_new)


def decode(cfg, weights, prompt_ids, n_blocks, seed, fixed_steps=None, commit="reencode"):
    """Block-autoregressive diffusion decode; returns committed ids and per-block records.

    commit="reencode" encodes each committed block causally like the prompt; "reuse_kv" keeps
    the canvas K/V of the block's last denoise step instead (commit_reusing_canvas_kv)."""
    if commit not in ("reencode", "reuse_kv"):
        raise ValueError(f"unknown commit mode {commit!r}")
    cache = KVCache()
    causal_encode(cfg, weights, prompt_ids, cache)
    blocks = []
    for b in range(n_blocks):
        res = smp.run_block(lambda t, canvas: denoise_logits(cfg, weights, canvas, cache),
                            seed, b, cfg.vocab, cfg.canvas, max_steps=cfg.max_steps,
                            fixed_steps=fixed_steps, tau=cfg.tau, h_bound=cfg.h_bound)
        if commit == "reencode":
            causal_encode(cfg, weights, res["committed"], cache)
        else:
            last = res["steps"][res["stop_step"] - 1]
            commit_reusing_canvas_kv(cfg, weights, last["canvas_in"], cache)
        blocks.append(res)
    out = np.concatenate([b["committed"] for b in blocks]) if blocks else np.zeros(0, np.int64)
    return out, blocks, cache


def decode_batch(cfg, weights, prompts, n_blocks, seed, fixed_steps=None, commit="reencode"):
    """Small-batch canvases: B sequences decoded in lockstep, one canvas each per denoise step.

    The pages only say the method's advantage is strongest at small-to-medium batch on one
    accelerator; the plainest reading keeps the sequences independent: sequence b is the
    single-sequence decode of prompts[b] whose Philox stream has key seed + b.  Lockstep (every
    canvas commits once all have stopped; a stopped canvas is frozen meanwhile) changes no
    sequence's result, because a stopped canvas's committed block is fixed at its stop step.
    Returns a list of decode() results."""
    return [decode(cfg, weights, np.asarray(p), n_blocks, seed + b, fixed_steps, commit)
            for b, p in enumerate(prompts)]
