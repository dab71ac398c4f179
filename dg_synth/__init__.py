"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and fixes shapes; it contains none of the
denoise path's arithmetic.  Both the CUDA library's callers and the CPU oracle
receive the tensors made here, so the two sides see identical inputs.

Recipes (the pages give no dataset; these stand in for their workloads, a
4,096-token prompt, 1,024 output tokens in 256-token canvases, and a
26B-total / ~3.8B-active MoE):
  * weights ~ N(0, 0.02), stored bf16 (fp32 for the all-fp32 shape);
    RMSNorm weights are 1 unless `norm_jitter` > 0 (then 1 + N(0, jitter));
  * activations and attention inputs ~ N(0, 1);
  * prompt ids uniform over the vocabulary;
  * sampler logits: row i is N(0,1) * s_i with s_i log-uniform in [0.5, 40];
  * quantiser inputs (scaled_rows): N(0,1) rows with per-row powers of two over 2^+-30.
"""
import math

import torch

# Model shapes.  Field names follow the pages' notation where they have one.
SHAPES = {
    # two-layer all-fp32 model used for end-to-end correctness
    "tiny_fp32": dict(n_layers=2, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64, n_experts=8,
                      top_k=2, expert_hidden=512, shared_hidden=0, vocab=4096, canvas=256,
                      storage="fp32", prompt=128),
    # small bf16 model with the production kernels' tile constraints (hd 128, d % 64 == 0)
    "small_bf16": dict(n_layers=2, d_model=512, n_heads=4, n_kv_heads=2, head_dim=128, n_experts=8,
                       top_k=2, expert_hidden=256, shared_hidden=384, vocab=8192, canvas=256,
                       storage="bf16", prompt=320),
    # Gemma-4-26B-A4B-like decoder: 30 layers, 128 experts top-8, V = 262144
    "a4b": dict(n_layers=30, d_model=2816, n_heads=16, n_kv_heads=8, head_dim=128, n_experts=128,
                top_k=8, expert_hidden=704, shared_hidden=2112, vocab=262144, canvas=256,
                storage="bf16", prompt=4096),
}


def _gen(seed, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, std, g, dtype, device):
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=g)
    return t.to(dtype)


def model_weights(shape, seed=0, device="cpu", norm_jitter=0.0, std=0.02):
    """Random-init weights for a SHAPES entry, as torch tensors on `device`.

    Layout (row-major): embed [V, d]; per layer attn_norm [d] fp32, wqkv
    [(Hq + 2 Hkv) hd, d] (q heads, then k heads, then v heads), wo [d, Hq hd],
    ffn_norm [d] fp32, wr [E, d], w_gu [E, 2h, d] with gate row j at 2j and up
    row j at 2j+1, w_d [E, d, h], ws_gu [2hs, d] (same interleave), ws_d [d, hs];
    final_norm [d] fp32.
    """
    s = SHAPES[shape] if isinstance(shape, str) else shape
    dt = torch.float32 if s["storage"] == "fp32" else torch.bfloat16
    g = _gen(seed, device)
    d, hd = s["d_model"], s["head_dim"]
    qkv_rows = (s["n_heads"] + 2 * s["n_kv_heads"]) * hd

    def norm():
        if norm_jitter > 0:
            return (1.0 + _normal((d,), norm_jitter, g, torch.float32, device)).contiguous()
        return torch.ones(d, dtype=torch.float32, device=device)

    w = dict(embed=_normal((s["vocab"], d), std, g, dt, device), layers=[])
    for _ in range(s["n_layers"]):
        lw = dict(
            attn_norm=norm(),
            wqkv=_normal((qkv_rows, d), std, g, dt, device),
            wo=_normal((d, s["n_heads"] * hd), std, g, dt, device),
            ffn_norm=norm(),
            wr=_normal((s["n_experts"], d), std, g, dt, device),
            w_gu=_normal((s["n_experts"], 2 * s["expert_hidden"], d), std, g, dt, device),
            w_d=_normal((s["n_experts"], d, s["expert_hidden"]), std, g, dt, device),
            ws_gu=None, ws_d=None,
        )
        if s["shared_hidden"]:
            lw["ws_gu"] = _normal((2 * s["shared_hidden"], d), std, g, dt, device)
            lw["ws_d"] = _normal((d, s["shared_hidden"]), std, g, dt, device)
        w["layers"].append(lw)
    w["final_norm"] = norm()
    return w


def uniform_ids(n, vocab, seed=0):
    """Token ids uniform over [0, vocab) (int32)."""
    return torch.randint(0, vocab, (n,), generator=_gen(seed), dtype=torch.int64).to(torch.int32)


def sampler_logits(rows=256, vocab=262144, seed=0, s_lo=0.5, s_hi=40.0):
    """bf16 logits [rows, vocab]: row i = N(0,1) * s_i, s_i log-uniform in [s_lo, s_hi]."""
    g = _gen(seed)
    z = torch.empty(rows, vocab).normal_(0.0, 1.0, generator=g)
    u = torch.empty(rows).uniform_(0.0, 1.0, generator=g)
    s = torch.exp(math.log(s_lo) + u * (math.log(s_hi) - math.log(s_lo)))
    return (z * s[:, None]).to(torch.bfloat16)


def planted_normal(rows, vocab, seed=0, margin=1.0):
    """N(0,1) rows [rows, vocab] fp32 whose maximum entry is raised by `margin`.

    Scaled copies of these rows keep a unique argmax, so a ramp of scales gives a
    logit sequence whose entropy falls while its argmax stays fixed.
    """
    g = _gen(seed)
    z = torch.empty(rows, vocab).normal_(0.0, 1.0, generator=g)
    idx = z.argmax(dim=1)
    z[torch.arange(rows), idx] += margin
    u = torch.empty(rows).uniform_(0.0, 1.0, generator=g)
    return z, u


def attention_inputs(n_heads=16, n_kv_heads=8, canvas=256, prefix=4096, head_dim=128, seed=0,
                     dtype=torch.bfloat16):
    """Q [Hq, T, hd]; K, V [Hkv, prefix + T, hd]; all N(0, 1)."""
    g = _gen(seed)
    q = _normal((n_heads, canvas, head_dim), 1.0, g, dtype, "cpu")
    k = _normal((n_kv_heads, prefix + canvas, head_dim), 1.0, g, dtype, "cpu")
    v = _normal((n_kv_heads, prefix + canvas, head_dim), 1.0, g, dtype, "cpu")
    return q, k, v


def moe_inputs(tokens=256, d_model=2816, n_experts=128, expert_hidden=704, shared_hidden=2112,
               seed=0, dtype=torch.bfloat16, device="cpu", std=0.02):
    """x [T, d] ~ N(0,1) and MoE weights ~ N(0, std) in the model's layout."""
    g = _gen(seed, device)
    x = _normal((tokens, d_model), 1.0, g, dtype, device)
    wr = _normal((n_experts, d_model), std, g, dtype, device)
    w_gu = _normal((n_experts, 2 * expert_hidden, d_model), std, g, dtype, device)
    w_d = _normal((n_experts, d_model, expert_hidden), std, g, dtype, device)
    ws_gu = ws_d = None
    if shared_hidden:
        ws_gu = _normal((2 * shared_hidden, d_model), std, g, dtype, device)
        ws_d = _normal((d_model, shared_hidden), std, g, dtype, device)
    return dict(x=x, wr=wr, w_gu=w_gu, w_d=w_d, ws_gu=ws_gu, ws_d=ws_d)


def scaled_rows(rows, cols, seed=0, device="cpu"):
    """bf16 rows ~ N(0,1) x 2^j with j uniform in [-30, 30] per row; for rows >= 3, row 1 is
    zero and every third element of row 2 is 2^-12 smaller than the rest (down to the e4m3
    subnormal range once the row is scaled to 448)."""
    g = _gen(seed, device)
    x = torch.empty(rows, cols, dtype=torch.float32, device=device).normal_(0.0, 1.0, generator=g)
    j = torch.randint(-30, 31, (rows, 1), generator=g, device=device).to(torch.float32)
    x = x * torch.exp2(j)
    if rows >= 3:
        x[1] = 0.0
        x[2, ::3] *= 2.0 ** -12
    return x.to(torch.bfloat16)
