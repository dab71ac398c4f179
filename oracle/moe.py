"""Top-k routed mixture-of-experts FFN with an optional shared expert (oracle side).

The backbone is a mixture of experts ([course] table 2.2: 26B total, 3.8B active;
[arch]: Gemma 4 26B-A4B).  The pages do not spell out the router, so the plainest
reading is used:

    logits_t = xn_t W_r^T                    (stored fp32 on the GPU path)
    p_t      = softmax(logits_t) over all E experts
    ids_t    = the k experts with the largest p_t, lowest index first on ties
    w_t,s    = p_t[ids_t,s] / sum_s' p_t[ids_t,s']

Each expert is a SiLU-gated linear unit: h = silu(xn W_g^T) * (xn W_u^T),
y = h W_d^T, with h stored in the path's storage type.  The token's output is the
weighted sum over its k slots taken in slot order, plus the shared expert
(weight 1) when there is one.

With e4m3 experts (moe_ffn_fp8) the router is unchanged and every expert GEMM takes e4m3
operands with per-row scales, as quant.py states.

Weights of the gate and up projections are stored interleaved by row,
w_gu[e][2j] = gate row j and w_gu[e][2j+1] = up row j; this is a storage layout
only and is undone here with strided views.
"""
import numpy as np

from .numerics import round_f32, round_storage
from .quant import dequantize_nvfp4, quantize_matrix, quantize_nvfp4_rows, quantize_rows


def silu(x):
    return x / (1.0 + np.exp(-x))


def router(xn, w_r, top_k):
    """Router logits (fp32-rounded), top-k expert ids and their renormalised weights."""
    logits = round_f32(np.asarray(xn, dtype=np.float64) @ np.asarray(w_r, dtype=np.float64).T)
    t, e = logits.shape
    if not 1 <= top_k <= e:
        raise ValueError("top_k must be in [1, E]")
    # stable sort on -logit keeps the lowest expert index first among equal logits;
    # softmax is strictly increasing, so ranking logits ranks probabilities.
    order = np.argsort(-logits, axis=1, kind="stable")
    ids = order[:, :top_k].astype(np.int64)
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    p = p / p.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, ids, axis=1)
    w = sel / sel.sum(axis=1, keepdims=True)
    return logits, ids, w


def expert_glu(xn, w_gu, w_d, storage):
    """One SiLU-GLU expert on rows xn [n, d]; w_gu [2h, d] row-interleaved, w_d [d, h]."""
    xn = np.asarray(xn, dtype=np.float64)
    w_gu = np.asarray(w_gu, dtype=np.float64)
    g = xn @ w_gu[0::2].T
    u = xn @ w_gu[1::2].T
    h = round_storage(silu(g) * u, storage)
    return h @ np.asarray(w_d, dtype=np.float64).T, h


def moe_ffn(xn, w_r, w_gu, w_d, top_k, storage, shared=None):
    """MoE output (without the residual) for tokens xn [T, d].

    w_gu [E, 2h, d], w_d [E, d, h]; shared = (ws_gu [2hs, d], ws_d [d, hs]) or None.
    Each token's expert outputs are the rows of per-expert products; every row is
    the same per-token computation, so gathering a token's rows does not reorder
    any token's arithmetic.  Returns (y [T, d] float64, dict of intermediates).
    """
    xn = np.asarray(xn, dtype=np.float64)
    t, d = xn.shape
    logits, ids, w = router(xn, w_r, top_k)
    y_slot = np.zeros((t, top_k, d), dtype=np.float64)
    for e in np.unique(ids):
        rows, slots = np.nonzero(ids == e)
        ye, _ = expert_glu(xn[rows], w_gu[e], w_d[e], storage)
        y_slot[rows, slots] = ye
    y = np.zeros((t, d), dtype=np.float64)
    for s in range(top_k):  # slot order 0..k-1
        y = y + w[:, s:s + 1] * y_slot[:, s]
    ys = None
    if shared is not None:
        ys, _ = expert_glu(xn, shared[0], shared[1], storage)
        y = y + ys
    return y, dict(router_logits=logits, ids=ids, weights=w, y_slot=y_slot, y_shared=ys)


# ---- e4m3 experts (the FP8 weight format; scheme and readings in quant.py) -------------------

def gate_up_fp8(xq, xs, gu_q, gu_s):
    """SiLU-GLU hidden h [n, hid] (bf16-stored) from e4m3 activations and gate/up weights.

    xq [n, d] e4m3 values with row scales xs [n]; gu_q [2hid, d] row-interleaved e4m3 values
    with row scales gu_s [2hid].  Sums of code products are scaled by (row scale) x (token scale).
    """
    acc = np.asarray(xq, dtype=np.float64) @ np.asarray(gu_q, dtype=np.float64).T
    gu = acc * np.asarray(gu_s, dtype=np.float64)[None, :] * np.asarray(xs, dtype=np.float64)[:, None]
    return round_storage(silu(gu[:, 0::2]) * gu[:, 1::2], "bf16")


def down_fp8(h, d_q, d_s):
    """Down projection of h [n, hid] (quantised per row here) with e4m3 weights d_q [d, hid]."""
    hq, hs = quantize_rows(h)
    acc = hq @ np.asarray(d_q, dtype=np.float64).T
    return acc * np.asarray(d_s, dtype=np.float64)[None, :] * hs.astype(np.float64)[:, None]


def moe_ffn_fp8(xn, w_r, w_gu, w_d, top_k, shared=None):
    """MoE output with e4m3 experts: the router as in moe_ffn (bf16 weights), then every expert
    (and the shared one) quantised row by row from the given weights, the token rows quantised
    once, and each expert's h quantised per token-slot.  Returns (y [T, d], intermediates)."""
    xn = np.asarray(xn, dtype=np.float64)
    t, d = xn.shape
    logits, ids, w = router(xn, w_r, top_k)
    xq, xs = quantize_rows(xn)
    y_slot = np.zeros((t, top_k, d), dtype=np.float64)
    for e in np.unique(ids):
        rows, slots = np.nonzero(ids == e)
        gq, gs = quantize_matrix(w_gu[e])
        dq, ds = quantize_matrix(w_d[e])
        h = gate_up_fp8(xq[rows], xs[rows], gq, gs)
        y_slot[rows, slots] = down_fp8(h, dq, ds)
    y = np.zeros((t, d), dtype=np.float64)
    for s in range(top_k):  # slot order 0..k-1
        y = y + w[:, s:s + 1] * y_slot[:, s]
    ys = None
    if shared is not None:
        gq, gs = quantize_matrix(shared[0])
        dq, ds = quantize_matrix(shared[1])
        ys = down_fp8(gate_up_fp8(xq, xs, gq, gs), dq, ds)
        y = y + ys
    return y, dict(router_logits=logits, ids=ids, weights=w, y_slot=y_slot, y_shared=ys,
                   x_codes=xq, x_scales=xs)


# ---- NVFP4 experts (e2m1 elements, e4m3 block scales, fp32 row scales; see quant.py) ---------

def _nvfp4(v):
    """Dequantised NVFP4 image of the rows of v (float64)."""
    return dequantize_nvfp4(*quantize_nvfp4_rows(v))


def gate_up_nvfp4(x, gu):
    """SiLU-GLU hidden (bf16-stored) from NVFP4-quantised token rows x [n, d] and gate/up rows
    gu [2hid, d] (row-interleaved): the sums of dequantised products, exact in float64."""
    acc = _nvfp4(x) @ _nvfp4(gu).T
    return round_storage(silu(acc[:, 0::2]) * acc[:, 1::2], "bf16")


def down_nvfp4(h, w_d):
    """Down projection of h [n, hid] (NVFP4-quantised per row here) with NVFP4 weights [d, hid]."""
    return _nvfp4(h) @ _nvfp4(w_d).T


def moe_ffn_nvfp4(xn, w_r, w_gu, w_d, top_k, shared=None):
    """MoE output with NVFP4 experts: the router as in moe_ffn (bf16 weights); expert weights,
    the token rows and each expert's h quantised to NVFP4 row by row."""
    xn = np.asarray(xn, dtype=np.float64)
    t, d = xn.shape
    logits, ids, w = router(xn, w_r, top_k)
    y_slot = np.zeros((t, top_k, d), dtype=np.float64)
    for e in np.unique(ids):
        rows, slots = np.nonzero(ids == e)
        h = gate_up_nvfp4(xn[rows], w_gu[e])
        y_slot[rows, slots] = down_nvfp4(h, w_d[e])
    y = np.zeros((t, d), dtype=np.float64)
    for s in range(top_k):  # slot order 0..k-1
        y = y + w[:, s:s + 1] * y_slot[:, s]
    ys = None
    if shared is not None:
        ys = down_nvfp4(gate_up_nvfp4(xn, shared[0]), shared[1])
        y = y + ys
    return y, dict(router_logits=logits, ids=ids, weights=w, y_slot=y_slot, y_shared=ys)
