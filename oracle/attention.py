"""Canvas attention and causal (prefill/commit) attention, written as the definition.

Denoising ([uniform], [arch]): every canvas query attends to the whole committed
history in the KV cache and to every canvas position, with no mask.  Prefill and
commit ([arch], [canvas] step 1 and step 4) use causal attention: a new token at
absolute position P+i sees the history [0, P) and the new tokens P..P+i.

Grouped-query attention: query head j reads key/value head j // (Hq / Hkv).
Each (head, query) row is a full float64 softmax over its visible keys followed
by the probability-weighted sum of values (matmul used as the dot-product step).
"""
import numpy as np


def attention(q, k, v, scale, causal_prefix=None):
    """q [Hq, T, hd]; k, v [Hkv, N, hd]; returns o [Hq, T, hd] in float64.

    causal_prefix=None: no mask (denoise).  causal_prefix=P: key n is visible to
    query i iff n <= P + i (keys 0..P-1 are the committed history, keys P.. are the
    new tokens in order).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    hq, t, hd = q.shape
    hkv, n, _ = k.shape
    if hq % hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    group = hq // hkv
    out = np.zeros((hq, t, hd), dtype=np.float64)
    if causal_prefix is not None:
        visible = np.arange(n)[None, :] <= (causal_prefix + np.arange(t))[:, None]
    for j in range(hq):
        g = j // group
        s = (q[j] @ k[g].T) * scale  # [T, N]
        if causal_prefix is not None:
            s = np.where(visible, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        p = e / e.sum(axis=1, keepdims=True)
        out[j] = p @ v[g]
    return out
