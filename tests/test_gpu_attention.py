"""Parity of the tcgen05 canvas attention against the oracle's naive attention."""
import numpy as np
import pytest
import torch

from dg_synth import attention_inputs
from oracle.attention import attention as o_attention
from oracle.numerics import round_bf16
from tests._helpers import np64, rel_close

pytestmark = pytest.mark.gpu
RTOL = 2e-2


def _case(hq, hkv, t, tq, prefix, causal, seed):
    from block_text_diffusion_dg_b200 import canvas_attention
    q, k, v = attention_inputs(hq, hkv, canvas=tq, prefix=prefix, head_dim=128, seed=seed)
    pad = (-k.shape[1]) % 8  # key stride must be a multiple of 8 (16-byte TMA rows)
    if pad:
        k = torch.cat([k, torch.zeros(hkv, pad, 128, dtype=k.dtype)], dim=1)
        v = torch.cat([v, torch.zeros(hkv, pad, 128, dtype=v.dtype)], dim=1)
    ldk = k.shape[1]
    n_keys = prefix + t
    vt = v.transpose(1, 2).contiguous()
    o = canvas_attention(q.cuda(), k.cuda(), vt.cuda(), n_keys, causal_prefix=prefix if causal else -1,
                         n_queries=t)
    torch.cuda.synchronize()
    ref = o_attention(np64(q[:, :t]), np64(k[:, :n_keys]), np64(v[:, :n_keys]), 128 ** -0.5,
                      causal_prefix=prefix if causal else None)
    ref = round_bf16(ref.transpose(1, 0, 2).reshape(t, hq * 128))
    ok, worst, nrel = rel_close(np64(o), ref, RTOL)
    assert ok, (worst, nrel)
    assert nrel < 5e-3
    return nrel


@pytest.mark.parametrize("hq,hkv,t,tq,prefix,causal", [
    (2, 1, 128, 128, 0, False),      # one tile of keys, one query tile
    (4, 2, 256, 256, 100, False),    # ragged key tail (356 keys)
    (4, 4, 200, 256, 0, True),       # causal prefill from an empty cache, ragged queries
    (2, 1, 256, 256, 300, True),     # causal commit after a 300-token history
    (8, 2, 256, 256, 1000, False),   # group of 4 query heads per kv head
])
def test_attention_small(hq, hkv, t, tq, prefix, causal):
    _case(hq, hkv, t, tq, prefix, causal, seed=hq * 7 + prefix)


def test_attention_full_size_denoise():
    # 16 query heads, 8 kv heads, 4096 committed + 256 canvas keys, no mask
    _case(16, 8, 256, 256, 4096, False, seed=0)


def test_attention_full_size_commit():
    _case(16, 8, 256, 256, 4096, True, seed=1)


def test_attention_single_key_returns_value():
    from block_text_diffusion_dg_b200 import canvas_attention
    q, k, v = attention_inputs(2, 1, canvas=128, prefix=0, head_dim=128, seed=3)
    vt = v.transpose(1, 2).contiguous()
    o = canvas_attention(q.cuda(), k.cuda(), vt.cuda(), 1, n_queries=128)
    torch.cuda.synchronize()
    exp = np.broadcast_to(np64(v[0, 0]), (128, 2, 128)).reshape(128, 256)
    assert np.array_equal(np64(o), exp)
