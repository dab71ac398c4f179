"""Pins for the oracle's canvas (no mask) and causal attention."""
import numpy as np
import pytest
import torch

from oracle.attention import attention


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_single_key_returns_its_value():
    q, k, v = _rand((2, 5, 8), 0), _rand((1, 1, 8), 1), _rand((1, 1, 8), 2)
    o = attention(q, k, v, 0.3)
    assert np.allclose(o, np.broadcast_to(v[0, 0], o.shape), atol=1e-15)


def test_zero_query_and_identical_keys_give_mean_value():
    v = _rand((2, 7, 4), 3)
    o = attention(np.zeros((2, 3, 4)), _rand((2, 7, 4), 4), v, 1.0)
    assert np.allclose(o, v.mean(axis=1)[:, None, :], atol=1e-14)
    k = np.repeat(_rand((2, 1, 4), 5), 7, axis=1)
    o = attention(_rand((2, 3, 4), 6), k, v, 1.0)
    assert np.allclose(o, v.mean(axis=1)[:, None, :], atol=1e-14)


def test_gqa_equals_mha_with_repeated_kv():
    q, k, v = _rand((8, 6, 16), 7), _rand((2, 11, 16), 8), _rand((2, 11, 16), 9)
    o = attention(q, k, v, 0.25)
    o2 = attention(q, np.repeat(k, 4, axis=0), np.repeat(v, 4, axis=0), 0.25)
    assert np.allclose(o, o2, atol=1e-14)


def test_key_permutation_invariance_without_mask():
    q, k, v = _rand((4, 6, 16), 10), _rand((2, 13, 16), 11), _rand((2, 13, 16), 12)
    perm = np.random.default_rng(13).permutation(13)
    assert np.allclose(attention(q, k, v, 0.5), attention(q, k[:, perm], v[:, perm], 0.5), atol=1e-13)


@pytest.mark.parametrize("prefix", [None, 0, 9])
def test_against_torch_sdpa(prefix):
    hq, hkv, t, hd = 8, 2, 6, 32
    n = (prefix or 0) + t if prefix is not None else 15
    q, k, v = _rand((hq, t, hd), 14), _rand((hkv, n, hd), 15), _rand((hkv, n, hd), 16)
    o = attention(q, k, v, hd ** -0.5, causal_prefix=prefix)
    mask = None
    if prefix is not None:
        mask = torch.from_numpy(np.arange(n)[None, :] <= (prefix + np.arange(t))[:, None])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(np.repeat(k, hq // hkv, 0))[None],
        torch.from_numpy(np.repeat(v, hq // hkv, 0))[None], attn_mask=mask, scale=hd ** -0.5)[0].numpy()
    assert np.allclose(o, ref, atol=1e-12)


def test_causal_first_new_token_sees_prefix_and_itself():
    q, k, v = _rand((1, 4, 8), 17), _rand((1, 7, 8), 18), _rand((1, 7, 8), 19)
    o = attention(q, k, v, 1.0, causal_prefix=3)
    o_first = attention(q[:, :1], k[:, :4], v[:, :4], 1.0)
    assert np.allclose(o[:, :1], o_first, atol=1e-15)
    # the last new token sees everything
    assert np.allclose(o[:, 3:], attention(q[:, 3:], k, v, 1.0), atol=1e-15)
