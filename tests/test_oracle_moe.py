"""Pins for the oracle's router and mixture-of-experts FFN."""
import numpy as np
import torch

from oracle.moe import expert_glu, moe_ffn, router


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def _torch_glu(x, wg, wu, wd):
    x, wg, wu, wd = (torch.from_numpy(a) for a in (x, wg, wu, wd))
    return (torch.nn.functional.silu(x @ wg.T) * (x @ wu.T)) @ wd.T


def test_single_expert_is_dense_glu():
    x, wgu, wd = _rand((9, 16), 0), _rand((1, 24, 16), 1, 0.3), _rand((1, 16, 12), 2, 0.3)
    y, info = moe_ffn(x, _rand((1, 16), 3), wgu, wd, 1, "fp32")
    assert np.all(info["ids"] == 0) and np.allclose(info["weights"], 1.0)
    ref = _torch_glu(x, wgu[0][0::2], wgu[0][1::2], wd[0]).numpy()
    assert np.allclose(y, ref, rtol=1e-6, atol=1e-6)  # h is rounded to fp32 storage


def test_router_topk_and_weights():
    x, wr = _rand((64, 32), 4), _rand((16, 32), 5)
    logits, ids, w = router(x, wr, 4)
    for t in range(64):
        sel = logits[t, ids[t]]
        rest = np.delete(logits[t], ids[t])
        assert sel.min() >= rest.max()
        assert np.all(np.diff(sel) <= 0)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-14) and (w > 0).all()
    # weights are the top-k probabilities of the full softmax, renormalised
    p = torch.softmax(torch.from_numpy(logits), dim=1).numpy()
    sel = np.take_along_axis(p, ids, 1)
    assert np.allclose(w, sel / sel.sum(1, keepdims=True), atol=1e-14)


def test_router_ties_take_lowest_index():
    x = np.ones((1, 4))
    wr = np.zeros((6, 4))
    wr[[1, 3, 4], :] = 0.5  # three experts tie at the top
    _, ids, w = router(x, wr, 2)
    assert ids.tolist() == [[1, 3]] and np.allclose(w, 0.5)


def test_k_equal_e_is_softmax_mixture():
    x = _rand((5, 8), 6)
    wr, wgu, wd = _rand((3, 8), 7), _rand((3, 10, 8), 8, 0.4), _rand((3, 8, 5), 9, 0.4)
    y, info = moe_ffn(x, wr, wgu, wd, 3, "fp32")
    p = torch.softmax(torch.from_numpy(info["router_logits"]), 1).numpy()
    ref = sum(p[:, e:e + 1] * _torch_glu(x, wgu[e][0::2], wgu[e][1::2], wd[e]).numpy() for e in range(3))
    assert np.allclose(y, ref, rtol=1e-6, atol=1e-6)


def test_expert_permutation_leaves_output_unchanged():
    x = _rand((12, 8), 10)
    wr, wgu, wd = _rand((6, 8), 11), _rand((6, 10, 8), 12, 0.4), _rand((6, 8, 5), 13, 0.4)
    perm = np.random.default_rng(14).permutation(6)
    y1, i1 = moe_ffn(x, wr, wgu, wd, 2, "fp32")
    y2, i2 = moe_ffn(x, wr[perm], wgu[perm], wd[perm], 2, "fp32")
    assert np.allclose(y1, y2, atol=1e-12)
    assert np.array_equal(perm[i2["ids"]], i1["ids"])


def test_shared_expert_adds_dense_glu():
    x = _rand((7, 8), 15)
    wr, wgu, wd = _rand((4, 8), 16), _rand((4, 10, 8), 17, 0.4), _rand((4, 8, 5), 18, 0.4)
    sgu, sd = _rand((12, 8), 19, 0.4), _rand((8, 6), 20, 0.4)
    y0, _ = moe_ffn(x, wr, wgu, wd, 2, "fp32")
    y1, _ = moe_ffn(x, wr, wgu, wd, 2, "fp32", shared=(sgu, sd))
    ref = _torch_glu(x, sgu[0::2], sgu[1::2], sd).numpy()
    assert np.allclose(y1 - y0, ref, rtol=1e-6, atol=1e-6)


def test_expert_h_is_rounded_to_storage():
    x, wgu, wd = _rand((3, 8), 21), _rand((6, 8), 22), _rand((8, 3), 23)
    _, h = expert_glu(x, wgu, wd, "bf16")
    assert np.array_equal(h, torch.from_numpy(h).to(torch.bfloat16).double().numpy())
