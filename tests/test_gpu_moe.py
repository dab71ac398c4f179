"""Parity of the MoE path (router GEMM, top-k, permutation, grouped tcgen05 GEMMs, combine)."""
import numpy as np
import pytest
import torch

from dg_synth import moe_inputs
from oracle.moe import moe_ffn as o_moe
from tests._helpers import np64, npf32, rel_close

pytestmark = pytest.mark.gpu
RTOL = 2e-2


def _case(t, d, e, k, h, hs, seed):
    from block_text_diffusion_dg_b200 import moe_ffn
    m = moe_inputs(t, d, e, h, hs, seed=seed)
    dev = {kk: (None if v is None else v.cuda()) for kk, v in m.items()}
    ids = torch.empty(t, k, dtype=torch.int32, device="cuda")
    wts = torch.empty(t, k, dtype=torch.float32, device="cuda")
    rl = torch.empty(t, e, dtype=torch.float32, device="cuda")
    y = moe_ffn(dev["x"], dev["wr"], dev["w_gu"], dev["w_d"], k, dev["ws_gu"], dev["ws_d"],
                ids=ids, weights=wts, router_logits=rl)
    torch.cuda.synchronize()
    shared = None if hs == 0 else (npf32(m["ws_gu"]), npf32(m["ws_d"]))
    y_ref, info = o_moe(np64(m["x"]), npf32(m["wr"]), npf32(m["w_gu"]), npf32(m["w_d"]), k, "bf16",
                        shared)
    g_logits = rl.cpu().numpy().astype(np.float64)
    ok, worst, _ = rel_close(g_logits, info["router_logits"], 1e-4)
    assert ok, worst
    # integer routing is bit-exact given identical logits ...
    g_ids = ids.cpu().numpy()
    topk_from_gpu_logits = np.argsort(-g_logits.astype(np.float32), axis=1, kind="stable")[:, :k]
    assert np.array_equal(g_ids, topk_from_gpu_logits)
    # ... and equal to the oracle's wherever the k-th / (k+1)-th logit gap is outside the guard
    srt = -np.sort(-info["router_logits"], axis=1)
    gap = srt[:, k - 1] - srt[:, k] if k < e else np.full(t, np.inf)
    clear = gap > 1e-3
    assert np.array_equal(g_ids[clear], info["ids"][clear])
    w_ref = info["weights"]
    assert np.max(np.abs(wts.cpu().numpy()[clear] - w_ref[clear])) < 1e-5
    same = np.all(g_ids == info["ids"], axis=1)
    ok, worst, nrel = rel_close(y.cpu().numpy()[same], y_ref[same], RTOL)
    assert ok, (worst, nrel)
    assert nrel < 5e-3
    return same.mean()


@pytest.mark.parametrize("t,d,e,k,h,hs", [
    (64, 256, 8, 2, 128, 0),         # tiny, no shared expert
    (256, 512, 8, 2, 256, 384),      # the small test model's MoE
    (200, 512, 16, 4, 192, 256),     # ragged token count
    (256, 1024, 128, 8, 64, 128),    # many experts, many empty
    (1100, 512, 16, 4, 128, 256),    # several router chunks; experts with several token chunks
    (2048, 256, 128, 8, 64, 0),      # a long prompt pass: 16 384 routed slots
    (4096, 256, 8, 2, 64, 0),        # the largest pass: routing over 4096 tokens
])
def test_moe_small(t, d, e, k, h, hs):
    assert _case(t, d, e, k, h, hs, seed=t + d) > 0.95


def test_moe_full_size():
    # 256 tokens, d 2816, 128 experts top-8 (SiLU-GLU 704) + shared expert 2112
    assert _case(256, 2816, 128, 8, 704, 2112, seed=0) > 0.95


def test_moe_residual_is_added():
    from block_text_diffusion_dg_b200 import moe_ffn
    m = moe_inputs(32, 256, 8, 128, 0, seed=4)
    dev = {kk: (None if v is None else v.cuda()) for kk, v in m.items()}
    r = torch.randn(32, 256, device="cuda")
    y0 = moe_ffn(dev["x"], dev["wr"], dev["w_gu"], dev["w_d"], 2)
    y1 = moe_ffn(dev["x"], dev["wr"], dev["w_gu"], dev["w_d"], 2, residual=r)
    torch.cuda.synchronize()
    assert torch.allclose(y1 - r, y0, atol=1e-5, rtol=0)
