"""Shared helpers for the parity tests (comparison rules and tensor conversion)."""
import numpy as np
import torch


def np64(t):
    """torch tensor (any device/dtype) -> float64 numpy (exact for bf16/fp32)."""
    return t.detach().to("cpu", torch.float64).numpy()


def npf32(t):
    return t.detach().to("cpu", torch.float32).numpy()


def rel_close(got, ref, rtol):
    """Elementwise |got - ref| <= rtol * (|ref| + rms(ref)); returns (ok, worst ratio, norm rel err)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    bound = rtol * (np.abs(ref) + rms)
    err = np.abs(got - ref)
    worst = float(np.max(err / np.maximum(bound, 1e-300))) if ref.size else 0.0
    nrel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    return bool(np.all(err <= bound)), worst, nrel


def weights_to_np(w):
    """Synthetic weight dict (torch) -> the oracle's numpy (float32 holds bf16 exactly)."""
    def cv(t):
        return None if t is None else npf32(t)
    out = dict(embed=cv(w["embed"]), final_norm=cv(w["final_norm"]), layers=[])
    for lw in w["layers"]:
        out["layers"].append({k: cv(v) for k, v in lw.items()})
    return out


def check_layer_parts(model, ocfg, lw, x_in, positions, cache_k, cache_v, layer, top_k,
                      causal=False, rtol=2e-2):
    """Teacher-forced parity of one layer, half by half, from identical inputs.

    Attention half: x_in -> x_attn on both sides.  MoE half: the GPU's own x_attn goes into both
    the GPU and the oracle, so the router sees (nearly) identical logits: routing must match as a
    set of experts except where the oracle's k-th and (k+1)-th router logits lie within 1e-3
    (then either set is valid), and every token with a matching set must match in value.
    Returns (x_attn parity, x_out parity, fraction of tokens with matching routing).
    """
    import torch
    from oracle import model as om
    x1_ref, _, _, _ = om.attention_block(ocfg, lw, x_in, positions, cache_k, cache_v, causal)
    x1_gpu = model.debug_layer_part(layer, 0, torch.from_numpy(np.asarray(x_in, np.float32)).cuda(),
                                    causal)
    x1 = np64(x1_gpu)
    att = rel_close(x1, x1_ref, rtol)
    x2_ref, info = om.moe_block(ocfg, lw, x1)
    x2_gpu = model.debug_layer_part(layer, 1, x1_gpu.contiguous(), causal)
    ids_g, _, _ = model.debug_routing(n=x1.shape[0])
    torch.cuda.synchronize()
    same = np.array_equal
    g_set = np.sort(ids_g.cpu().numpy(), axis=1)
    o_set = np.sort(info["moe"]["ids"], axis=1)
    match = np.all(g_set == o_set, axis=1)
    srt = -np.sort(-info["moe"]["router_logits"], axis=1)
    gap = srt[:, top_k - 1] - srt[:, top_k] if top_k < srt.shape[1] else np.full(len(srt), np.inf)
    assert np.all(gap[~match] < 1e-3), ("routing set differs away from a near-tie", layer,
                                        gap[~match])
    moe = rel_close(np64(x2_gpu)[match], x2_ref[match], rtol)
    return att, moe, float(match.mean())


def router_gaps(ocfg, ow, ids, pos, cache, causal=True):
    """Oracle top-k router margin (k-th minus (k+1)-th logit) of every token at every layer of a
    pass over ids (causal, or bidirectional like a denoise step): [n_layers, n]."""
    from oracle import model as om
    _, _, infos = om.forward_tokens(ocfg, ow, ids, pos, cache, causal=causal, keep_info=True)
    k = ocfg.top_k
    out = []
    for info in infos:
        srt = -np.sort(-info["moe"]["router_logits"], axis=1)
        out.append(srt[:, k - 1] - srt[:, k] if k < srt.shape[1] else np.full(len(srt), np.inf))
    return np.array(out)


# Router near-ties.  Teacher-forced (the GPU's own attention output feeds both sides' MoE half):
# the two sides' router inputs differ only by the re-rounding of the RMSNorm output, margins
# below 1e-3 may flip.  Untethered forward passes (prefill, commit, denoise over the GPU's own
# activations): the bf16 storage of the attention output and of the normed hidden state lets the
# router input differ by up to half a bf16 step per element, i.e. a router-logit change of
# standard deviation 2^-9 / sqrt(3) * ||w_r|| ~ 5e-4 for the test models (||w_r|| = 0.02 sqrt(512));
# margins below ten of those, 5e-3, may flip.
NEAR_TIE = 1e-3
NEAR_TIE_FORWARD = 5e-3


def kv_tokens_close(got, ref, gaps, layer, rtol, near_tie=NEAR_TIE_FORWARD):
    """Per-token parity of a K (or V) slice [H, n, hd] of `layer`.

    In these two-layer models a token's layer-1 K/V depend on the layer-0 K/V of the tokens it
    attends to (functions of their embeddings only) and on its own layer-0 MoE routing.  Where the
    oracle's top-k margin of that token at an earlier layer is below `near_tie` the GPU may
    legitimately route it to another expert and its K/V differ.  Every other token must be within
    rtol.  Returns (ok, the offending tokens with their smallest earlier margin, count of excused
    tokens that differ)."""
    got = np.asarray(got)
    ref = np.asarray(ref)
    n = ref.shape[1]
    good = np.array([rel_close(got[:, j], ref[:, j], rtol)[0] for j in range(n)])
    earlier = gaps[:layer].min(axis=0) if layer else np.full(n, np.inf)
    excused = earlier < near_tie
    bad = np.nonzero(~good & ~excused)[0]
    return bad.size == 0, [(int(j), float(earlier[j])) for j in bad[:8]], int((~good & excused).sum())
