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
