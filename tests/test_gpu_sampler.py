"""Parity of the canvas sampler (statistics, lock/re-noise, stop rule) against the oracle."""
import math

import numpy as np
import pytest
import torch

from dg_synth import planted_normal, sampler_logits
from oracle import sampler as osmp
from tests._helpers import np64

pytestmark = pytest.mark.gpu

TAU, HB = 0.9, 0.005
GUARD_CONF = 1e-4


def _gpu_sampler(rows, vocab):
    from block_text_diffusion_dg_b200 import Sampler
    s = Sampler(rows, vocab)
    s.reset()
    return s


def _check_step(s, logits_cpu, seed, block, step):
    conf, ent, amax = osmp.row_stats(np64(logits_cpu))
    nxt, locked = osmp.sample_update(conf, amax, seed, block, step, logits_cpu.shape[1], TAU)
    torch.cuda.synchronize()
    g_amax = s.argmax.cpu().numpy()
    g_ent = s.entropy.cpu().numpy().astype(np.float64)
    g_conf = s.conf.cpu().numpy().astype(np.float64)
    g_canvas = s.canvas.cpu().numpy()
    assert np.array_equal(g_amax, amax), "argmax must be bit-exact (lowest index on ties)"
    assert np.max(np.abs(g_ent - ent)) <= 1e-5, np.max(np.abs(g_ent - ent))
    assert np.max(np.abs(g_conf - conf) / conf) <= 1e-5
    outside = np.abs(conf - TAU) >= GUARD_CONF
    assert np.array_equal(g_canvas[outside], nxt[outside])
    # inside the guard band either decision is valid, but the id must be one of the two choices
    from oracle.philox import uniform_ids
    for i in np.nonzero(~outside)[0]:
        draw = int(uniform_ids(seed, block, step, [i], 1, logits_cpu.shape[1])[0])
        assert g_canvas[i] in (int(amax[i]), draw)
    return conf, ent, amax, outside


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,vocab", [(5, 20000), (3, 8), (64, 8192 * 3 + 8)])
def test_sampler_small_ragged(rows, vocab, dtype):
    logits = sampler_logits(rows, vocab, seed=rows + vocab).to(dtype)
    s = _gpu_sampler(rows, vocab)
    s.step(logits.cuda(), seed=77, block=2, step=1)
    _check_step(s, logits, 77, 2, 1)


def test_sampler_exact_ties_take_lowest_index():
    rows, vocab = 4, 16384
    x = torch.zeros(rows, vocab, dtype=torch.bfloat16)
    x[0, [5, 9000, 16383]] = 3.0     # ties across slices
    x[1, [8191, 8192]] = 2.0         # tie straddling the slice boundary
    x[2, :] = 1.0                    # all equal: argmax 0, entropy ln V
    x[3, 16383] = 100.0              # one certain token at the very end
    s = _gpu_sampler(rows, vocab)
    s.step(x.cuda(), seed=1, block=0, step=1)
    _check_step(s, x, 1, 0, 1)
    torch.cuda.synchronize()
    assert s.argmax.cpu().tolist() == [5, 8191, 0, 16383]
    assert abs(float(s.entropy[2]) - math.log(vocab)) < 1e-5
    assert int(s.canvas[3]) == 16383  # conf ~ 1 locks


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_sampler_ties_and_masked_entries_at_lane_and_segment_edges(dtype):
    """Each warp streams groups of 8 vectors per lane (2048 bf16 / 1024 fp32 columns, one row
    segment) and finds a lane's first maximal column only at the end, in the group where the lane
    met its maximum: ties between lanes, within a lane's vector, across a lane's groups and across
    segment edges must all give the lowest column; -inf (masked) entries contribute nothing."""
    rows, vocab = 8, 3 * 4096 + 8
    x = sampler_logits(rows, vocab, seed=11).to(dtype)
    top = float(x.float().max()) + 4.0
    x[0, [100, 40]] = top               # two lanes of one group
    x[1, [8 + 2048, 8]] = top           # one lane meets its maximum again two groups later
    x[2, [17, 16]] = top                # two maxima in one lane's vector
    x[3, [2048, 2047]] = top            # bf16 group / segment edge
    x[4, [1024, 1023]] = top            # fp32 group / segment edge
    x[5, ::3] = -math.inf               # masked entries around the maximum
    x[5, 4000] = top
    x[6, :] = -math.inf                 # only two entries unmasked
    x[6, 5], x[6, vocab - 1] = 1.0, 2.0
    x[7, vocab - 8:] = top              # the maximum in the ragged end of the row
    s = _gpu_sampler(rows, vocab)
    s.step(x.cuda(), seed=4, block=0, step=1)
    _check_step(s, x, 4, 0, 1)
    torch.cuda.synchronize()
    assert s.argmax.cpu().tolist() == [40, 8, 16, 2047, 1023, 4000, vocab - 1, vocab - 8]
    assert abs(float(s.conf[6]) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-6


def test_sampler_full_size_stats():
    logits = sampler_logits(256, 262144, seed=0)
    s = _gpu_sampler(256, 262144)
    s.step(logits.cuda(), seed=0, block=0, step=1)
    conf, ent, amax, outside = _check_step(s, logits, 0, 0, 1)
    assert outside.sum() >= 250  # the guard band holds almost no rows


def _ramp(t):
    return 0.5 * 1.12 ** t


def _step_logits(z, s_row, t, device):
    return (z.to(device) * s_row.to(device)[:, None] * _ramp(t)).to(torch.bfloat16)


def test_sampler_stop_sequence_full_size():
    """48-step logit sequence with a fixed planted argmax and rising scale: it stops at the first
    step whose mean entropy is below 0.005 (the argmax never changes)."""
    rows, vocab = 256, 262144
    z, u = planted_normal(rows, vocab, seed=5)
    s_row = torch.exp(math.log(0.5) + u * (math.log(40.0) - math.log(0.5)))
    # oracle: mean entropy falls monotonically along the ramp; bisect for the first t below HB
    cache = {}

    def hbar(t):
        if t not in cache:
            cache[t] = float(osmp.row_stats(np64(_step_logits(z, s_row, t, "cpu")))[1].mean())
        return cache[t]

    lo, hi = 1, 48
    assert hbar(hi) < HB and hbar(lo) > HB
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if hbar(mid) < HB:
            hi = mid
        else:
            lo = mid
    t_stop = max(2, hi)
    assert abs(hbar(hi) - HB) > 5e-5 and abs(hbar(hi - 1) - HB) > 5e-5, "crossing inside guard band"
    s = _gpu_sampler(rows, vocab)
    # the GPU path receives bit-identical logits (same fp32 arithmetic, RNE to bf16)
    x_gpu = _step_logits(z, s_row, hi, "cuda")
    assert torch.equal(x_gpu.cpu(), _step_logits(z, s_row, hi, "cpu"))
    for t in range(1, 49):
        s.step(_step_logits(z, s_row, t, "cuda"), seed=9, block=1, step=t)
    torch.cuda.synchronize()
    st = s.state.cpu().tolist()
    assert st[0] == 1 and st[1] == t_stop and st[2] == t_stop and st[3] == t_stop, st
    assert np.array_equal(s.argmax.cpu().numpy(), z.argmax(dim=1).numpy())


def test_sampler_fixed_mode_and_noop_after_done():
    rows, vocab = 16, 4096
    s = _gpu_sampler(rows, vocab)
    for t in range(1, 8):
        s.step(sampler_logits(rows, vocab, seed=t).cuda(), seed=3, block=0, step=t, fixed_steps=5)
        if t == 5:
            torch.cuda.synchronize()
            canvas5 = s.canvas.clone()
    torch.cuda.synchronize()
    st = s.state.cpu().tolist()
    assert st[0] == 1 and st[1] == 5 and st[3] == 5
    assert torch.equal(s.canvas, canvas5)  # steps 6 and 7 were no-ops
