"""dg_sampler_step_static: the canvas sampler for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: for example code inside a host framework whose memory pool
owns the whole device budget, or a latency-critical path that may not risk cudaMalloc's implicit
device synchronisation.  This entry point keeps the sampler's temporaries and its step-to-step
stop-test state in a fixed device array inside the library instead of a caller workspace.  The
test calls it through the C ABI and compares it with dg_sampler_step (the workspace version) on
two consecutive steps of one sequence, for both logit types at the array's size limit (256 rows,
V = 262144; fp32 rows use the finer 4096-column slices, which fix the array's size):
  * "confident": every row has a unique far-ahead maximum, so every position locks and step 2
    meets the stop rule, which needs the state the first call left in the array;
  * "mixed": half the rows are flat, so those positions are re-noised from the Philox stream.
It passes alone in a fresh process and after the other tests.
"""
import ctypes as C

import pytest
import torch

from dg_synth import planted_normal

pytestmark = pytest.mark.gpu


def _p(t):
    return C.c_void_p(t.data_ptr())


def _logits(kind, rows, vocab, dtype):
    z, _ = planted_normal(rows, vocab, seed=21)
    if kind == "confident":
        x = z * 50.0
    else:  # even rows confident, odd rows flat (conf far below 0.9)
        scale = torch.where(torch.arange(rows) % 2 == 0, 50.0, 0.5)[:, None]
        x = z * scale
    return x.to(dtype).cuda()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("kind", ["confident", "mixed"])
def test_static_sampler_matches_workspace_sampler(dtype, kind):
    from block_text_diffusion_dg_b200 import Sampler
    from block_text_diffusion_dg_b200 import _lib as L
    lib = L.lib()
    rows, vocab = 256, 262144
    x = _logits(kind, rows, vocab, torch.bfloat16 if dtype == "bf16" else torch.float32)
    code = L.DTYPE_BF16 if dtype == "bf16" else L.DTYPE_FP32
    ref = Sampler(rows, vocab)
    ref.reset()
    canvas = torch.empty(rows, dtype=torch.int32, device="cuda")
    argmax = torch.empty(rows, dtype=torch.int32, device="cuda")
    entropy = torch.empty(rows, dtype=torch.float32, device="cuda")
    conf = torch.empty(rows, dtype=torch.float32, device="cuda")
    state = torch.zeros(L.STATE_WORDS, dtype=torch.int32, device="cuda")
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for step in (1, 2):
        ref.step(x, seed=5, block=1, step=step)
        rc = lib.dg_sampler_step_static(_p(x), code, rows, vocab, C.c_uint64(5), 1, step,
                                        0.9, 0.005, 48, 0, _p(canvas), _p(argmax), _p(entropy),
                                        _p(conf), _p(state), stream)
        assert rc == 0, lib.dg_last_error()
        torch.cuda.synchronize()
        assert torch.equal(argmax, ref.argmax) and torch.equal(canvas, ref.canvas)
        assert torch.max(torch.abs(entropy - ref.entropy)).item() <= 1e-5
        assert torch.max(torch.abs(conf - ref.conf) / ref.conf).item() <= 1e-5
        assert torch.equal(state, ref.state)
        if kind == "mixed":  # re-noised rows take a Philox draw, not their argmax
            assert torch.any(canvas[1::2] != argmax[1::2])
            assert torch.equal(canvas[0::2], argmax[0::2])
    st = state.cpu().tolist()
    if kind == "confident":
        assert st[L.STATE_DONE] == 1 and st[L.STATE_STOP_STEP] == 2
    else:
        assert st[L.STATE_DONE] == 0 and st[L.STATE_STEPS_RUN] == 2


def test_static_sampler_rejects_oversize():
    from block_text_diffusion_dg_b200 import _lib as L
    lib = L.lib()
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    rc = lib.dg_sampler_step_static(_p(dummy), L.DTYPE_BF16, 257, 262144, C.c_uint64(0), 0, 1, 0.9,
                                    0.005, 48, 0, _p(dummy), _p(dummy), _p(dummy), _p(dummy),
                                    _p(dummy), None)
    assert rc == -2 and b"at most 256 rows" in lib.dg_last_error()
    rc = lib.dg_sampler_step_static(_p(dummy), L.DTYPE_BF16, 4, 262144 * 2, C.c_uint64(0), 0, 1,
                                    0.9, 0.005, 48, 0, _p(dummy), _p(dummy), _p(dummy), _p(dummy),
                                    _p(dummy), None)
    assert rc == -2
