"""dg_sampler_step_static: the canvas sampler for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: for example code inside a host framework whose memory pool
owns the whole device budget, or a latency-critical path that may not risk cudaMalloc's implicit
device synchronisation.  This entry point keeps the sampler's temporaries and its step-to-step
stop-test state in a fixed device array inside the library instead of a caller workspace.  The
test calls it through the C ABI and compares it with dg_sampler_step (the workspace version) on
two consecutive steps of one sequence; the second step stops, which needs the state the first
call left in the array.  It passes alone in a fresh process and after the other tests.
"""
import ctypes as C

import pytest
import torch

from dg_synth import planted_normal

pytestmark = pytest.mark.gpu


def _p(t):
    return C.c_void_p(t.data_ptr())


def test_static_sampler_matches_workspace_sampler():
    from block_text_diffusion_dg_b200 import Sampler
    from block_text_diffusion_dg_b200 import _lib as L
    lib = L.lib()
    rows, vocab = 256, 262144
    z, _ = planted_normal(rows, vocab, seed=21)
    # a unique, far-ahead maximum in every row: near-zero entropy, so step 2 meets the stop rule
    x = (z * 50.0).to(torch.bfloat16).cuda()
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
        rc = lib.dg_sampler_step_static(_p(x), L.DTYPE_BF16, rows, vocab, C.c_uint64(5), 1, step,
                                        0.9, 0.005, 48, 0, _p(canvas), _p(argmax), _p(entropy),
                                        _p(conf), _p(state), stream)
        assert rc == 0, lib.dg_last_error()
        torch.cuda.synchronize()
        assert torch.equal(argmax, ref.argmax) and torch.equal(canvas, ref.canvas)
        assert torch.max(torch.abs(entropy - ref.entropy)).item() <= 1e-5
        assert torch.max(torch.abs(conf - ref.conf) / ref.conf).item() <= 1e-5
        assert torch.equal(state, ref.state)
    st = state.cpu().tolist()
    assert st[L.STATE_DONE] == 1 and st[L.STATE_STOP_STEP] == 2


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
