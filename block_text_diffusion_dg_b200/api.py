"""Python binding of libdg: the same entry points as include/dg.h, taking torch CUDA tensors.

PyTorch provides device memory and streams only; every step of the denoise path runs in
libdg's kernels.  Each wrapper checks the library's status and raises on failure.
"""
import ctypes as C

import torch

from . import _lib as L
from ._lib import check, lib


def _ptr(t):
    return C.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _need_cuda(t, name, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def make_config(shape, *, kv_capacity, fixed_steps=16, max_steps=48, tau=0.9, h_bound=0.005,
                eps=1e-6, rope_theta=10000.0, prefill_chunk=0, experts="bf16",
                lock_rule="confidence", entropy_lock=0.1, sticky=False, temperature=1.0,
                commit="reencode", batch=1, head="bf16"):
    """Config of a model shape; experts="e4m3" selects the FP8 expert format (bf16 model);
    lock_rule="entropy_bound" locks positions with entropy <= entropy_lock (nats) instead of
    confidence >= tau; sticky=True keeps a locked position's token for the rest of the block;
    temperature sets T of the sampler's softmax(logits / T); commit="reuse_kv" commits a block
    by keeping the canvas K/V of its last denoise step instead of re-encoding it causally;
    batch=B decodes B sequences in lockstep (sequence b's Philox key is seed + b); head="e4m3"
    runs the LM head on e4m3 operands (weights from quantize_head)."""
    if head not in ("bf16", "e4m3"):
        raise ValueError("head must be 'bf16' or 'e4m3'")
    if commit not in ("reencode", "reuse_kv"):
        raise ValueError("commit must be 'reencode' or 'reuse_kv'")
    s = shape
    if experts not in ("bf16", "e4m3", "nvfp4"):
        raise ValueError("experts must be 'bf16', 'e4m3' or 'nvfp4'")
    rules = {"confidence": 0, "entropy_bound": 1}
    if lock_rule not in rules:
        raise ValueError("lock_rule must be 'confidence' or 'entropy_bound'")
    if s["storage"] == "fp32":
        if experts != "bf16":
            raise ValueError("the all-fp32 model has no e4m3 expert format")
        dtype = L.DTYPE_FP32
    else:
        dtype = {"bf16": L.DTYPE_BF16, "e4m3": L.DTYPE_BF16_E4M3,
                 "nvfp4": L.DTYPE_BF16_NVFP4}[experts]
    return L.Config(
        n_layers=s["n_layers"], d_model=s["d_model"], n_heads=s["n_heads"],
        n_kv_heads=s["n_kv_heads"], head_dim=s["head_dim"], n_experts=s["n_experts"],
        top_k=s["top_k"], expert_hidden=s["expert_hidden"], shared_hidden=s["shared_hidden"],
        vocab=s["vocab"], canvas=s["canvas"], kv_capacity=kv_capacity,
        dtype=dtype, eps=eps,
        rope_theta=rope_theta, tau=tau, h_bound=h_bound, max_steps=max_steps,
        fixed_steps=fixed_steps, prefill_chunk=prefill_chunk, lock_rule=rules[lock_rule],
        entropy_lock=entropy_lock, sticky_locks=int(bool(sticky)), temperature=temperature,
        commit_reuse_kv=int(commit == "reuse_kv"), batch=int(batch),
        lm_head_e4m3=int(head == "e4m3"))


def workspace_bytes(cfg):
    kv, scratch = C.c_size_t(), C.c_size_t()
    check(lib().dg_workspace_bytes(C.byref(cfg), C.byref(kv), C.byref(scratch)),
          "dg_workspace_bytes")
    return kv.value, scratch.value


class DiffusionModel:
    """A bound model context (dg_ctx): weights, KV cache and scratch owned by torch tensors."""

    def __init__(self, cfg, weights, device="cuda", stream=None):
        self.cfg = cfg
        self.batch = max(1, cfg.batch)
        self.n_tok = self.batch * cfg.canvas  # canvas positions of all sequences
        self.weights = weights  # keep the tensors alive
        self.device = torch.device(device)
        kv_b, sc_b = workspace_bytes(cfg)
        self.kv = torch.empty(kv_b, dtype=torch.uint8, device=self.device)
        self.scratch = torch.empty(sc_b, dtype=torch.uint8, device=self.device)
        layers = (L.LayerWeights * cfg.n_layers)()
        for i, lw in enumerate(weights["layers"]):
            for name in ("attn_norm", "wqkv", "wo", "ffn_norm", "wr", "w_gu", "w_d", "ws_gu", "ws_d",
                         "w_gu_scale", "w_d_scale", "ws_gu_scale", "ws_d_scale",
                         "w_gu_sf", "w_d_sf", "ws_gu_sf", "ws_d_sf"):
                t = lw.get(name)
                _need_cuda(t, name)
                setattr(layers[i], name, None if t is None else t.data_ptr())
        _need_cuda(weights["embed"], "embed")
        _need_cuda(weights["final_norm"], "final_norm")
        self._layers = layers
        hc, hs = weights.get("head_codes"), weights.get("head_scale")
        _need_cuda(hc, "head_codes")
        _need_cuda(hs, "head_scale")
        w = L.Weights(embed=weights["embed"].data_ptr(), final_norm=weights["final_norm"].data_ptr(),
                      layers=layers, head_codes=None if hc is None else hc.data_ptr(),
                      head_scale=None if hs is None else hs.data_ptr())
        h = C.c_void_p()
        check(lib().dg_create(C.byref(cfg), C.byref(w), _ptr(self.kv), _ptr(self.scratch),
                              _stream(stream), C.byref(h)), "dg_create")
        self.handle = h
        bufs = [C.c_void_p() for _ in range(5)]
        check(lib().dg_get_buffers(h, *[C.byref(b) for b in bufs]), "dg_get_buffers")
        self._bufs = [b.value for b in bufs]
        self.out_ids = torch.empty(self.n_tok, dtype=torch.int32, device=self.device)
        self.out_state = torch.empty(self.batch, L.STATE_WORDS, dtype=torch.int32,
                                     device=self.device).squeeze(0)

    def close(self):
        if getattr(self, "handle", None):
            lib().dg_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # --- the five entry points of the decode loop ---
    def kv_append(self, ids, stream=None):
        """ids [n] (one sequence) or [batch, n] (row b: sequence b's next n tokens)."""
        _need_cuda(ids, "ids", torch.int32)
        if ids.numel() % self.batch:
            raise ValueError("ids must hold the same number of tokens for every sequence")
        check(lib().dg_kv_append(self.handle, _ptr(ids), ids.numel() // self.batch,
                                 _stream(stream)), "dg_kv_append")

    def canvas_init(self, seed, block, stream=None):
        check(lib().dg_canvas_init(self.handle, C.c_uint64(seed), block, _stream(stream)),
              "dg_canvas_init")

    def reset_block(self, stream=None):
        check(lib().dg_reset_block(self.handle, _stream(stream)), "dg_reset_block")

    def denoise_step(self, step, stream=None):
        check(lib().dg_denoise_step(self.handle, step, _stream(stream)), "dg_denoise_step")

    def sample_update(self, step, stream=None):
        check(lib().dg_sample_update(self.handle, step, _stream(stream)), "dg_sample_update")

    def commit_block(self, out_ids=None, out_state=None, stream=None):
        out_ids = self.out_ids if out_ids is None else out_ids
        out_state = self.out_state if out_state is None else out_state
        check(lib().dg_commit_block(self.handle, _ptr(out_ids), _ptr(out_state), _stream(stream)),
              "dg_commit_block")
        return out_ids, out_state

    # --- inspection ---
    @property
    def kv_length(self):
        return lib().dg_kv_length(self.handle)

    def kv_truncate(self, n):
        check(lib().dg_kv_truncate(self.handle, n), "dg_kv_truncate")

    def _view(self, ptr, n, dtype):
        # a non-owning view of a scratch buffer (offset into self.scratch)
        off = ptr - self.scratch.data_ptr()
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return self.scratch[off:off + nbytes].view(dtype)

    def buffers(self):
        """Views of the canvas, argmax, entropy and confidence ([batch * canvas], sequence-major)
        and of the state words ([STATE_WORDS], or [batch, STATE_WORDS] when batched)."""
        t = self.n_tok
        st = self._view(self._bufs[4], self.batch * L.STATE_WORDS, torch.int32)
        return dict(canvas=self._view(self._bufs[0], t, torch.int32),
                    argmax=self._view(self._bufs[1], t, torch.int32),
                    entropy=self._view(self._bufs[2], t, torch.float32),
                    conf=self._view(self._bufs[3], t, torch.float32),
                    state=st if self.batch == 1 else st.view(self.batch, L.STATE_WORDS))

    def check_device_status(self, stream=None):
        check(lib().dg_check_device_status(self.handle, _stream(stream)), "dg_check_device_status")

    def debug_logits(self, stream=None):
        out = torch.empty(self.n_tok, self.cfg.vocab, dtype=torch.float32, device=self.device)
        check(lib().dg_debug_logits(self.handle, _ptr(out), _stream(stream)), "dg_debug_logits")
        return out

    def debug_hidden(self):
        p = C.c_void_p()
        check(lib().dg_debug_hidden(self.handle, C.byref(p)), "dg_debug_hidden")
        return self._view(p.value, self.n_tok * self.cfg.d_model, torch.float32).view(
            self.n_tok, self.cfg.d_model)

    def debug_routing(self, n=None):
        """(ids [n, k], weights [n, k], router logits [n, E]) of the last layer run."""
        n = self.n_tok if n is None else n
        ps = [C.c_void_p() for _ in range(3)]
        check(lib().dg_debug_routing(self.handle, *[C.byref(x) for x in ps]), "dg_debug_routing")
        k, e = self.cfg.top_k, self.cfg.n_experts
        return (self._view(ps[0].value, n * k, torch.int32).view(n, k),
                self._view(ps[1].value, n * k, torch.float32).view(n, k),
                self._view(ps[2].value, n * e, torch.float32).view(n, e))

    def debug_tensors(self, n=None):
        """(q, o, xn) views of the most recent layer's intermediates."""
        n = self.cfg.canvas if n is None else n
        c = self.cfg
        dt = torch.float32 if c.dtype == L.DTYPE_FP32 else torch.bfloat16
        tq = c.canvas if c.dtype == L.DTYPE_FP32 else 256
        ps = [C.c_void_p() for _ in range(3)]
        check(lib().dg_debug_tensors(self.handle, *[C.byref(x) for x in ps]), "dg_debug_tensors")
        q = self._view(ps[0].value, c.n_heads * tq * c.head_dim, dt).view(c.n_heads, tq, c.head_dim)
        o = self._view(ps[1].value, n * c.n_heads * c.head_dim, dt).view(n, c.n_heads * c.head_dim)
        xn = self._view(ps[2].value, n * c.d_model, dt).view(n, c.d_model)
        return q, o, xn

    def debug_layer_part(self, layer, part, x_in, causal, stream=None):
        """Half a layer: part 0 attention sub-block, part 1 MoE sub-block (x_out = x_in + ...)."""
        _need_cuda(x_in, "x_in", torch.float32)
        out = torch.empty_like(x_in)
        check(lib().dg_debug_layer_part(self.handle, layer, part, _ptr(x_in), _ptr(out),
                                        x_in.shape[0], int(bool(causal)), _stream(stream)),
              "dg_debug_layer_part")
        return out

    def debug_layer(self, layer, x_in, causal, stream=None):
        _need_cuda(x_in, "x_in", torch.float32)
        out = torch.empty_like(x_in)
        check(lib().dg_debug_layer(self.handle, layer, _ptr(x_in), _ptr(out), x_in.shape[0],
                                   int(bool(causal)), _stream(stream)), "dg_debug_layer")
        return out


def generate(model, prompt_ids, n_blocks, seed, stream=None):
    """Block-autoregressive decode through the C ABI.

    One sequence: returns (ids [n_blocks * T], states [n_blocks, STATE_WORDS]).  A batched model
    takes prompt_ids [batch, n] and returns (ids [batch, n_blocks * T], states [n_blocks, batch,
    STATE_WORDS]); sequence b's canvases draw from the Philox key seed + b."""
    cfg = model.cfg
    if prompt_ids is not None and prompt_ids.numel():
        model.kv_append(prompt_ids, stream)
    steps = cfg.fixed_steps if cfg.fixed_steps > 0 else cfg.max_steps
    nb, t = model.batch, cfg.canvas
    out = torch.empty(n_blocks, nb * t, dtype=torch.int32, device=model.device)
    states = torch.empty(n_blocks, nb, L.STATE_WORDS, dtype=torch.int32, device=model.device)
    for b in range(n_blocks):
        model.canvas_init(seed, b, stream)
        for s in range(1, steps + 1):
            model.denoise_step(s, stream)
            model.sample_update(s, stream)
        model.commit_block(out[b], states[b], stream)
    if nb == 1:
        return out.view(n_blocks * t), states.view(n_blocks, L.STATE_WORDS)
    return (out.view(n_blocks, nb, t).transpose(0, 1).reshape(nb, n_blocks * t), states)


# ---------------------------------------------------------------------------------------
# standalone operators
class Sampler:
    """The canvas sampler over caller-provided logits [rows, V] (bf16 or fp32)."""

    def __init__(self, rows, vocab, device="cuda"):
        self.rows, self.vocab = rows, vocab
        n = C.c_size_t()
        check(lib().dg_sampler_workspace_bytes(rows, vocab, C.byref(n)), "dg_sampler_workspace_bytes")
        self.ws = torch.empty(n.value, dtype=torch.uint8, device=device)
        self.state = torch.zeros(L.STATE_WORDS, dtype=torch.int32, device=device)
        self.canvas = torch.empty(rows, dtype=torch.int32, device=device)
        self.argmax = torch.empty(rows, dtype=torch.int32, device=device)
        self.entropy = torch.empty(rows, dtype=torch.float32, device=device)
        self.conf = torch.empty(rows, dtype=torch.float32, device=device)

    def reset(self, stream=None):
        check(lib().dg_sampler_reset(self.rows, self.vocab, _ptr(self.ws), _ptr(self.state),
                                     _stream(stream)), "dg_sampler_reset")

    def step(self, logits, seed, block, step, tau=0.9, h_bound=0.005, max_steps=48,
             fixed_steps=0, stream=None):
        _need_cuda(logits, "logits")
        if tuple(logits.shape) != (self.rows, self.vocab):
            raise ValueError("logits shape mismatch")
        dt = {torch.bfloat16: L.DTYPE_BF16, torch.float32: L.DTYPE_FP32}[logits.dtype]
        check(lib().dg_sampler_step(_ptr(logits), dt, self.rows, self.vocab, C.c_uint64(seed),
                                    block, step, tau, h_bound, max_steps, fixed_steps, _ptr(self.ws),
                                    _ptr(self.canvas), _ptr(self.argmax), _ptr(self.entropy),
                                    _ptr(self.conf), _ptr(self.state), _stream(stream)),
              "dg_sampler_step")


def canvas_attention(q, k, vt, n_keys, causal_prefix=-1, scale=None, n_queries=None, out=None,
                     workspace=None, stream=None):
    """q [Hq, Tq, 128] bf16, k [Hkv, ldk, 128] bf16, vt [Hkv, 128, ldk] bf16 -> o [T, Hq*128]."""
    for t, n in ((q, "q"), (k, "k"), (vt, "vt")):
        _need_cuda(t, n, torch.bfloat16)
    hq, tq, hd = q.shape
    hkv, ldk, _ = k.shape
    t = tq if n_queries is None else n_queries
    scale = hd ** -0.5 if scale is None else scale
    if out is None:
        out = torch.empty(t, hq * hd, dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        n = C.c_size_t()
        check(lib().dg_attention_workspace_bytes(hq, hkv, tq, n_keys, C.byref(n)),
              "dg_attention_workspace_bytes")
        workspace = torch.empty(n.value, dtype=torch.uint8, device=q.device)
    check(lib().dg_canvas_attention(_ptr(q), _ptr(k), _ptr(vt), _ptr(out), hq, hkv, t, tq, n_keys,
                                    ldk, causal_prefix, scale, _ptr(workspace), workspace.numel(),
                                    _stream(stream)), "dg_canvas_attention")
    return out


def moe_workspace(t, d, e, k, h, hs, device="cuda"):
    n = C.c_size_t()
    check(lib().dg_moe_workspace_bytes(t, d, e, k, h, hs, C.byref(n)), "dg_moe_workspace_bytes")
    return torch.empty(n.value, dtype=torch.uint8, device=device)


def moe_ffn(x, wr, w_gu, w_d, top_k, ws_gu=None, ws_d=None, residual=None, workspace=None,
            out=None, ids=None, weights=None, router_logits=None, stream=None):
    """Top-k MoE over x [T, d] bf16 -> y [T, d] fp32 (= residual + MoE(x))."""
    for t, n in ((x, "x"), (wr, "wr"), (w_gu, "w_gu"), (w_d, "w_d"), (ws_gu, "ws_gu"), (ws_d, "ws_d")):
        _need_cuda(t, n, torch.bfloat16)
    t, d = x.shape
    e, two_h, _ = w_gu.shape
    h = two_h // 2
    hs = 0 if ws_gu is None else ws_gu.shape[0] // 2
    if workspace is None:
        workspace = moe_workspace(t, d, e, top_k, h, hs, x.device)
    if out is None:
        out = torch.empty(t, d, dtype=torch.float32, device=x.device)
    check(lib().dg_moe_ffn(_ptr(x), _ptr(residual), _ptr(wr), _ptr(w_gu), _ptr(w_d), _ptr(ws_gu),
                           _ptr(ws_d), _ptr(out), _ptr(ids), _ptr(weights), _ptr(router_logits), t,
                           d, e, top_k, h, hs, _ptr(workspace), workspace.numel(), _stream(stream)),
          "dg_moe_ffn")
    return out


def e4m3_pitch(cols):
    """Row pitch (bytes) of an e4m3 matrix with `cols` codes per row (DG_E4M3_PITCH)."""
    return (cols + 127) // 128 * 128


def quantize_e4m3(x, pitch=None, stream=None):
    """Row-wise e4m3 quantisation of a bf16 tensor [..., cols] (cols % 16 == 0).

    Returns (codes uint8 [..., pitch], scales fp32 [...]): scale = max|row| / 448 and
    code = rn_satfinite(x / scale), the FP8 expert format of dg_quantize_e4m3; codes past `cols`
    are zero.  The default pitch is the expert-weight pitch e4m3_pitch(cols).
    """
    _need_cuda(x, "x", torch.bfloat16)
    cols = x.shape[-1]
    pitch = e4m3_pitch(cols) if pitch is None else pitch
    rows = x.numel() // max(cols, 1)
    codes = torch.empty(x.shape[:-1] + (pitch,), dtype=torch.uint8, device=x.device)
    scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    check(lib().dg_quantize_e4m3(_ptr(x), rows, cols, cols, _ptr(codes), pitch, _ptr(scales),
                                 _stream(stream)), "dg_quantize_e4m3")
    return codes, scales


def quantize_nvfp4(x, stream=None):
    """NVFP4 quantisation of a bf16 tensor [..., cols] (cols % 64 == 0), rows flattened.

    Returns (codes uint8 [..., e4m3_pitch(cols / 2)] with two e2m1 codes per byte, block-scale
    atoms uint8 [ceil(rows / 128), 4 * ceil(cols / 256), 512], row scales fp32 [...]) as
    dg_quantize_nvfp4 lays them out.
    """
    _need_cuda(x, "x", torch.bfloat16)
    cols = x.shape[-1]
    rows = x.numel() // max(cols, 1)
    pitch = e4m3_pitch(cols // 2)
    codes = torch.empty(x.shape[:-1] + (pitch,), dtype=torch.uint8, device=x.device)
    sf = torch.empty(((rows + 127) // 128, 4 * ((cols + 255) // 256), 512), dtype=torch.uint8,
                     device=x.device)
    scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    check(lib().dg_quantize_nvfp4(_ptr(x), rows, cols, cols, _ptr(codes), pitch, _ptr(sf),
                                  _ptr(scales), _stream(stream)), "dg_quantize_nvfp4")
    return codes, sf, scales


def quantize_head(weights, stream=None):
    """A copy of a weight dict with the e4m3 head added: head_codes (codes of the embedding table
    at e4m3_pitch) and head_scale (one fp32 scale per vocabulary row).  The bf16 embedding stays
    for the canvas embedding gather."""
    out = dict(weights)
    out["head_codes"], out["head_scale"] = quantize_e4m3(weights["embed"], stream=stream)
    return out


def quantize_experts(weights, fmt="e4m3", stream=None):
    """A copy of a bf16 weight dict with every layer's expert matrices (routed and shared) in the
    e4m3 format (w_gu, w_d, ws_gu, ws_d become codes at e4m3_pitch, *_scale their row scales) or
    the NVFP4 format (codes, *_scale row scales and *_sf block-scale atoms)."""
    if fmt not in ("e4m3", "nvfp4"):
        raise ValueError("fmt must be 'e4m3' or 'nvfp4'")
    out = dict(weights)
    out["layers"] = []
    for lw in weights["layers"]:
        q = dict(lw)
        for name in ("w_gu", "w_d", "ws_gu", "ws_d"):
            if lw.get(name) is None:
                continue
            if fmt == "e4m3":
                q[name], q[name + "_scale"] = quantize_e4m3(lw[name], stream)
            else:
                q[name], q[name + "_sf"], q[name + "_scale"] = quantize_nvfp4(lw[name], stream)
        out["layers"].append(q)
    return out


def moe_ffn_e4m3(x, wr, w_gu, w_gu_scale, w_d, w_d_scale, top_k, ws_gu=None, ws_gu_scale=None,
                 ws_d=None, ws_d_scale=None, residual=None, workspace=None, out=None, ids=None,
                 weights=None, router_logits=None, stream=None):
    """moe_ffn with e4m3 experts (codes uint8 with rows at e4m3_pitch + fp32 row scales, as
    quantize_e4m3 returns them)."""
    for t, n in ((x, "x"), (wr, "wr")):
        _need_cuda(t, n, torch.bfloat16)
    for t, n in ((w_gu, "w_gu"), (w_d, "w_d"), (ws_gu, "ws_gu"), (ws_d, "ws_d")):
        _need_cuda(t, n, torch.uint8)
    for t, n in ((w_gu_scale, "w_gu_scale"), (w_d_scale, "w_d_scale"),
                 (ws_gu_scale, "ws_gu_scale"), (ws_d_scale, "ws_d_scale")):
        _need_cuda(t, n, torch.float32)
    t, d = x.shape
    e, two_h, _ = w_gu.shape
    h = two_h // 2
    hs = 0 if ws_gu is None else ws_gu.shape[0] // 2
    for wt, n, rows, cols in ((w_gu, "w_gu", e * 2 * h, d), (w_d, "w_d", e * d, h),
                              (ws_gu, "ws_gu", 2 * hs, d), (ws_d, "ws_d", d, hs)):
        if wt is not None and (wt.shape[-1] != e4m3_pitch(cols) or wt.numel() != rows * e4m3_pitch(cols)):
            raise ValueError(f"{n} must be [.., {rows} rows, e4m3_pitch({cols})] codes")
    if workspace is None:
        workspace = moe_workspace(t, d, e, top_k, h, hs, x.device)
    if out is None:
        out = torch.empty(t, d, dtype=torch.float32, device=x.device)
    check(lib().dg_moe_ffn_e4m3(_ptr(x), _ptr(residual), _ptr(wr), _ptr(w_gu), _ptr(w_gu_scale),
                                _ptr(w_d), _ptr(w_d_scale), _ptr(ws_gu), _ptr(ws_gu_scale),
                                _ptr(ws_d), _ptr(ws_d_scale), _ptr(out), _ptr(ids), _ptr(weights),
                                _ptr(router_logits), t, d, e, top_k, h, hs, _ptr(workspace),
                                workspace.numel(), _stream(stream)), "dg_moe_ffn_e4m3")
    return out


def moe_ffn_nvfp4(x, wr, w_gu, w_d, top_k, ws_gu=None, ws_d=None, residual=None, workspace=None,
                  out=None, ids=None, weights=None, router_logits=None, stream=None):
    """moe_ffn with NVFP4 experts: each of w_gu, w_d, ws_gu, ws_d is the (codes, atoms, row
    scales) triple quantize_nvfp4 returns for the stacked matrix."""
    _need_cuda(x, "x", torch.bfloat16)
    _need_cuda(wr, "wr", torch.bfloat16)
    t, d = x.shape
    e = wr.shape[0]
    h = w_gu[0].shape[-2] // 2
    hs = 0 if ws_gu is None else ws_gu[0].shape[-2] // 2
    trip = [w_gu, w_d, ws_gu, ws_d]
    ptrs = []
    for tr in trip:
        if tr is None:
            ptrs += [None, None, None]
        else:
            codes, sf, scales = tr
            ptrs += [codes, scales, sf]
    if workspace is None:
        workspace = moe_workspace(t, d, e, top_k, h, hs, x.device)
    if out is None:
        out = torch.empty(t, d, dtype=torch.float32, device=x.device)
    check(lib().dg_moe_ffn_nvfp4(_ptr(x), _ptr(residual), _ptr(wr), *[_ptr(p) for p in ptrs],
                                 _ptr(out), _ptr(ids), _ptr(weights), _ptr(router_logits), t, d, e,
                                 top_k, h, hs, _ptr(workspace), workspace.numel(), _stream(stream)),
          "dg_moe_ffn_nvfp4")
    return out
