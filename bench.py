#!/usr/bin/env python
"""Committed canvas tokens/s of block text diffusion on B200 (one JSON line on rank 0).

Workload (the full block decode): a random-init 30-layer MoE decoder shaped like Gemma 4
26B-A4B (d 2816, 16 q / 8 kv heads x 128, 128 experts top-8 SiLU-GLU 704 + shared 2112,
tied vocab 262144, bf16), a 4,096-token uniform prompt prefilled into the KV cache once, then
4 canvases of 256 tokens, 16 fixed denoise steps each (1,024 committed tokens).  One bench
step is that whole 4-block decode (KV cache cut back to the prompt before each step).

  value  : committed tokens / s over K timed steps, device time (CUDA events), max over ranks
  e2e    : the same through the public API from pinned host buffers: prompt H2D, prefill,
           4 blocks, committed ids + states D2H, all inside the timed region
  roofline: the dominant kernel's launches timed with CUDA events on its own stream (a
           profiled pass after the timed region) against the measured HBM copy bandwidth
  cpu_baseline: the CPU oracle on one denoise layer + 1/16 of the LM head + the sampler,
           extrapolated to the decode (rank 0, N = 1)

--experts e4m3 runs the same decode with the FP8 expert format (routed and shared expert weights
e4m3 with per-row scales, expert activations quantised per row; everything else bf16).

Multi-GPU: every rank decodes its own sequence with its own weights ("replicas only": the
one-canvas, batch-1 decode has no data-path exchange); value sums all ranks.
"""
import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PROMPT, BLOCKS, FIXED_STEPS, CANVAS, MAX_STEPS = 4096, 4, 16, 256, 48
LONG_PROMPT = 32768  # the long-context measurement
BATCH = 4  # sequences of the small-batch measurement
PREFILL_CHUNK = 4096  # prompt tokens per causal-encode pass (the whole prompt)
WORKLOAD = ("full block decode: 30-layer MoE decoder (d 2816, 16/8 heads x 128, 128 experts "
            "top-8 x 704 + shared 2112, vocab 262144, bf16, random init), 4096-token prompt "
            "prefilled in one pass, 4 canvases x 256 tokens x 16 fixed denoise steps")
WORKLOAD_E4M3 = WORKLOAD.replace("bf16, random init", "bf16 with e4m3 experts, random init")
WORKLOAD_NVFP4 = WORKLOAD.replace("bf16, random init", "bf16 with NVFP4 experts, random init")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--roofline-kernel", default="expert_gate_up")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--head", choices=["bf16", "e4m3"], default="bf16",
                    help="LM head format (e4m3: the head on e4m3 operands)")
    ap.add_argument("--experts", choices=["bf16", "e4m3", "nvfp4"], default="bf16",
                    help="expert weight format of the decode model")
    ap.add_argument("--profile", choices=["decode_step", "decode_step_small", "decode_step_e4m3",
                                          "moe", "moe_e4m3", "moe_nvfp4", "attention", "sampler"],
                    help="run one profiled region between cudaProfilerStart/Stop and exit "
                         "(for ncu --profile-from-start off); prints no JSON")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------------------
class Clocks:
    """nvidia-smi sampling (200 ms) of this process's GPU during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        if not self.uuid.startswith("GPU-"):
            self.uuid = "GPU-" + self.uuid
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        self.p.wait()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------------------
def cpu_oracle_sample(seed=0):
    """Time the CPU oracle on a bounded sample of the decode and extrapolate to tokens/s.

    Sample: one bidirectional denoise layer over the 256-token canvas against a 4,096-token
    history, the LM head over 1/16 of the vocabulary, and the sampler statistics over the full
    vocabulary.  Extrapolation: a denoise step = 30 layers + 16 x LM-head slice + sampler; a
    block = 16 steps + a causal commit (30 layers); 4 blocks = 1,024 tokens.
    """
    import numpy as np
    from dg_synth import SHAPES
    from oracle import model as om
    from oracle import sampler as osmp
    s = SHAPES["a4b"]
    g = torch.Generator().manual_seed(seed)
    d, hd, e, h, hs, v = (s["d_model"], s["head_dim"], s["n_experts"], s["expert_hidden"],
                          s["shared_hidden"], s["vocab"])

    def n(*shape, std=0.02):
        return (torch.empty(shape).normal_(0, std, generator=g)).to(torch.bfloat16).float().numpy()

    lw = dict(attn_norm=np.ones(d, np.float32), ffn_norm=np.ones(d, np.float32),
              wqkv=n((s["n_heads"] + 2 * s["n_kv_heads"]) * hd, d), wo=n(d, s["n_heads"] * hd),
              wr=n(e, d), w_gu=n(e, 2 * h, d), w_d=n(e, d, h), ws_gu=n(2 * hs, d), ws_d=n(d, hs))
    cfg = om.ModelConfig(**{k: s[k] for k in ("n_layers", "d_model", "n_heads", "n_kv_heads",
                                              "head_dim", "n_experts", "top_k", "expert_hidden",
                                              "shared_hidden", "vocab", "canvas", "storage")})
    x = n(CANVAS, d, std=1.0).astype(np.float64)
    ck = n(s["n_kv_heads"], PROMPT, hd, std=1.0)
    cv = n(s["n_kv_heads"], PROMPT, hd, std=1.0)
    pos = PROMPT + np.arange(CANVAS)
    t0 = time.perf_counter()
    om.layer_forward(cfg, lw, x, pos, ck, cv, causal=False)
    t_layer = time.perf_counter() - t0
    emb = n(v // 16, d)
    t0 = time.perf_counter()
    logits = om.lm_head(cfg, dict(embed=emb, final_norm=np.ones(d)), x)
    t_head = (time.perf_counter() - t0) * 16
    full = np.tile(logits, (1, 16))
    t0 = time.perf_counter()
    osmp.row_stats(full)
    t_samp = time.perf_counter() - t0
    t_step = s["n_layers"] * t_layer + t_head + t_samp
    t_decode = BLOCKS * (FIXED_STEPS * t_step + s["n_layers"] * t_layer)
    sample_s = t_layer + t_head / 16 + t_samp
    return dict(value=BLOCKS * CANVAS / t_decode, unit="tok/s", cores=len(os.sched_getaffinity(0)),
                kind="oracle",
                sample=(f"1 denoise layer ({t_layer:.2f} s) + LM head on V/16 ({t_head / 16:.2f} s) "
                        f"+ sampler over V ({t_samp:.2f} s), extrapolated to 4 blocks x 16 steps "
                        f"x 30 layers; sample wall {sample_s:.1f} s"),
                sample_seconds=sample_s)


# ---------------------------------------------------------------------------------------
def run_reference(args, rank):
    if rank != 0:
        return
    steps = []
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(seed=i)
        if i >= args.warmup:
            steps.append(r)
    val = statistics.median(r["value"] for r in steps)
    cb = dict(value=val, unit="tok/s", cores=steps[0]["cores"], kind="oracle",
              sample=steps[0]["sample"])
    out = dict(impl="reference", metric="committed canvas tokens/s", value=val, unit="tok/s",
               n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
               ms_per_step=1e3 * BLOCKS * CANVAS / val, higher_is_better=True, scaling="weak",
               vs_baseline=None, dtype="f64", data="synthetic",
               config=dict(workload=WORKLOAD, global_batch=1, seq_len=PROMPT + BLOCKS * CANVAS,
                           parallelism="replicas"),
               cpu_baseline=cb,
               e2e=dict(value=val, unit="tok/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(out), flush=True)


def max_over_ranks(x, world, device=None):
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    on_gpu = dist.get_backend() == "nccl"
    t = torch.tensor([float(x)], dtype=torch.float64, device=device if on_gpu else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank, world, ms_max):
    """Whole-job tokens/s: every rank decodes its own sequence; time is the slowest rank's."""
    return world * tokens_per_rank / (ms_max / 1e3)


def _time_op(fn, stream, reps=10, flush=None):
    """Average device time (ms) of fn() over reps, CUDA events on `stream`, L2 flushed between reps."""
    for _ in range(3):
        fn()
    total = 0.0
    for _ in range(reps):
        if flush is not None:
            # read (not write) the flush buffer: L2 ends up holding clean lines only
            torch.sum(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        total += e0.elapsed_time(e1)
    return total / reps


def run_ops(dev, stream, hbm, tf_burst):
    """The standalone operators at their full sizes, each against its roofline (kernel timed
    alone: burst peaks).  sampler: bf16 logits [256, 262144]; attention: 16 q / 8 kv heads x 128,
    4096 + 256 keys; MoE: 256 tokens, d 2816, 128 experts top-8 x 704 + shared 2112."""
    import block_text_diffusion_dg_b200 as dg
    from dg_synth import attention_inputs, moe_inputs, sampler_logits
    # 1 GB flush (> L2): it also keeps the GPU busy while the host enqueues the timed call, so
    # the event interval holds device time only
    flush = torch.ones(256 * 1024 * 1024, dtype=torch.float32, device=dev)
    out = {}
    x = sampler_logits(256, 262144, seed=0).to(dev)
    s = dg.Sampler(256, 262144, device=dev)
    s.reset()
    ms = _time_op(lambda: s.step(x, seed=0, block=0, step=1, stream=stream), stream, flush=flush)
    gbs = 256 * 262144 * 2 / (ms / 1e3) / 1e9
    out["sampler"] = dict(us=round(ms * 1e3, 2), bound="hbm", achieved_gbs=round(gbs, 1),
                          frac=round(gbs / hbm, 4), bytes=256 * 262144 * 2)
    del x, s
    q, k, v = (t.to(dev) for t in attention_inputs(seed=0))
    vt = v.transpose(1, 2).contiguous()
    ws = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
    o = torch.empty(256, 16 * 128, dtype=torch.bfloat16, device=dev)
    ms = _time_op(lambda: dg.canvas_attention(q, k, vt, 4096 + 256, out=o, workspace=ws,
                                              stream=stream), stream, flush=flush)
    flops = 4 * 16 * 256 * 4352 * 128
    tf = flops / (ms / 1e3) / 1e12
    out["attention"] = dict(us=round(ms * 1e3, 2), bound="tensor", achieved_tflops=round(tf, 1),
                            frac=round(tf / tf_burst, 4), flops=flops)
    del q, k, v, vt, ws, o
    m = {kk: (None if vv is None else vv.to(dev)) for kk, vv in moe_inputs(seed=0).items()}
    wsm = dg.moe_workspace(256, 2816, 128, 8, 704, 2112, dev)
    y = torch.empty(256, 2816, dtype=torch.float32, device=dev)
    ms = _time_op(lambda: dg.moe_ffn(m["x"], m["wr"], m["w_gu"], m["w_d"], 8, m["ws_gu"], m["ws_d"],
                                     workspace=wsm, out=y, stream=stream), stream, flush=flush)
    nbytes = sum(t.numel() * 2 for t in (m["wr"], m["w_gu"], m["w_d"], m["ws_gu"], m["ws_d"]))
    gbs = nbytes / (ms / 1e3) / 1e9
    out["moe"] = dict(us=round(ms * 1e3, 2), bound="hbm", achieved_gbs=round(gbs, 1),
                      frac=round(gbs / hbm, 4), bytes=nbytes)
    # the same MoE with e4m3 experts (1 byte per weight + one fp32 scale per row)
    q = {}
    for name in ("w_gu", "w_d", "ws_gu", "ws_d"):
        q[name], q[name + "_scale"] = dg.quantize_e4m3(m[name])
    ms = _time_op(lambda: dg.moe_ffn_e4m3(m["x"], m["wr"], q["w_gu"], q["w_gu_scale"], q["w_d"],
                                          q["w_d_scale"], 8, q["ws_gu"], q["ws_gu_scale"],
                                          q["ws_d"], q["ws_d_scale"], workspace=wsm, out=y,
                                          stream=stream), stream, flush=flush)
    nbytes = m["wr"].numel() * 2 + sum(m[n].numel() + q[n + "_scale"].numel() * 4
                                       for n in ("w_gu", "w_d", "ws_gu", "ws_d"))
    gbs = nbytes / (ms / 1e3) / 1e9
    out["moe_e4m3"] = dict(us=round(ms * 1e3, 2), bound="hbm", achieved_gbs=round(gbs, 1),
                           frac=round(gbs / hbm, 4), bytes=nbytes)
    del m, q, wsm, y, flush
    return out


def step_bytes(shape, prefix, experts="bf16", head="bf16"):
    """Algorithmic HBM bytes of one denoise step at committed length `prefix`: every weight the
    step reads once (QKV, O, router, all routed experts' gate/up and down, the shared expert; all
    128 experts are routed at these shapes) per layer, the K/V cache read over prefix + canvas
    keys and the canvas K/V written per layer, and the LM head's table.  Activations (a few MB per
    layer) are left out.  e4m3: one byte per weight plus one fp32 scale per weight row; NVFP4:
    half a byte per weight, one e4m3 block scale per 16 weights, one fp32 scale per row."""
    d, hq, hkv, hd = shape["d_model"], shape["n_heads"], shape["n_kv_heads"], shape["head_dim"]
    e, h, hs, v = shape["n_experts"], shape["expert_hidden"], shape["shared_hidden"], shape["vocab"]
    dense = ((hq + 2 * hkv) * hd * d + d * hq * hd + e * d) * 2
    n_w = e * 3 * h * d + 3 * hs * d                     # expert weights
    n_rows = e * 2 * h + e * d + 2 * hs + d               # expert weight rows
    per_w = {"bf16": 2.0, "e4m3": 1.0, "nvfp4": 0.5 + 1.0 / 16}[experts]
    ex = int(n_w * per_w) + (0 if experts == "bf16" else n_rows * 4)
    kv = (prefix + CANVAS) * hkv * hd * 2 * 2 + CANVAS * hkv * hd * 2 * 2
    lm = v * d * 2 if head == "bf16" else v * d + v * 4
    return shape["n_layers"] * (dense + ex + kv) + lm


def live_kernel_table(model, stream, L):
    """Live per-kernel table: for each kernel kind, one denoise step with CUDA events around that
    kind's launches (on their stream); microseconds per launch and per step, and share."""
    import ctypes as C
    table = {}
    for kname, kk in L.KERNEL_KINDS.items():
        L.check(L.lib().dg_profile_kernel(kk, 64), "dg_profile_kernel")
        model.kv_truncate(PROMPT)
        model.canvas_init(9, 0, stream)
        model.denoise_step(1, stream)
        model.sample_update(1, stream)
        torch.cuda.synchronize()
        buf2 = (C.c_float * 64)()
        nrec = L.lib().dg_profile_read(buf2, 64)
        L.check(L.lib().dg_profile_kernel(0, 0), "dg_profile_kernel")
        if nrec > 0:
            tot = sum(buf2[:nrec]) * 1e3
            table[kname] = dict(launches=nrec, us_per_launch=round(tot / nrec, 2),
                                us_per_step=round(tot, 1))
    step_us = sum(v["us_per_step"] for v in table.values())
    for v in table.values():
        v["share"] = round(v["us_per_step"] / step_us, 4)
    return table


def decode(model, seed, out_ids, out_states, stream, fixed=True):
    model.kv_truncate(PROMPT)
    for b in range(BLOCKS):
        model.canvas_init(seed, b, stream)
        # adaptive mode enqueues the 48-step cap; steps after the device-side stop are no-ops
        for t in range(1, (FIXED_STEPS if fixed else MAX_STEPS) + 1):
            model.denoise_step(t, stream)
            model.sample_update(t, stream)
        model.commit_block(out_ids[b * CANVAS:(b + 1) * CANVAS], out_states[b], stream)


def run_ours(args, rank, world, local_rank):
    from block_text_diffusion_dg_b200 import (DiffusionModel, generate, make_config, quantize_experts,
                                              quantize_head)
    from block_text_diffusion_dg_b200 import _lib as L
    from dg_synth import SHAPES, model_weights, uniform_ids
    import torch.distributed as dist

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    shape = SHAPES["a4b"]
    cap = PROMPT + BLOCKS * CANVAS + CANVAS
    f8 = args.experts != "bf16"  # quantised experts (e4m3 or NVFP4)
    f4 = args.experts == "nvfp4"
    cfg = make_config(shape, kv_capacity=cap, fixed_steps=FIXED_STEPS,
                      prefill_chunk=1024 if f4 else PREFILL_CHUNK, experts=args.experts, head=args.head)
    weights = model_weights("a4b", seed=1000 + rank, device=dev)
    if args.head == "e4m3":
        weights = quantize_head(weights)
    if f8:  # the bf16 expert matrices are dropped once quantised
        weights = quantize_experts(weights, fmt=args.experts)
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    model = DiffusionModel(cfg, weights, device=dev)
    stream = torch.cuda.current_stream(dev)
    prompt = uniform_ids(PROMPT, shape["vocab"], seed=rank).pin_memory()
    prompt_dev = prompt.to(dev)
    out_ids = torch.empty(BLOCKS * CANVAS, dtype=torch.int32, device=dev)
    out_states = torch.empty(BLOCKS, L.STATE_WORDS, dtype=torch.int32, device=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # prefill once (timed separately)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    model.kv_append(prompt_dev, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    prefill_ms = e0.elapsed_time(e1)

    for i in range(args.warmup):
        decode(model, 100 + i, out_ids, out_states, stream)
    model.check_device_status(stream)
    clocks = Clocks(dev)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    n0 = L.lib().dg_launch_count()
    e0.record(stream)
    for i in range(args.steps):
        decode(model, i, out_ids, out_states, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    n1 = L.lib().dg_launch_count()
    barrier()
    ck = clocks.stop()
    ms_max = max_over_ranks(e0.elapsed_time(e1), world, dev)
    model.check_device_status(stream)
    value = replica_throughput(args.steps * BLOCKS * CANVAS, world, ms_max)

    # denoise step time on its own (16 steps of block 0)
    model.kv_truncate(PROMPT)
    model.canvas_init(7, 0, stream)
    e0.record(stream)
    for tt in range(1, FIXED_STEPS + 1):
        model.denoise_step(tt, stream)
        model.sample_update(tt, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    us_step = 1e3 * e0.elapsed_time(e1) / FIXED_STEPS

    # profiled pass: the roofline kernel's launches timed on its stream
    kind = L.KERNEL_KINDS[args.roofline_kernel]
    n_pairs = shape["n_layers"] * FIXED_STEPS
    import ctypes as C
    L.check(L.lib().dg_profile_kernel(kind, n_pairs), "dg_profile_kernel")
    model.kv_truncate(PROMPT)
    model.canvas_init(8, 0, stream)
    for tt in range(1, FIXED_STEPS + 1):
        model.denoise_step(tt, stream)
        model.sample_update(tt, stream)
    torch.cuda.synchronize()
    buf = (C.c_float * n_pairs)()
    rec = L.lib().dg_profile_read(buf, n_pairs)
    if rec < 0:
        L.check(rec, "dg_profile_read")
    L.check(L.lib().dg_profile_kernel(0, 0), "dg_profile_kernel")
    durs = list(buf[:rec])
    avg_ms = sum(durs) / max(1, len(durs))
    hbm, tf_burst, tf_sust, src = peaks()
    d, e, h, k = shape["d_model"], shape["n_experts"], shape["expert_hidden"], shape["top_k"]
    hs = shape["shared_hidden"]
    slots = CANVAS * k
    # algorithmic bytes per launch: every routed expert's weights (all 128 are routed at these
    # shapes) and the shared expert's, which rides in the same launch, plus tokens in and out;
    # e4m3: one byte per weight and per quantised activation, plus the fp32 row scales
    wb = 0.5625 if f4 else 1 if f8 else 2  # NVFP4: half a byte + one e4m3 scale per 16
    scale_b = 4 if f8 else 0  # one fp32 scale per weight row and per quantised token row
    algo = {
        "expert_gate_up": int((e * 2 * h + 2 * hs) * d * wb + (slots + CANVAS) * d * wb)
                          + slots * h * 2 + CANVAS * hs * 2
                          + (e * 2 * h + 2 * hs + slots + CANVAS) * scale_b,
        "expert_down": int((e * h + hs) * d * wb + slots * h * wb + CANVAS * hs * wb)
                       + (slots + CANVAS) * d * 4 + (e * d + d + slots + CANVAS) * scale_b,
        "lm_head": shape["vocab"] * d * 2 + CANVAS * d * 2 + CANVAS * (shape["vocab"] // 256) * 16,
    }
    # DRAM bytes (read + write) of one launch from the ncu captures summarised in profiles/
    # (dram__bytes_read.sum + dram__bytes_write.sum of the standalone MoE operator's launches);
    # None for the NVFP4 kernels until they are captured
    traffic = ({} if f4 else
               {"expert_gate_up": 527095808 + 4883712, "expert_down": 286693632 + 5061632} if f8
               else {"expert_gate_up": 1052264192 + 5308672, "expert_down": 523554560 + 4555520})
    roof = None
    if args.roofline_kernel in algo and rec:
        achieved = algo[args.roofline_kernel] / (avg_ms / 1e3) / 1e9
        roof = dict(kernel=args.roofline_kernel, bound="hbm", achieved=round(achieved, 1),
                    peak=hbm, unit="GB/s", frac=round(achieved / hbm, 4),
                    traffic=traffic.get(args.roofline_kernel),
                    launches_timed=rec, avg_launch_us=round(avg_ms * 1e3, 2),
                    algorithmic_bytes_per_launch=algo[args.roofline_kernel],
                    peak_source=f"{src} (MEASURED_PEAKS.json hbm_gbs)")

    table = live_kernel_table(model, stream, L)

    # the whole denoise step against the HBM roofline (block 0: 4,096 committed positions)
    sb = step_bytes(shape, PROMPT, args.experts, args.head)
    step_gbs = sb / (us_step / 1e6) / 1e9
    step_roof = dict(bound="hbm", achieved=round(step_gbs, 1), peak=hbm, unit="GB/s",
                     frac=round(step_gbs / hbm, 4), algorithmic_bytes_per_step=sb,
                     us_per_step=round(us_step, 1), floor_us=round(sb / hbm / 1e3, 1),
                     peak_source=f"{src} (MEASURED_PEAKS.json hbm_gbs)")

    # adaptive stop, 48-step cap ([canvas] step 3): random-init weights never reach the stop
    # rule, so every block runs to the cap
    cfg_a = make_config(shape, kv_capacity=cap, fixed_steps=0, max_steps=MAX_STEPS,
                        prefill_chunk=PREFILL_CHUNK, experts=args.experts, head=args.head)
    model_a = DiffusionModel(cfg_a, weights, device=dev)
    model_a.kv_append(prompt_dev, stream)
    decode(model_a, 300, out_ids, out_states, stream, fixed=False)  # warm-up
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    decode(model_a, 301, out_ids, out_states, stream, fixed=False)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_a = max_over_ranks(e0.elapsed_time(e1), world, dev)
    st_a = out_states.cpu()
    model_a.check_device_status(stream)
    model_a.close()
    adaptive = dict(value=round(replica_throughput(BLOCKS * CANVAS, world, ms_a), 2), unit="tok/s",
                    max_steps=MAX_STEPS, ms_per_decode=round(ms_a, 2),
                    steps_per_block=[int(x) for x in st_a[:, 1].tolist()],
                    would_stop=[int(x) for x in st_a[:, 2].tolist()])

    # long context ([canvas] step 1 prefill; the pages' weak spot is the time to the first
    # output): a 32,768-token prompt in 4,096-token passes, then the first block of 16 steps
    cfg_l = make_config(shape, kv_capacity=LONG_PROMPT + 2 * CANVAS, fixed_steps=FIXED_STEPS,
                        prefill_chunk=PREFILL_CHUNK, experts=args.experts, head=args.head)
    model_l = DiffusionModel(cfg_l, weights, device=dev)
    long_prompt = uniform_ids(LONG_PROMPT, shape["vocab"], seed=77 + rank).to(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    torch.cuda.synchronize()
    barrier()
    ev[0].record(stream)
    model_l.kv_append(long_prompt, stream)
    ev[1].record(stream)
    model_l.canvas_init(5, 0, stream)
    for tt in range(1, FIXED_STEPS + 1):
        model_l.denoise_step(tt, stream)
        model_l.sample_update(tt, stream)
    ev[2].record(stream)
    model_l.commit_block(out_ids[:CANVAS], out_states[0], stream)
    ev[3].record(stream)
    torch.cuda.synchronize()
    model_l.check_device_status(stream)
    model_l.close()
    del long_prompt
    long_ctx = dict(prompt=LONG_PROMPT, prefill_ms=round(max_over_ranks(ev[0].elapsed_time(ev[1]), world, dev), 2),
                    us_per_denoise_step=round(1e3 * ev[1].elapsed_time(ev[2]) / FIXED_STEPS, 1),
                    first_block_ms=round(max_over_ranks(ev[0].elapsed_time(ev[3]), world, dev), 2),
                    note="first_block_ms: prompt prefill + 16 denoise steps + commit of block 0")

    # small-batch canvases: BATCH sequences (own prompts and caches) decoded in lockstep, every
    # denoise step carrying BATCH x 256 canvas tokens through one weight stream
    cfg_b = make_config(shape, kv_capacity=cap, fixed_steps=FIXED_STEPS,
                        prefill_chunk=PREFILL_CHUNK, experts=args.experts, head=args.head, batch=BATCH)
    model_b = DiffusionModel(cfg_b, weights, device=dev)
    prompts_b = torch.stack([uniform_ids(PROMPT, shape["vocab"], seed=90 + BATCH * rank + b)
                             for b in range(BATCH)]).to(dev)
    model_b.kv_append(prompts_b, stream)
    ids_b = torch.empty(BATCH * CANVAS, dtype=torch.int32, device=dev)
    st_b = torch.empty(BATCH, L.STATE_WORDS, dtype=torch.int32, device=dev)

    def decode_b(seed):
        model_b.kv_truncate(PROMPT)
        for blk in range(BLOCKS):
            model_b.canvas_init(seed, blk, stream)
            for tt in range(1, FIXED_STEPS + 1):
                model_b.denoise_step(tt, stream)
                model_b.sample_update(tt, stream)
            model_b.commit_block(ids_b, st_b, stream)

    decode_b(400)  # warm-up
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    decode_b(401)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_b = max_over_ranks(e0.elapsed_time(e1), world, dev)
    model_b.kv_truncate(PROMPT)
    model_b.canvas_init(402, 0, stream)
    e0.record(stream)
    for tt in range(1, FIXED_STEPS + 1):
        model_b.denoise_step(tt, stream)
        model_b.sample_update(tt, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    us_step_b = 1e3 * e0.elapsed_time(e1) / FIXED_STEPS
    table_b = live_kernel_table(model_b, stream, L)
    model_b.check_device_status(stream)
    model_b.close()
    del prompts_b
    batched = dict(batch=BATCH, value=round(replica_throughput(BATCH * BLOCKS * CANVAS, world, ms_b), 2),
                   unit="tok/s", ms_per_decode=round(ms_b, 2), us_per_denoise_step=round(us_step_b, 1),
                   note=f"{BATCH} sequences x 4 blocks x 256 tokens, 16 fixed steps, lockstep",
                   kernels_live=table_b)

    ops = run_ops(dev, stream, hbm, tf_burst)

    # end to end through the public API, pinned host buffers in and out
    host_ids = torch.empty(BLOCKS * CANVAS, dtype=torch.int32).pin_memory()
    host_states = torch.empty(BLOCKS, L.STATE_WORDS, dtype=torch.int32).pin_memory()
    e2e_ms = []
    for i in range(1 + args.e2e_steps):
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        dev_prompt = prompt.to(dev, non_blocking=True)
        model.kv_truncate(0)
        ids, states = generate(model, dev_prompt, BLOCKS, seed=500 + i, stream=stream)
        host_ids.copy_(ids, non_blocking=True)
        host_states.copy_(states, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if i > 0:
            e2e_ms.append(e0.elapsed_time(e1))
    e2e_val = replica_throughput(BLOCKS * CANVAS, world, max_over_ranks(max(e2e_ms), world, dev))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = cpu_oracle_sample()
        cpu = dict(value=r["value"], unit="tok/s", cores=r["cores"], kind="oracle", sample=r["sample"])
    if rank == 0:
        out = dict(metric="committed canvas tokens/s", value=round(value, 2), unit="tok/s",
                   n_gpus=world, steps=args.steps, warmup=args.warmup,
                   ms_per_step=round(ms_max / args.steps, 3), higher_is_better=True,
                   scaling="weak", vs_baseline=None,
                   dtype={"bf16": "bf16", "e4m3": "bf16+e4m3", "nvfp4": "bf16+nvfp4"}[args.experts]
                         + ("+e4m3 head" if args.head == "e4m3" else ""),
                   data="synthetic",
                   config=dict(workload={"bf16": WORKLOAD, "e4m3": WORKLOAD_E4M3,
                                         "nvfp4": WORKLOAD_NVFP4}[args.experts]
                               + (", LM head on e4m3 operands" if args.head == "e4m3" else ""),
                               global_batch=world,
                               seq_len=PROMPT + BLOCKS * CANVAS,
                               parallelism=f"replicas x{world}",
                               l2="inputs larger than L2: ~%d GB of weights streamed per denoise "
                                  "step" % (15 if f4 else 25 if f8 else 49)),
                   us_per_denoise_step=round(us_step, 1), prefill_ms=round(prefill_ms, 2),
                   roofline=roof, step_roofline=step_roof, adaptive_stop=adaptive,
                   long_context=long_ctx, small_batch=batched,
                   cpu_baseline=cpu,
                   e2e=dict(value=round(e2e_val, 2), unit="tok/s",
                            h2d_bytes_per_step=prompt.numel() * 4,
                            d2h_bytes_per_step=host_ids.numel() * 4 + host_states.numel() * 4,
                            includes="prompt H2D, 4096-token prefill, 4 blocks, ids D2H"),
                   gpu_launches=int((n1 - n0) // args.steps), clocks=ck,
                   kernels_live=table, ops=ops)
        print(json.dumps(out), flush=True)
    model.close()


def run_profile(args):
    """One region for ncu: after warm-up, the profiled calls sit between profiler start/stop.

    decode_step: the full decode model, prompt prefilled, then canvas init + one denoise step
                 + one sampler update.
    decode_step_small: the same with 2 layers and a 32768-token vocabulary (a few GB on the
                 device, for multi-pass captures of single kernels).
    decode_step_e4m3: decode_step with e4m3 experts.
    moe:         the MoE operator at 256 tokens, d 2816, 128 experts top-8 + shared (1.5 GB).
    moe_e4m3:    the same operator with e4m3 experts (0.8 GB of expert weights).
    moe_nvfp4:   the same operator with NVFP4 experts (0.45 GB of expert weights).
    attention:   canvas attention, 16/8 heads x 128, 4096 + 256 keys.
    sampler:     the sampler on bf16 logits [256, 262144].
    """
    import block_text_diffusion_dg_b200 as dg
    from dg_synth import SHAPES, attention_inputs, model_weights, moe_inputs, sampler_logits, uniform_ids
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    prof = torch.cuda.profiler
    if args.profile in ("decode_step", "decode_step_small", "decode_step_e4m3"):
        shape = dict(SHAPES["a4b"])
        if args.profile == "decode_step_small":
            shape.update(n_layers=2, vocab=32768)
        f8 = args.profile == "decode_step_e4m3"
        cfg = dg.make_config(shape, kv_capacity=PROMPT + BLOCKS * CANVAS + CANVAS,
                             prefill_chunk=PREFILL_CHUNK,
                             fixed_steps=FIXED_STEPS, experts="e4m3" if f8 else "bf16")
        w = model_weights(shape, seed=1000, device=dev)
        if f8:
            w = dg.quantize_experts(w)
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        model = dg.DiffusionModel(cfg, w, device=dev)
        model.kv_append(uniform_ids(PROMPT, shape["vocab"], seed=0).to(dev))
        model.canvas_init(1, 0)
        model.denoise_step(1)
        model.sample_update(1)
        torch.cuda.synchronize()
        prof.start()
        model.canvas_init(2, 0)
        model.denoise_step(1)
        model.sample_update(1)
        torch.cuda.synchronize()
        prof.stop()
        model.check_device_status()
        model.close()
        return
    if args.profile == "moe":
        m = {k: (None if v is None else v.to(dev)) for k, v in moe_inputs(seed=0).items()}
        ws = dg.moe_workspace(256, 2816, 128, 8, 704, 2112, dev)
        call = lambda: dg.moe_ffn(m["x"], m["wr"], m["w_gu"], m["w_d"], 8, m["ws_gu"], m["ws_d"],
                                  workspace=ws)
    elif args.profile == "moe_e4m3":
        m = {k: (None if v is None else v.to(dev)) for k, v in moe_inputs(seed=0).items()}
        q = {}
        for name in ("w_gu", "w_d", "ws_gu", "ws_d"):
            q[name], q[name + "_scale"] = dg.quantize_e4m3(m[name])
            m[name] = None
        ws = dg.moe_workspace(256, 2816, 128, 8, 704, 2112, dev)
        call = lambda: dg.moe_ffn_e4m3(m["x"], m["wr"], q["w_gu"], q["w_gu_scale"], q["w_d"],
                                       q["w_d_scale"], 8, q["ws_gu"], q["ws_gu_scale"], q["ws_d"],
                                       q["ws_d_scale"], workspace=ws)
    elif args.profile == "moe_nvfp4":
        m = {k: (None if v is None else v.to(dev)) for k, v in moe_inputs(seed=0).items()}
        q = {}
        for name in ("w_gu", "w_d", "ws_gu", "ws_d"):
            q[name] = dg.quantize_nvfp4(m[name])
            m[name] = None
        ws = dg.moe_workspace(256, 2816, 128, 8, 704, 2112, dev)
        call = lambda: dg.moe_ffn_nvfp4(m["x"], m["wr"], q["w_gu"], q["w_d"], 8, q["ws_gu"],
                                        q["ws_d"], workspace=ws)
    elif args.profile == "attention":
        q, k, v = (t.to(dev) for t in attention_inputs(seed=0))
        vt = v.transpose(1, 2).contiguous()
        call = lambda: dg.canvas_attention(q, k, vt, 4096 + 256)
    else:
        x = sampler_logits(256, 262144, seed=0).to(dev)
        s = dg.Sampler(256, 262144)
        s.reset()
        call = lambda: s.step(x, seed=0, block=0, step=1)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    prof.start()
    call()
    torch.cuda.synchronize()
    prof.stop()


def main():
    args = parse()
    if args.profile:
        run_profile(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
