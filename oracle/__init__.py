"""CPU oracle for the block-text-diffusion denoise path (test infrastructure only).

This package is a plain, slow, obviously-correct restatement of what the denoise
hot path computes.  It exists so that tests, the smoke check and the benchmark's
CPU-baseline leg can compare the CUDA library against an independent answer.
Nothing on the product path imports it: the CUDA library and its Python binding
share no code, table or constant with this package, and this package imports
nothing from them.

Arithmetic is numpy in float64 unless stated otherwise.  Where the GPU path
stores an intermediate in bf16 or fp32, the oracle rounds at the same point
(round-to-nearest-even, `numerics.round_storage`) and computes everything else
in float64.

Sources (the pages describe the method in prose only; no code, no equations):

[canvas]  alphalab.site, "DiffusionGemma 是什麼？看懂 256-token Canvas 與本機 A/B Test",
          section "256-token Canvas 怎麼從雜訊變成文字？", steps (1) prompt encoded
          left-to-right into a reusable KV cache, (2) canvas filled with ids drawn
          uniformly from the whole vocabulary, (3) repeated denoising: confident tokens
          stay, uncertain positions may be re-randomised; at most 48 steps; stop when the
          mean canvas entropy is below 0.005 and the highest-probability prediction is
          identical on two consecutive steps, (4) the converged block is committed to the
          KV cache before the next canvas starts.
[uniform] k7ail.com (Arabic rendering of the MarkTechPost launch article),
          section "كيف يعمل نشر النص" (how text diffusion works): uniform-state diffusion;
          a 256-token canvas processed in parallel; bidirectional attention during
          denoising (every canvas token attends to every other); a token whose
          confidence drops can be re-noised by the sampler and replaced later.
[arch]    same article, section "العمارة" (architecture): prefill uses causal attention
          and writes the KV cache, denoising uses bidirectional attention; block
          autoregressive diffusion commits each denoised 256-token block to the KV cache
          and starts a new canvas conditioned on that history; the backbone is the
          Gemma 4 26B-A4B mixture-of-experts.
[course]  ai-directories.com, "Diffusion Gemma - Google AI教學課程", part 2, table 2.1
          (lay out a 256-token canvas of random placeholders, denoise over several
          rounds, lock high-confidence tokens first, use them to fix the rest) and
          table 2.2 (MoE, 26B total / 3.8B active).
[blog]    aitoday.skyai.vn (Vietnamese rendering of Google's launch post), section
          "Cách thức hoạt động của khuếch tán văn bản": canvas of random placeholder
          tokens, iterative refinement that locks correct tokens and uses them as
          context; a new "diffusion head" on the Gemma 4 base.
[pl]      jakiprompt.pl, "Diffusion Gemma – nowy model językowy Google", section
          "Wymagania sprzętowe" (hardware requirements): the model ships as BF16, FP8 and NVFP4
          weights (52 / 27 / 18 GB); [course] table 2.2 quotes fp8 on an H100.
[philox]  Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as easy as 1, 2, 3",
          SC'11: the Philox4x32-10 counter-based generator.

Readings taken where the pages are silent (each is also a parameter or a flag):
confidence is the maximum softmax probability at temperature 1, locked when
>= 0.9; locks are stateless (re-decided every step from that step's logits);
entropy is in nats over the full vocabulary and averaged over all canvas
positions; the argmax takes the lowest index among equal maxima; the router
takes a softmax over all experts, keeps the top-k (lowest index on ties) and
renormalises the k probabilities; a shared expert is added with weight 1;
RoPE is rotate-half with theta 10000 at absolute positions; RMSNorm is
pre-norm with eps 1e-6; embeddings are tied with the LM head; commit re-encodes
the final argmax block causally, exactly like the prompt; FP8 experts are e4m3 with
one scale per weight row and per activation row (quant.py); NVFP4 is e2m1 with an e4m3
scale per 16-element block and an fp32 row scale.

Parity status: every function here is pinned by a CPU test against a closed
form, a brute-force evaluation, a library routine, published known-answer
vectors or an invariant (see tests/test_oracle_*.py).  No function is
"parity unpinned".
"""
