/*
 * dg.h -- C ABI of libdg, the B200 (sm_100a) denoise path for block text diffusion.
 *
 * What the path computes (sources, all prose web pages; no code is printed on them):
 *  [canvas]  alphalab.site, "DiffusionGemma: 256-token Canvas and a local A/B test",
 *            section "how the 256-token canvas turns noise into text", steps 1-4:
 *            causal prompt encode into a reusable KV cache; a canvas of ids drawn
 *            uniformly from the whole vocabulary; repeated denoising where confident
 *            tokens stay and uncertain ones are re-randomised, at most 48 steps, stopping
 *            when mean canvas entropy < 0.005 and the argmax prediction is identical on two
 *            consecutive steps; commit of the converged block to the KV cache.
 *  [uniform] k7ail.com (Arabic rendering of the MarkTechPost launch article), section
 *            "how text diffusion works": uniform-state diffusion, bidirectional attention
 *            over the whole canvas while denoising, re-noising of tokens whose confidence
 *            drops.
 *  [arch]    same article, section "architecture": causal prefill writes the KV cache,
 *            bidirectional denoise; block-autoregressive diffusion commits each block to the
 *            KV cache; Gemma 4 26B-A4B mixture-of-experts backbone.
 *  [course]  ai-directories.com course outline, part 2 tables 2.1 (lock high-confidence
 *            tokens first) and 2.2 (MoE 26B total, 3.8B active).
 *  [philox]  Salmon et al., "Parallel random numbers: as easy as 1, 2, 3" (SC'11).
 *
 * Conventions for every entry point:
 *  - All pointers named d_* are DEVICE pointers owned by the caller; the library keeps
 *    raw copies and never frees them.  Host pointers are only read during the call.
 *  - `stream` is a cudaStream_t passed as void*; every call only enqueues work on it and
 *    returns without synchronising.  NULL means the legacy default stream.
 *  - Return value: DG_OK (0) or a negative DG_ERR_* code.  Argument checks run before any
 *    launch, so a failed check enqueues nothing.  dg_last_error() gives a text for the
 *    most recent failure on the calling thread.
 *  - Tensors are dense row-major; shapes are written [outer, ..., inner].
 *  - bf16 is IEEE binary32's upper half; "bf16 config" stores weights, Q/K/V, the KV cache
 *    and activations between kernels in bf16 (round-to-nearest-even), keeps the residual
 *    stream, router logits and softmax statistics in fp32, and accumulates in fp32.  The
 *    "fp32 config" stores everything in fp32.
 */
#ifndef DG_H_
#define DG_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DG_API __attribute__((visibility("default")))
#else
#define DG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = -1, /* null pointer, bad size or shape, misaligned pointer */
  DG_ERR_CAPACITY = -2,    /* KV cache or workspace too small for the request */
  DG_ERR_CUDA = -3,        /* a CUDA call or launch failed; text in dg_last_error() */
  DG_ERR_TIMEOUT = -4,     /* a device wait gave up (read by dg_check_device_status) */
  DG_ERR_UNSUPPORTED = -5  /* shape outside what the kernels implement */
};

/* Model storage types.  DG_DTYPE_BF16_E4M3 is the bf16 model with the FP8 expert format
 * ([pl]: the model ships as BF16, FP8 or NVFP4 weights): the routed and shared expert
 * weights are e4m3 codes with one fp32 scale per weight row, and the expert GEMMs take e4m3
 * activations, quantised per row on the fly (scale = max|row| / 448, codes = rn_satfinite(x /
 * scale)); attention, router, norms and the LM head stay bf16. */
enum { DG_DTYPE_BF16 = 0, DG_DTYPE_FP32 = 1, DG_DTYPE_BF16_E4M3 = 2, DG_DTYPE_BF16_NVFP4 = 3 };
/* DG_DTYPE_BF16_NVFP4 is the same with the NVFP4 expert format ([pl]: 18 GB; [blog]: NVFP4
 * kernels on Blackwell): e2m1 codes (two per byte, low nibble first, rows at
 * DG_E4M3_PITCH(K / 2) bytes), one e4m3 scale per 16 codes in 512-byte atoms (see
 * dg_quantize_nvfp4) and one fp32 scale per row; the expert GEMMs take NVFP4 activations. */

/* Model and decode configuration.  Shapes follow the pages' model ([course], [arch]). */
typedef struct dg_config {
  int32_t n_layers;
  int32_t d_model;        /* bf16: multiple of 64 */
  int32_t n_heads;        /* query heads Hq */
  int32_t n_kv_heads;     /* key/value heads Hkv; Hq % Hkv == 0 (grouped-query attention) */
  int32_t head_dim;       /* bf16: 128; fp32: even, <= 128 */
  int32_t n_experts;      /* E */
  int32_t top_k;          /* k <= min(E, 8) */
  int32_t expert_hidden;  /* h; bf16: multiple of 64 */
  int32_t shared_hidden;  /* hs (0 = no shared expert); bf16: multiple of 64 */
  int32_t vocab;          /* V; bf16: multiple of 256 */
  int32_t canvas;         /* canvas length T; 256 in the pages ([canvas]); 1..256 */
  int32_t kv_capacity;    /* positions the caller's KV cache holds (multiple of 8); L * Hkv * cap
                             and Hkv * hd * cap below 2^31 (long contexts: 256K positions fit) */
  int32_t dtype;          /* DG_DTYPE_BF16, DG_DTYPE_FP32 or DG_DTYPE_BF16_E4M3 */
  float eps;              /* RMSNorm epsilon (1e-6) */
  float rope_theta;       /* RoPE base (10000) */
  double tau;             /* lock threshold on max-probability confidence (0.9) */
  double h_bound;         /* mean-entropy stop bound in nats (0.005, [canvas] step 3) */
  int32_t max_steps;      /* adaptive step cap (48, [canvas] step 3) */
  int32_t fixed_steps;    /* > 0: fixed-step mode, exactly this many steps; 0: adaptive */
  int32_t prefill_chunk;  /* tokens per causal-encode pass of dg_kv_append (0 = canvas); a
                             multiple of 128, <= 4096; larger chunks stream the weights fewer
                             times per prompt at the cost of scratch memory */
  /* Sampler variants (zero = the plain rule above).  The recipe's "entropy_bound" sampler
   * ([canvas], A/B commands: bound 0.1) has no definition on the pages; read as: */
  int32_t lock_rule;      /* 0: lock when conf >= tau; 1: lock when entropy <= entropy_lock */
  double entropy_lock;    /* nats, >= 0 (rule 1) */
  int32_t sticky_locks;   /* 1: a locked position keeps its token for the rest of the block
                             and the commit takes it (0: locks are re-decided every step) */
  float temperature;      /* sampler statistics of softmax(logits / T); 0 or 1 = plain */
  /* Commit encoding ([canvas] step 4, [arch] only say the block is committed to the KV cache):
   * 0: re-encode the committed ids causally, exactly like the prompt;
   * 1: keep the K/V the last denoise step wrote for the canvas (the bidirectional forward of
   *    that step's input canvas), so the commit launches nothing but a copy of the ids. */
  int32_t commit_reuse_kv;
  /* Small-batch canvases (the pages: the advantage is strongest at small-to-medium batch on one
   * accelerator): B independent sequences decoded in lockstep, each with its own KV cache, canvas,
   * sampler state and stop test, sharing every weight stream of a denoise step (B * T tokens per
   * forward).  0 or 1: one sequence.  B > 1 needs a bf16 dtype, canvas % 128 == 0 and
   * B * canvas <= 4096; all sequences hold the same committed length (equal-length prompts, blocks
   * committed together once every canvas has stopped; a stopped canvas is frozen meanwhile), and
   * sequence b draws its Philox stream with key seed + b. */
  int32_t batch;
  /* FP8 LM head (the FP8 weight format of [pl] applied to the tied head; bf16 dtypes only): the
   * head multiplies e4m3 codes of the final normed tokens (quantised per row on the fly,
   * scale = max|row| / 448) by an e4m3 copy of the embedding table with one fp32 scale per
   * vocabulary row (dg_weights.head_codes / head_scale, written by dg_quantize_e4m3 at a pitch of
   * DG_E4M3_PITCH(d)); the canvas embedding gather keeps the bf16 table.  0: bf16 head. */
  int32_t lm_head_e4m3;
} dg_config;

/* Per-layer weights, all device pointers, dtype = config dtype unless noted (bf16 for
 * DG_DTYPE_BF16_E4M3, except the four expert matrices, which are then e4m3 codes).
 * Gate and up projections are stored row-interleaved: row 2j is gate unit j, row 2j+1 is
 * up unit j.  The *_scale arrays are read only with DG_DTYPE_BF16_E4M3 (dg_quantize_e4m3
 * writes codes and scales in this layout).  An e4m3 matrix row of c codes is stored with a
 * pitch of round_up(c, 128) bytes (DG_E4M3_PITCH), so that every 128-byte K slab of every row
 * starts on a 128-byte boundary; the pad bytes are never read. */
#define DG_E4M3_PITCH(cols) ((((cols) + 127) / 128) * 128)
typedef struct dg_layer_weights {
  const float* attn_norm; /* fp32 [d] */
  const void* wqkv;       /* [(Hq + 2 Hkv) * hd, d]: q heads, then k heads, then v heads */
  const void* wo;         /* [d, Hq * hd] */
  const float* ffn_norm;  /* fp32 [d] */
  const void* wr;         /* router [E, d] */
  const void* w_gu;       /* experts gate/up [E, 2h, d] */
  const void* w_d;        /* experts down [E, d, h] */
  const void* ws_gu;      /* shared expert gate/up [2hs, d], or NULL */
  const void* ws_d;       /* shared expert down [d, hs], or NULL */
  const float* w_gu_scale;  /* fp32 [E, 2h], one per w_gu row */
  const float* w_d_scale;   /* fp32 [E, d], one per w_d row */
  const float* ws_gu_scale; /* fp32 [2hs], or NULL */
  const float* ws_d_scale;  /* fp32 [d], or NULL */
  const void* w_gu_sf;      /* DG_DTYPE_BF16_NVFP4: block-scale atoms of w_gu (as written by */
  const void* w_d_sf;       /*   dg_quantize_nvfp4 for the stacked [E * rows, K] matrix),    */
  const void* ws_gu_sf;     /*   of w_d, ws_gu and ws_d; NULL otherwise                       */
  const void* ws_d_sf;
} dg_layer_weights;

typedef struct dg_weights {
  const void* embed;              /* tied embedding / LM head [V, d] */
  const float* final_norm;        /* fp32 [d] */
  const dg_layer_weights* layers; /* HOST array of n_layers entries (copied by dg_create) */
  const void* head_codes;         /* lm_head_e4m3: e4m3 codes of embed [V, DG_E4M3_PITCH(d)] */
  const float* head_scale;        /* lm_head_e4m3: fp32 [V], one per vocabulary row */
} dg_weights;

/* Device-side decode state words (int32), readable by the caller after a block. */
enum {
  DG_STATE_DONE = 0,        /* 1 once the block stopped (adaptive) or ran its fixed steps */
  DG_STATE_STOP_STEP = 1,   /* step whose argmax is committed */
  DG_STATE_WOULD_STOP = 2,  /* first step meeting the stop rule, 0 if none yet */
  DG_STATE_STEPS_RUN = 3,   /* sampler updates applied in this block */
  DG_STATE_LOCKED = 4,      /* positions locked by the last update */
  DG_STATE_ERROR = 5,       /* nonzero: a device wait timed out (DG_ERR_TIMEOUT) */
  DG_STATE_WORDS = 16
};

typedef struct dg_ctx dg_ctx;

/* ---- model context ---------------------------------------------------------------- */

/* Bytes of the KV cache and of the scratch workspace the caller must allocate for cfg.
 * KV cache layout: K [L, Hkv, cap, hd] followed by V transposed [L, Hkv, hd, cap]. */
DG_API int dg_workspace_bytes(const dg_config* cfg, size_t* kv_bytes, size_t* scratch_bytes);

/* Bind weights and caller-allocated buffers (kv: kv_bytes, scratch: scratch_bytes, both
 * 256-byte aligned).  Builds the TMA descriptors, zero-fills kv and scratch on `stream`,
 * and sets the cache length to 0.  Allocates no device memory. */
DG_API int dg_create(const dg_config* cfg, const dg_weights* w, void* d_kv, void* d_scratch,
              void* stream, dg_ctx** out);
DG_API void dg_destroy(dg_ctx* ctx);

/* Committed cache length (host-side counter advanced by dg_kv_append / dg_commit_block). */
DG_API int32_t dg_kv_length(const dg_ctx* ctx);
/* Forget committed positions >= length (0 <= length <= current length). */
DG_API int dg_kv_truncate(dg_ctx* ctx, int32_t length);

/* Causal encode ([canvas] step 1, [arch] prefill): run every layer over ids[0..n) at
 * positions P..P+n-1 with a causal mask and append their K/V to the cache (P += n).
 * d_ids: int32 [n], each in [0, V); a batched context takes [batch, n], row b into sequence b's
 * cache.  Processed in passes of prefill_chunk (else canvas) tokens.
 * DG_ERR_CAPACITY if P + n + canvas > kv_capacity (room for the next canvas is kept). */
DG_API int dg_kv_append(dg_ctx* ctx, const int32_t* d_ids, int32_t n, void* stream);

/* Fill the canvas with ids uniform over [0, V) ([canvas] step 2): Philox4x32-10 with
 * counter (position, 0, block, 0) and key (seed lo32, seed hi32); id = floor(r0 V / 2^32).
 * Resets the decode state words (done, steps, stop step).  Batched: canvas b uses key seed + b. */
DG_API int dg_canvas_init(dg_ctx* ctx, uint64_t seed, uint32_t block, void* stream);

/* Start the current block's denoising over ([canvas] step 4: after a commit the next canvas starts
 * with a fresh decode; the same holds for a block the caller abandons before committing it): zero
 * the decode state words (done, stop step, would-stop step, steps run, locked count, error) and the
 * per-position lock flags, keep the canvas ids and the committed cache.  Later dg_denoise_step and
 * dg_sample_update calls run again (step numbering restarts at 1) even if the block had stopped.
 * dg_canvas_init performs this reset itself before it fills the canvas, so a caller that starts
 * every block with dg_canvas_init never needs this call.  Asynchronous on `stream`. */
DG_API int dg_reset_block(dg_ctx* ctx, void* stream);

/* One denoise forward ([uniform], [canvas] step 3): embed the canvas, run every layer with
 * bidirectional attention over [committed cache | canvas] (canvas K/V are written to the
 * cache slots P..P+T-1 but P does not advance), final RMSNorm, and the LM head fused with
 * per-row vocab-tile softmax statistics (logits are not written to memory).
 * A no-op on the device once the block is done.  step is 1-based. */
DG_API int dg_denoise_step(dg_ctx* ctx, uint32_t step, void* stream);

/* Sampler and stop test for step `step` ([canvas] step 3, [uniform], [course] 2.1):
 * merge the statistics to conf (max probability), entropy (nats) and argmax (lowest
 * index on ties); next canvas id = argmax if conf >= tau else Philox draw with counter
 * (position, step, block, 1); mean entropy and the two-step argmax equality decide the
 * stop, all on the device.  A no-op once the block is done. */
DG_API int dg_sample_update(dg_ctx* ctx, uint32_t step, void* stream);

/* Commit ([canvas] step 4, [arch]): copy the stop step's argmax block to d_out_ids (int32
 * [T], batched [batch * T], may be NULL), the decode state words to d_state (int32
 * [DG_STATE_WORDS], batched [batch, DG_STATE_WORDS], may be NULL), then causally re-encode the block into the cache (P += T), or with commit_reuse_kv
 * keep the canvas K/V of the last denoise step in place (P += T). */
DG_API int dg_commit_block(dg_ctx* ctx, int32_t* d_out_ids, int32_t* d_state, void* stream);

/* Device buffers of the context (for inspection; owned by the caller's scratch):
 * canvas int32 [T], argmax int32 [T], entropy fp32 [T], conf fp32 [T], state int32 [16]; a
 * batched context has [batch * T] (sequence-major) and state [batch, 16]. */
DG_API int dg_get_buffers(const dg_ctx* ctx, int32_t** canvas, int32_t** argmax, float** entropy,
                   float** conf, int32_t** state);

/* Blocking: synchronise `stream` and return DG_ERR_TIMEOUT if a device wait gave up, or
 * DG_ERR_INVALID_ARG if a token id outside [0, V) reached the embedding gather (from the caller's
 * ids, or an argmax over a row of NaN logits): such an id is never used as an address, row 0 of
 * the table is read in its place and the results of that call are invalid.  The error word stays
 * set for the life of the context; once it is set, later device waits give up early. */
DG_API int dg_check_device_status(dg_ctx* ctx, void* stream);

/* ---- standalone operators (the same kernels the context runs) -------------------- */

/* Sampler over given logits ([canvas] step 3): d_logits [rows, V] (dtype), one call per
 * step, two launches (a streaming pass over the logits, then one warp per row to merge, lock /
 * re-noise and run the stop test).  Logits are finite or -inf (a masked vocabulary entry:
 * probability 0, no contribution to the entropy); a logit below -1e30 counts as masked, and every
 * row needs a logit above -1e30.  d_state int32[DG_STATE_WORDS] and the workspace carry the stop
 * test across calls; zero both (dg_sampler_reset) before step 1.  Outputs: d_canvas (next ids),
 * d_argmax, d_entropy, d_conf, each [rows].  Requires V % 8 == 0, rows <= 1024. */
DG_API int dg_sampler_workspace_bytes(int32_t rows, int32_t vocab, size_t* bytes);
DG_API int dg_sampler_reset(int32_t rows, int32_t vocab, void* d_workspace, int32_t* d_state,
                     void* stream);
DG_API int dg_sampler_step(const void* d_logits, int32_t dtype, int32_t rows, int32_t vocab,
                    uint64_t seed, uint32_t block, uint32_t step, double tau, double h_bound,
                    int32_t max_steps, int32_t fixed_steps, void* d_workspace,
                    int32_t* d_canvas, int32_t* d_argmax, float* d_entropy, float* d_conf,
                    int32_t* d_state, void* stream);

/* The sampler step above without a caller-provided workspace (the pages have no
 * counterpart: this is a deployment variant).  For callers that cannot allocate device memory,
 * such as a host framework whose memory pool owns the whole device budget, or a latency-critical
 * path that may not risk cudaMalloc's implicit device synchronisation.  Its temporaries and the
 * step-to-step stop-test state live in one file-scope device array of about 266 KB, held by every
 * GPU that loads the library until the process exits.  Limits: rows <= 256, V <= 262144,
 * V % 8 == 0; larger requests return DG_ERR_CAPACITY.  Arguments and outputs are those of
 * dg_sampler_step; the caller zeroes d_state before step 1.  The first call on each device looks
 * up the array's device address (cudaGetSymbolAddress) with that device current, so make that
 * first call before any stream capture.  The address is kept per CUDA context: the first call
 * after the device's context was replaced (cudaDeviceReset) looks it up again, under the same
 * rule.  Every call on a device shares the one array, which keeps
 * the previous call's contents: calls that overlap on the GPU (other streams, other threads) race,
 * so serialise them.  Allocates no memory (no cudaMalloc, cudaFree or allocating library call). */
DG_API int dg_sampler_step_static(const void* d_logits, int32_t dtype, int32_t rows,
                                  int32_t vocab, uint64_t seed, uint32_t block, uint32_t step,
                                  double tau, double h_bound, int32_t max_steps,
                                  int32_t fixed_steps, int32_t* d_canvas, int32_t* d_argmax,
                                  float* d_entropy, float* d_conf, int32_t* d_state, void* stream);

/* Canvas attention ([uniform], [arch]): bf16 q [Hq, Tq, 128] (head stride Tq), keys
 * k [Hkv, ldk, 128] and values TRANSPOSED vt [Hkv, 128, ldk], keys 0..n_keys-1 used;
 * causal_prefix < 0: no mask; >= 0: query t sees keys n <= causal_prefix + t.
 * Output o bf16 [T, Hq*128].  Requires Tq % 128 == 0, T <= Tq, ldk % 8 == 0, n_keys >= 1. */
DG_API int dg_attention_workspace_bytes(int32_t n_heads, int32_t n_kv_heads, int32_t tq,
                                 int32_t n_keys, size_t* bytes);
DG_API int dg_canvas_attention(const void* d_q, const void* d_k, const void* d_vt, void* d_o,
                        int32_t n_heads, int32_t n_kv_heads, int32_t t, int32_t tq,
                        int32_t n_keys, int32_t ldk, int32_t causal_prefix, float scale,
                        void* d_workspace, size_t workspace_bytes, void* stream);

/* Top-k routed MoE FFN ([course] 2.2, [arch]): x bf16 [T, d] (already normalised),
 * router wr bf16 [E, d], experts w_gu [E, 2h, d] (row-interleaved gate/up), w_d [E, d, h],
 * optional shared expert ws_gu [2hs, d], ws_d [d, hs] (NULL, hs = 0 for none).
 * y fp32 [T, d] = (residual or 0) + sum over slots in order of w * expert(x) + shared(x).
 * Router: softmax over all E, top-k lowest index on ties, weights renormalised over k.
 * Optional outputs: ids int32 [T, k], weights fp32 [T, k], router logits fp32 [T, E].
 * Shapes: 1 <= T <= 4096; d a multiple of 64 in [128, 4096]; E a multiple of 4, <= 128 (one
 * router tile); 1 <= k <= min(8, E); h, hs multiples of 64.  Other shapes return
 * DG_ERR_INVALID_ARG (or DG_ERR_UNSUPPORTED for T > 4096) before any launch. */
DG_API int dg_moe_workspace_bytes(int32_t t, int32_t d, int32_t n_experts, int32_t top_k,
                           int32_t hidden, int32_t shared_hidden, size_t* bytes);
DG_API int dg_moe_ffn(const void* d_x, const float* d_residual, const void* d_wr, const void* d_w_gu,
               const void* d_w_d, const void* d_ws_gu, const void* d_ws_d, float* d_y,
               int32_t* d_ids, float* d_weights, float* d_router_logits, int32_t t, int32_t d,
               int32_t n_experts, int32_t top_k, int32_t hidden, int32_t shared_hidden,
               void* d_workspace, size_t workspace_bytes, void* stream);

/* The same MoE with e4m3 experts (the FP8 format of DG_DTYPE_BF16_E4M3): w_gu, w_d, ws_gu,
 * ws_d are e4m3 codes in the layouts above, rows at DG_E4M3_PITCH, with fp32 row scales w_gu_scale [E, 2h],
 * w_d_scale [E, d], ws_gu_scale [2hs], ws_d_scale [d] (the shared ones NULL when hs = 0).
 * x and the router stay bf16; x is quantised per token and each expert's SiLU-GLU output
 * per token-slot.  Same shapes, outputs, errors and workspace size as dg_moe_ffn. */
DG_API int dg_moe_ffn_e4m3(const void* d_x, const float* d_residual, const void* d_wr,
               const void* d_w_gu, const float* d_w_gu_scale, const void* d_w_d,
               const float* d_w_d_scale, const void* d_ws_gu, const float* d_ws_gu_scale,
               const void* d_ws_d, const float* d_ws_d_scale, float* d_y, int32_t* d_ids,
               float* d_weights, float* d_router_logits, int32_t t, int32_t d, int32_t n_experts,
               int32_t top_k, int32_t hidden, int32_t shared_hidden, void* d_workspace,
               size_t workspace_bytes, void* stream);

/* Row-wise e4m3 quantisation (the FP8 expert format): for each of `rows` bf16 rows of `cols`
 * values (row pitch ld_in elements) writes `cols` codes (uint8) at a row pitch of ld_codes
 * bytes, zero from cols to ld_codes, and one fp32 scale per row: scale = max|row| / 448 (IEEE
 * division), code = rn_satfinite(x / scale), an all-zero row giving scale 0 and zero codes.
 * Weights for the model and dg_moe_ffn_e4m3 take ld_codes = DG_E4M3_PITCH(cols).
 * cols % 16 == 0, ld_in % 8 == 0, ld_codes % 16 == 0, ld_codes >= cols and 16-byte aligned
 * pointers, else DG_ERR_INVALID_ARG before any launch.  Asynchronous on `stream`. */
DG_API int dg_quantize_e4m3(const void* d_in, int32_t rows, int32_t cols, int64_t ld_in,
                            uint8_t* d_codes, int64_t ld_codes, float* d_scales, void* stream);

/* NVFP4 quantisation of `rows` bf16 rows of `cols` values (row pitch ld_in elements), the
 * 4-bit expert format: per row g = max|row| / 2688 (fp32, IEEE division); per 16 consecutive
 * values s = e4m3_rn_satfinite(max|block| / 6 / g); codes e2m1_rn_satfinite(x / (s * g)), two
 * per byte with the lower column in the low nibble, rows at ld_codes bytes (zero past cols / 2).
 * Block scales go to 512-byte atoms, one per (128-row tile, 64 columns): tile t's atoms start
 * at d_sf + t * 4 * ceil(cols / 256) * 512 (the ones past cols / 64 are zero); inside an atom
 * the scale of tile row r and 16-wide block b is byte (r % 32) * 16 + (r / 32) * 4 + b.
 * d_sf must hold ceil(rows / 128) * 4 * ceil(cols / 256) * 512 bytes.  cols % 64 == 0,
 * ld_codes >= cols / 2 and a multiple of 16, ld_in % 8 == 0, 16-byte aligned pointers, else
 * DG_ERR_INVALID_ARG before any launch.  Asynchronous on `stream`. */
DG_API int dg_quantize_nvfp4(const void* d_in, int32_t rows, int32_t cols, int64_t ld_in,
                             uint8_t* d_codes, int64_t ld_codes, uint8_t* d_sf,
                             float* d_row_scales, void* stream);

/* The MoE with NVFP4 experts: codes, row scales and scale atoms of w_gu, w_d (and ws_gu, ws_d
 * when hs > 0) as dg_quantize_nvfp4 writes them for the stacked matrices.  Shapes as
 * dg_moe_ffn, with d a multiple of 128; workspace size from dg_moe_workspace_bytes. */
DG_API int dg_moe_ffn_nvfp4(const void* d_x, const float* d_residual, const void* d_wr,
               const void* d_w_gu, const float* d_w_gu_scale, const void* d_w_gu_sf,
               const void* d_w_d, const float* d_w_d_scale, const void* d_w_d_sf,
               const void* d_ws_gu, const float* d_ws_gu_scale, const void* d_ws_gu_sf,
               const void* d_ws_d, const float* d_ws_d_scale, const void* d_ws_d_sf, float* d_y,
               int32_t* d_ids, float* d_weights, float* d_router_logits, int32_t t, int32_t d,
               int32_t n_experts, int32_t top_k, int32_t hidden, int32_t shared_hidden,
               void* d_workspace, size_t workspace_bytes, void* stream);

/* ---- tracing ------------------------------------------------------------------------- */

/* Kernels that dg_profile_kernel can time. */
enum {
  DG_KERNEL_EXPERT_GATE_UP = 0, /* grouped expert gate/up GEMM + SiLU-GLU */
  DG_KERNEL_EXPERT_DOWN = 1,    /* grouped expert down GEMM + weighted scatter */
  DG_KERNEL_ATTENTION = 2,      /* canvas attention, split merge included */
  DG_KERNEL_LM_HEAD = 3,        /* LM head fused with vocab-tile statistics */
  DG_KERNEL_QKV = 4,            /* QKV projection (bf16: RoPE and cache writes included) */
  DG_KERNEL_O_PROJ = 5,         /* attention output projection (bf16: residual add included) */
  DG_KERNEL_SAMPLER = 6,        /* sampler merge + stop test */
  DG_KERNEL_SHARED_EXPERT = 7,  /* reserved: the shared expert runs inside kinds 0 and 1 */
  DG_KERNEL_ROUTER = 8,         /* router (bf16: top-k and expert permutation included) */
  DG_KERNEL_QKV_FINALIZE = 9,   /* reserved: RoPE + K/V cache store (inside kind 4 on bf16) */
  DG_KERNEL_ATTN_COMBINE = 10,  /* reserved: split-KV merge (inside kind 2) */
  DG_KERNEL_RESIDUAL_NORM = 11, /* residual add + RMSNorm */
  DG_KERNEL_ROUTER_TOPK = 12,   /* reserved: top-k selection (inside kind 8 on bf16) */
  DG_KERNEL_ROUTE = 13,         /* reserved: expert permutation (inside kind 8 on bf16) */
  DG_KERNEL_GATHER = 14,        /* permuted token rows (e4m3 experts: quantised as well) */
  DG_KERNEL_COMBINE_NORM = 15,  /* weighted expert sum + RMSNorm */
  DG_KERNEL_EMBED = 16,         /* embedding gather + RMSNorm */
  DG_KERNEL_QUANT_H = 17,       /* e4m3 experts: per-row quantisation of the SiLU-GLU output */
  DG_KERNEL_KINDS = 18
};

/* Number of kernels this library has launched in the calling process (all entry points). */
DG_API uint64_t dg_launch_count(void);

/* Time launches of one kernel kind: before/after each of its next n_pairs launches the library
 * records a pair of CUDA events (created here, timing enabled) on the stream the kernel is
 * launched on.  n_pairs = 0 disables the hook and releases the events.  Host-side only, one hook
 * per process. */
DG_API int dg_profile_kernel(int32_t kernel_kind, int32_t n_pairs);
/* Blocking: waits for the recorded pairs and writes their durations (milliseconds) to the host
 * array durations_ms[0..max_pairs).  Returns the number of pairs written (>= 0) or an error. */
DG_API int32_t dg_profile_read(float* durations_ms, int32_t max_pairs);

/* ---- test exports ------------------------------------------------------------------ */

/* Unfused LM head of the context on its current final hidden state: logits fp32 [T, V]
 * from the same MMA core as the fused path (for parity of the statistics). */
DG_API int dg_debug_logits(dg_ctx* ctx, float* d_logits, void* stream);
/* Teacher-forced layer: x_out fp32 [n, d] = layer `layer` applied to the residual stream
 * x_in fp32 [n, d] at positions P..P+n-1 (P = committed length) against that layer's cache.
 * causal != 0 masks causally over the n tokens, 0 attends bidirectionally.  The n tokens'
 * K/V are written to cache slots P..P+n-1 like a denoise step; P does not advance. */
DG_API int dg_debug_layer(dg_ctx* ctx, int32_t layer, const float* d_x_in, float* d_x_out, int32_t n,
                   int32_t causal, void* stream);
/* Routing of the most recent layer the context ran: ids int32 [n, k], weights fp32 [n, k]
 * (renormalised over the k experts), router logits fp32 [n, E] (device pointers into scratch). */
DG_API int dg_debug_routing(const dg_ctx* ctx, int32_t** d_ids, float** d_weights,
                            float** d_router_logits);
/* Half of a teacher-forced layer: part 0 = attention sub-block (x_out = x_in + O-projection of
 * the attention over RMSNorm(x_in), K/V written to slots P..P+n-1), part 1 = MoE sub-block
 * (x_out = x_in + MoE(RMSNorm(x_in)) with the shared expert).  Shapes as dg_debug_layer. */
DG_API int dg_debug_layer_part(dg_ctx* ctx, int32_t layer, int32_t part, const float* d_x_in,
                               float* d_x_out, int32_t n, int32_t causal, void* stream);
/* Intermediate buffers of the most recent layer the context ran (device pointers into scratch):
 * q [Hq, 256, hd] (bf16 model; [Hq, T, hd] fp32 model), attention output o [n, Hq*hd] and the
 * normalised activations xn [n, d] in the storage type. */
DG_API int dg_debug_tensors(const dg_ctx* ctx, void** d_q, void** d_o, void** d_xn);
/* Final hidden state (fp32 [T, d]) of the last denoise step, for LM-head checks. */
DG_API int dg_debug_hidden(const dg_ctx* ctx, float** d_x);

DG_API const char* dg_last_error(void);
DG_API const char* dg_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DG_H_ */
