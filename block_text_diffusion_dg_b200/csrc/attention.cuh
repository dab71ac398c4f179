// attention.cuh -- canvas attention on tcgen05.
//
// O = softmax(Q K^T * scale) V per query head, grouped-query (head j reads kv head
// j / (Hq/Hkv)), over the committed history plus the canvas ([uniform]: no mask while
// denoising; [arch]: causal over the new tokens when a block or the prompt is encoded).
//
// One CTA per (128-row query tile, kv head, key split).  The query tile packs rows of the
// group's heads (row = head * Tq + token), so every K/V tile is used by all of them.
// Roles: warp 0 TMA (Q once, then K and V^T tiles of 128 keys through separate 2-deep rings:
// a K slot frees as soon as its S = Q K^T is done, so K runs one tile ahead of V),
// warp 1 UMMA (S = Q K^T into one of two TMEM buffers, then O += P V with P read from TMEM),
// warps 2-9 softmax: two threads per query row, each owning 64 of the tile's 128 keys (the
// partners sit in different warps of the same TMEM lane quarter and trade their partial row
// maxima through a spare TMEM column); exp2 with the scale folded in, P (bf16 pairs) written
// over the first 64 columns of the S buffer it came from (both partners have read their S by
// the exchange barrier, and the next S into that buffer is issued after this tile's P V, the
// UMMAs running in order).  O lives in TMEM for the whole key range;
// its running maximum is only moved (and O rescaled) when a new tile raises the row max by
// more than 2^8, otherwise exponents relative to the stale maximum stay below 256.
// Each split writes its unnormalised O, its max and its denominator; the splits of a query tile
// form a thread-block cluster and merge their rows exactly after a cluster barrier.  V is read from a transposed copy (V^T [hd, keys]) so that both UMMA
// operands of P V are K-major.
#pragma once
#include "dg_common.cuh"

namespace dg {

struct AttnParams {
  int group;          // Hq / Hkv
  int tq;             // query rows per head in the Q buffer (multiple of 128)
  int tiles_per_head; // 128-row query tiles per head in use (ceil(n_queries / 128))
  int n_queries;      // valid tokens per head
  int n_keys;         // keys in use
  int causal_prefix;  // < 0: no mask
  float scale_log2;   // softmax scale * log2(e)
  int tiles_per_split;
  int q_row_base;     // tm_q row of head 0, token 0
  long long k_row_base;  // tm_k row of kv head 0, key 0
  int ldk;            // keys per kv head in tm_k rows
  int vt_row_base;    // tm_vt row of kv head 0, dim 0
  int n_heads;
  // Batched canvases: queries come in runs of seq_len tokens (a multiple of 128; 0 = one
  // sequence), run b attending to sequence b's cache, k_seq_rows / vt_seq_rows further down tm_k /
  // tm_vt; key counts, positions and the causal prefix are relative to the run
  int seq_len;
  long long k_seq_rows;
  int vt_seq_rows;
  float* o_part;      // [splits, Hq, tq, 128]
  float2* ml_part;    // [splits, Hq, tq] (max in log2 units, denominator)
  __nv_bfloat16* o;   // [T, Hq * 128] merged output
  // weights the next kernels stream (the shared expert's): prefetched into L2 while the
  // attention, which hardly uses HBM, runs; null for none
  const void* pf0;
  long long pf0_bytes;
  const void* pf1;
  long long pf1_bytes;
  int* err;
  const int* done;
};

constexpr int kAttnTile = 16384;  // one 128-row x 128-byte swizzled slab
// Q (2 slabs) + K,V^T ring (2 stages x 4 slabs) + barriers
constexpr int kAttnSmemBytes = 10 * kAttnTile + 1024 + 256;

constexpr int kAttnThreads = 64 + 32 * 8;

// 2^t for a pair of exponents on the FMA pipe, taking load off the special-function unit (which
// sets the softmax's pace with two softmax warps per scheduler).  t is clamped to >= -125, rounded
// to n with the 1.5 * 2^23 addition (n lands in the low mantissa bits), f = t - n in [-1/2, 1/2],
// 2^f = c0 + c1 f + c2 f^2 + c3 f^3 + c4 f^4, and n is added to the exponent field.  The quartic is
// a least-squares fit of 2^f on [-1/2, 1/2] weighted towards its largest relative errors: at most
// 2.7e-6 relative in this fp32 Horner form, so P's bf16 values almost never differ from those of
// the special-function unit's 2^t.  Valid for t <= 8 (the lazy rescale keeps exponents there);
// -inf gives 2^-125.
DG_DEV float2 exp2_fma_pipe(float2 t) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const float2 tc = make_float2(fmaxf(t.x, -125.0f), fmaxf(t.y, -125.0f));
  const float2 r = __fadd2_rn(tc, make_float2(kRound, kRound));
  const float2 n = __fadd2_rn(r, make_float2(-kRound, -kRound));
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), tc);
  float2 q = __ffma2_rn(make_float2(0.0095701320f, 0.0095701320f), f,
                        make_float2(0.055918001f, 0.055918001f));
  q = __ffma2_rn(q, f, make_float2(0.24024744f, 0.24024744f));
  q = __ffma2_rn(q, f, make_float2(0.69312179f, 0.69312179f));
  q = __ffma2_rn(q, f, make_float2(0.99999928f, 0.99999928f));
  // the bits of r are those of 1.5 * 2^23 plus n, and 1.5 * 2^23 shifted by 23 vanishes mod 2^32
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(r.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(r.y) << 23)));
}
constexpr int kAttnPolyEvery = 3;  // every third pair of a thread's 64 scores takes exp2_fma_pipe
constexpr int kMaxAttnSplits = 8;  // the key splits of a query tile form one cluster

// Merge of the key splits of one (token, head) by one warp: O = sum_s 2^(m_s - M) O_s /
// sum_s 2^(m_s - M) l_s, lane d4 owning dims 4 d4 .. 4 d4 + 3, stored as bf16 into o [T, Hq * 128]
// (token-major, the O projection's token operand).  Lane s < n_splits reads split s's
// (max, denominator); the partials of other CTAs are read through L2.  In two phases, so that a
// warp can have the loads of two rows in flight together.
struct AttnMergeIn {
  float2 ml;                    // lane s < n_splits: split s's (max, denominator)
  float4 v[kMaxAttnSplits];     // split s's 4 dims of this lane
};

DG_DEV void attn_merge_load(const AttnParams& p, int n_splits, int tok, int head, AttnMergeIn& in) {
  const int lane = lane_id();
  in.ml = make_float2(-INFINITY, 0.f);
  if (lane < n_splits)
    in.ml = __ldcg(p.ml_part + (static_cast<long long>(lane) * p.n_heads + head) * p.tq + tok);
#pragma unroll
  for (int s = 0; s < kMaxAttnSplits; ++s)
    if (s < n_splits) {
      const long long row = (static_cast<long long>(s) * p.n_heads + head) * p.tq + tok;
      in.v[s] = __ldcg(reinterpret_cast<const float4*>(p.o_part + row * 128) + lane);
    }
}

DG_DEV void attn_merge_store(const AttnParams& p, int n_splits, int tok, int head,
                             const AttnMergeIn& in) {
  const int lane = lane_id();
  float mmax = in.ml.x;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
  const float w_mine = (lane < n_splits && in.ml.y != 0.f) ? exp2f(in.ml.x - mmax) : 0.f;
  float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
#pragma unroll
  for (int s = 0; s < kMaxAttnSplits; ++s)
    if (s < n_splits) {
      const float w = __shfl_sync(0xffffffffu, w_mine, s);
      const float l = __shfl_sync(0xffffffffu, in.ml.y, s);
      if (w != 0.f) {
        num.x += w * in.v[s].x;
        num.y += w * in.v[s].y;
        num.z += w * in.v[s].z;
        num.w += w * in.v[s].w;
        den += w * l;
      }
    }
  const float inv = 1.0f / den;
  const __nv_bfloat162 lo = __floats2bfloat162_rn(num.x * inv, num.y * inv);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(num.z * inv, num.w * inv);
  *reinterpret_cast<uint2*>(p.o + static_cast<long long>(tok) * p.n_heads * 128 + head * 128 +
                            4 * lane) = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                                   *reinterpret_cast<const uint32_t*>(&hi));
}

__global__ void __launch_bounds__(kAttnThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_vt, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* s_q = smem;                   // slabs: hd 0-63, hd 64-127
  uint8_t* s_k = smem + 2 * kAttnTile;   // K stage s: 2 slabs (hd 0-63, 64-127)
  uint8_t* s_v = s_k + 4 * kAttnTile;    // V^T stage s: 2 slabs (keys 0-63, 64-127)
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_v + 4 * kAttnTile);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;    // [2] per K stage
  uint64_t* k_empty = bars + 3;   // [2] (S = Q K^T of that stage completed)
  uint64_t* v_full = bars + 5;    // [2] per V stage
  uint64_t* v_empty = bars + 7;   // [2] (P V of that stage completed)
  uint64_t* s_full = bars + 9;    // [2] per S buffer
  uint64_t* p_full = bars + 11;   // [2] per S buffer (its P written)
  uint64_t* pv_done = bars + 13;  // [2] per S buffer (P V of its P completed)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 15);

  const int warp = threadIdx.x >> 5;
  const int mt = blockIdx.x;  // query tile inside the kv group
  const int g = blockIdx.y;   // kv head
  const int split = blockIdx.z;
  const int head = g * p.group + mt / p.tiles_per_head;
  const int tok0 = (mt % p.tiles_per_head) * 128;
  // the sequence this query tile belongs to, and the tile's first token within it
  const int seq = p.seq_len > 0 ? tok0 / p.seq_len : 0;
  const int rel0 = tok0 - seq * p.seq_len;
  const int n_kv_tiles = (p.n_keys + 127) >> 7;
  int tile_end = n_kv_tiles;
  if (p.causal_prefix >= 0) tile_end = min(tile_end, (p.causal_prefix + rel0 + 127) / 128 + 1);
  const int tile0 = split * p.tiles_per_split;
  const int n_tiles = max(0, min(tile0 + p.tiles_per_split, tile_end) - tile0);

  if (warp == 0 && lane_id() == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 256);
      mbar_init(&pv_done[s], 1);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_vt);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // TMEM columns: [0,128) O, [128,256) S0, [256,384) S1, [384,390) partner exchange
  const uint32_t tmem_base = *tmem_holder;
  // the setup above overlaps the previous kernel; from here on its results are needed
  pdl_enter();
  if (block_done(p.done)) {  // uniform over the grid: release TMEM and leave
    if (warp == 1) tmem_dealloc(tmem_base, 512);
    return;
  }

  if (warp == 0) {
    if (elect_one() && n_tiles > 0) {
      const uint64_t pol = policy_evict_last();
      const int q_row = p.q_row_base + head * p.tq + tok0;
      mbar_arrive_expect_tx(q_full, 2 * kAttnTile);
      tma_load_2d(&tm_q, q_full, s_q, 0, q_row, pol);
      tma_load_2d(&tm_q, q_full, s_q + kAttnTile, 64, q_row, pol);
      const int vt_row = p.vt_row_base + seq * p.vt_seq_rows + g * 128;
      const long long k_base = p.k_row_base + seq * p.k_seq_rows + static_cast<long long>(g) * p.ldk;
      auto load_k = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&k_empty[st], ((j >> 1) & 1) ^ 1u, p.err)) return false;
        const int key0 = (tile0 + j) * 128;
        const int k_row = static_cast<int>(k_base + key0);
        uint8_t* sk = s_k + st * 2 * kAttnTile;
        mbar_arrive_expect_tx(&k_full[st], 2 * kAttnTile);
        tma_load_2d(&tm_k, &k_full[st], sk, 0, k_row, pol);
        tma_load_2d(&tm_k, &k_full[st], sk + kAttnTile, 64, k_row, pol);
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&v_empty[st], ((j >> 1) & 1) ^ 1u, p.err)) return false;
        const int key0 = (tile0 + j) * 128;
        uint8_t* sv = s_v + st * 2 * kAttnTile;
        mbar_arrive_expect_tx(&v_full[st], 2 * kAttnTile);
        tma_load_2d(&tm_vt, &v_full[st], sv, key0, vt_row, pol);
        tma_load_2d(&tm_vt, &v_full[st], sv + kAttnTile, key0 + 64, vt_row, pol);
        return true;
      };
      // the UMMA needs K of tile j + 1 (for S) before V of tile j (for P V)
      bool ok = load_k(0);
      for (int j = 0; j < n_tiles && ok; ++j) {
        if (j + 1 < n_tiles) ok = load_k(j + 1);
        if (ok) ok = load_v(j);
      }
      // every K / V load is issued: hint the next kernels' weights into L2 behind them
      const int cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
      const int n_cta = gridDim.x * gridDim.y * gridDim.z;
      prefetch_l2_slice(p.pf0, p.pf0_bytes, cta, n_cta);
      prefetch_l2_slice(p.pf1, p.pf1_bytes, cta, n_cta);
    }
  } else if (warp == 1) {
    if (elect_one() && n_tiles > 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128);
      const uint32_t a_q = smem_u32(s_q);
      bool ok = mbar_wait(q_full, 0, p.err);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&k_full[st], (j >> 1) & 1, p.err)) return false;
        tc_fence_after();
        const uint32_t a_k = smem_u32(s_k + st * 2 * kAttnTile);
        const uint32_t d = tmem_base + 128 + st * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * kAttnTile;
          umma_bf16(d, sdesc_sw128(a_q + off) + 2 * (k & 3), sdesc_sw128(a_k + off) + 2 * (k & 3),
                    idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[st]);
        umma_commit(&k_empty[st]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n_tiles && ok; ++j) {
        // S of the next tile overlaps the softmax of this one
        if (j + 1 < n_tiles && !issue_s(j + 1)) break;
        const int b = j & 1;
        if (!mbar_wait(&p_full[b], (j >> 1) & 1, p.err)) break;
        if (!mbar_wait(&v_full[b], (j >> 1) & 1, p.err)) break;
        tc_fence_after();
        const uint32_t a_v = smem_u32(s_v + b * 2 * kAttnTile);
        const uint32_t p_tmem = tmem_base + 128 + b * 128;  // P over the S buffer's first columns
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * kAttnTile;
          umma_bf16_ts(tmem_base, p_tmem + 8 * k, sdesc_sw128(a_v + off) + 2 * (k & 3), idesc,
                       (j > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&pv_done[b]);
        umma_commit(&v_empty[b]);
      }
    }
  } else {
    const int q4 = warp & 3;             // TMEM lane quarter
    const int half = (warp - 2) >> 2;    // keys [64 half, 64 half + 64) of each tile
    const int r = q4 * 32 + lane_id();   // query row of the tile
    const int tok = tok0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t xchg = tmem_base + 384 + lane_off;  // partner exchange columns
    const int bar_id = 1 + q4;                         // the two warps of this lane quarter
    const int key_lim =
        p.causal_prefix >= 0 ? min(p.n_keys, p.causal_prefix + rel0 + r + 1) : p.n_keys;
    // Every thread passes the same named barriers whatever happens (one per tile and one at
    // the end), so a failed wait only turns the remaining work off: `ok` is warp-uniform.
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j & 1;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&s_full[st], (j >> 1) & 1, p.err));
      tc_fence_after();
      const int key0 = (tile0 + j) * 128 + 64 * half;
      const bool full_tile = key0 + 64 <= key_lim;  // none of my 64 keys is masked
      float x[64];
      tmem_ld64(tmem_base + 128 + st * 128 + 64 * half + lane_off, x);
      if (!full_tile) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (key0 + i >= key_lim) x[i] = -INFINITY;
      }
      float mp;
      {  // three-input maxima: 64 -> 22 -> 8 -> 3 -> 1
        float t[22];
#pragma unroll
        for (int i = 0; i < 21; ++i) t[i] = fmax3(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
        t[21] = x[63];
#pragma unroll
        for (int i = 0; i < 7; ++i) t[i] = fmax3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
        t[7] = t[21];
        t[0] = fmax3(t[0], t[1], t[2]);
        t[1] = fmax3(t[3], t[4], t[5]);
        t[2] = fmaxf(t[6], t[7]);
        mp = fmax3(t[0], t[1], t[2]);
      }
      // row maximum of the tile: my half and my partner's (raw scores, scale applied after)
      tmem_st1(xchg + 2 * st + half, mp);
      tc_fence_before();
      named_barrier(bar_id, 64);
      tc_fence_after();
      const float mo = tmem_ld1(xchg + 2 * st + (1 - half));
      if (!ok) continue;
      const float m_tile = fmaxf(mp, mo) * p.scale_log2;  // -inf stays -inf
      // move the reference maximum only when it grows by more than 8 (factor 256); both
      // partners take the same decision from the same values
      float alpha = 1.0f;
      bool rescale = false;
      if (m_tile > m_run + 8.0f || (m_run == -INFINITY && m_tile > -INFINITY)) {
        if (m_run != -INFINITY) {
          alpha = fast_exp2(m_run - m_tile);
          rescale = true;
        }
        m_run = m_tile;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // O must hold every earlier P V before it is rescaled
        if (j > 0)
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, p.err));
        if (!ok) continue;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float v[32];
          const uint32_t oa = tmem_base + 64 * half + 32 * c + lane_off;
          tmem_ld32(oa, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= alpha;
          tmem_st32(oa, v);
        }
      }
      const int b = j & 1;
      // e = 2^(x scale log2e - m): a masked key holds x = -inf, so e = 0 on the special-function
      // unit and 2^-125 on the FMA pipe (also when the whole tile is masked and m is still -inf, m
      // then taken as 0)
      const float mr = (m_run == -INFINITY) ? 0.f : m_run;
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-mr, -mr);
      float2 part[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        const float2 t = __ffma2_rn(make_float2(x[i], x[i + 1]), sc2, nm2);
        const float2 e = (i / 2) % kAttnPolyEvery == kAttnPolyEvery - 1
                             ? exp2_fma_pipe(t)
                             : make_float2(fast_exp2(t.x), fast_exp2(t.y));
        x[i] = e.x;
        x[i + 1] = e.y;
        part[(i >> 1) & 3] = __fadd2_rn(part[(i >> 1) & 3], e);
      }
      // probabilities (bf16 pairs) of my 64 keys into TMEM columns 32 half .. 32 half + 31 of
      // the S buffer (keys 2c, 2c + 1 of my half in column c)
      {
        float pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(x[2 * c], x[2 * c + 1]);
          pk[c] = __uint_as_float(*reinterpret_cast<const uint32_t*>(&h2));
        }
        tmem_st32(tmem_base + 128 + b * 128 + 32 * half + lane_off, pk);
      }
      const float2 ps = __fadd2_rn(__fadd2_rn(part[0], part[1]), __fadd2_rn(part[2], part[3]));
      const float rowsum = ps.x + ps.y;
      l_run = l_run * alpha + rowsum;
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    // denominators of the two halves
    tmem_st1(xchg + 4 + half, l_run);
    tc_fence_before();
    named_barrier(bar_id, 64);
    tc_fence_after();
    const float l_tot = l_run + tmem_ld1(xchg + 4 + (1 - half));
    const long long row = (static_cast<long long>(split) * p.n_heads + head) * p.tq + tok;
    const bool have_o =
        __all_sync(0xffffffffu, ok && n_tiles > 0 &&
                                    mbar_wait(&pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1,
                                              p.err));
    // the warp's 32 half rows (256 bytes each) go through shared memory so that every store to
    // o_part writes whole 256-byte half rows.  Staging: the K ring, idle once the last P V is
    // done; warp region (warp - 2) * 8 KB, row i at i * 256, 16-byte unit c at (c ^ (i % 16)).
    uint8_t* stage = s_k + (warp - 2) * 8192;
    const int lane = lane_id();
    if (have_o) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float v[32];
        tmem_ld32(tmem_base + 64 * half + 32 * c + lane_off, v);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(stage + lane * 256 + (((c * 8 + i) ^ (lane & 15)) << 4)) =
              make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
    __syncwarp();
    const int tok_w = tok - lane;  // token of the warp's row 0
    const long long row_w = row - lane;
    for (int i0 = 0; i0 < 32; i0 += 2) {
      const int i = i0 + (lane >> 4), c = lane & 15;
      if (tok_w + i < p.n_queries) {
        const float4 val =
            have_o ? *reinterpret_cast<const float4*>(stage + i * 256 + ((c ^ (i & 15)) << 4))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(p.o_part + (row_w + i) * 128 + 64 * half)[c] = val;
      }
    }
    if (tok < p.n_queries && half == 0)
      p.ml_part[row] = have_o ? make_float2(m_run, l_tot) : make_float2(-INFINITY, 0.f);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
  // the key splits of this query tile are one cluster (dims (1, 1, splits)): once every split's
  // partial rows are written, the CTA of split s merges rows [128 s / S, 128 (s + 1) / S) of
  // the tile.  Every thread of every CTA reaches the barrier.
  __threadfence();
  cluster_sync_all();
  const int n_splits = gridDim.z;
  const int r0 = 128 * split / n_splits, r1 = 128 * (split + 1) / n_splits;
  constexpr int kWarps = kAttnThreads / 32;
  for (int rr = r0 + warp; rr < r1; rr += 2 * kWarps) {  // two rows per warp at a time
    const int rr2 = rr + kWarps;
    const bool a = tok0 + rr < p.n_queries, b = rr2 < r1 && tok0 + rr2 < p.n_queries;
    AttnMergeIn in_a, in_b;
    if (a) attn_merge_load(p, n_splits, tok0 + rr, head, in_a);
    if (b) attn_merge_load(p, n_splits, tok0 + rr2, head, in_b);
    if (a) attn_merge_store(p, n_splits, tok0 + rr, head, in_a);
    if (b) attn_merge_store(p, n_splits, tok0 + rr2, head, in_b);
  }
}

}  // namespace dg
