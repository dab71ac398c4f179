// attention.cuh -- canvas attention on tcgen05.
//
// O = softmax(Q K^T * scale) V per query head, grouped-query (head j reads kv head
// j / (Hq/Hkv)), over the committed history plus the canvas ([uniform]: no mask while
// denoising; [arch]: causal over the new tokens when a block or the prompt is encoded).
//
// One CTA per (128-row query tile, kv head, key split).  The query tile packs rows of the
// group's heads (row = head * Tq + token), so every K/V tile is used by all of them.
// Roles: warp 0 TMA (Q once, then K and V^T tiles of 128 keys through a 2-deep ring),
// warp 1 UMMA (S = Q K^T into one of two TMEM buffers, then O += P V), warps 2-5 softmax
// (one query row per thread, exp2 with the scale folded in, P written to shared memory in
// the UMMA's 128-byte swizzled K-major layout).  O lives in TMEM for the whole key range;
// its running maximum is only moved (and O rescaled) when a new tile raises the row max by
// more than 2^8, otherwise exponents relative to the stale maximum stay below 256.
// Each split writes its unnormalised O, its max and its denominator; a combine kernel merges
// splits exactly.  V is read from a transposed copy (V^T [hd, keys]) so that both UMMA
// operands of P V are K-major.
#pragma once
#include "dg_common.cuh"

namespace dg {

struct AttnParams {
  int group;          // Hq / Hkv
  int tq;             // query rows per head in the Q buffer (multiple of 128)
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
  float* o_part;      // [splits, Hq, tq, 128]
  float2* ml_part;    // [splits, Hq, tq] (max in log2 units, denominator)
  int* err;
  const int* done;
};

constexpr int kAttnTile = 16384;  // one 128-row x 128-byte swizzled slab
// Q (2 slabs) + K,V^T ring (2 stages x 4 slabs) + P (2 buffers x 2 slabs) + barriers
constexpr int kAttnSmemBytes = 14 * kAttnTile + 1024 + 256;

__global__ void __launch_bounds__(192, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_vt, const AttnParams p) {
  if (block_done(p.done)) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* s_q = smem;                   // slabs: hd 0-63, hd 64-127
  uint8_t* s_kv = smem + 2 * kAttnTile;  // stage s: K (2 slabs) then V^T (2 slabs)
  uint8_t* s_p = s_kv + 8 * kAttnTile;   // buffer b: 2 slabs (keys 0-63, 64-127)
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_p + 4 * kAttnTile);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;   // [2] per K/V stage
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2] per S buffer
  uint64_t* p_full = bars + 7;    // [2] per P buffer
  uint64_t* pv_done = bars + 9;   // [2] per P buffer (P V of that buffer completed)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 11);

  const int warp = threadIdx.x >> 5;
  const int mt = blockIdx.x;  // query tile inside the kv group
  const int g = blockIdx.y;   // kv head
  const int split = blockIdx.z;
  const int head = g * p.group + (mt * 128) / p.tq;
  const int tok0 = (mt * 128) % p.tq;
  const int n_kv_tiles = (p.n_keys + 127) >> 7;
  int tile_end = n_kv_tiles;
  if (p.causal_prefix >= 0) tile_end = min(tile_end, (p.causal_prefix + tok0 + 127) / 128 + 1);
  const int tile0 = split * p.tiles_per_split;
  const int n_tiles = max(0, min(tile0 + p.tiles_per_split, tile_end) - tile0);

  if (warp == 0 && lane_id() == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
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
  const uint32_t tmem_base = *tmem_holder;  // cols [0,128): O, [128,256) S0, [256,384) S1

  if (warp == 0) {
    if (elect_one() && n_tiles > 0) {
      const uint64_t pol = policy_evict_last();
      const int q_row = p.q_row_base + head * p.tq + tok0;
      mbar_arrive_expect_tx(q_full, 2 * kAttnTile);
      tma_load_2d(&tm_q, q_full, s_q, 0, q_row, pol);
      tma_load_2d(&tm_q, q_full, s_q + kAttnTile, 64, q_row, pol);
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&kv_empty[st], ((j >> 1) & 1) ^ 1u, p.err)) break;
        uint8_t* sk = s_kv + st * 4 * kAttnTile;
        const int key0 = (tile0 + j) * 128;
        const int k_row = static_cast<int>(p.k_row_base + static_cast<long long>(g) * p.ldk + key0);
        const int vt_row = p.vt_row_base + g * 128;
        mbar_arrive_expect_tx(&kv_full[st], 4 * kAttnTile);
        tma_load_2d(&tm_k, &kv_full[st], sk, 0, k_row, pol);
        tma_load_2d(&tm_k, &kv_full[st], sk + kAttnTile, 64, k_row, pol);
        tma_load_2d(&tm_vt, &kv_full[st], sk + 2 * kAttnTile, key0, vt_row, pol);
        tma_load_2d(&tm_vt, &kv_full[st], sk + 3 * kAttnTile, key0 + 64, vt_row, pol);
      }
    }
  } else if (warp == 1) {
    if (elect_one() && n_tiles > 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128);
      const uint32_t a_q = smem_u32(s_q);
      bool ok = mbar_wait(q_full, 0, p.err);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&kv_full[st], (j >> 1) & 1, p.err)) return false;
        tc_fence_after();
        const uint32_t a_k = smem_u32(s_kv + st * 4 * kAttnTile);
        const uint32_t d = tmem_base + 128 + st * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * kAttnTile;
          umma_bf16(d, sdesc_sw128(a_q + off) + 2 * (k & 3), sdesc_sw128(a_k + off) + 2 * (k & 3),
                    idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[st]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n_tiles && ok; ++j) {
        // S of the next tile overlaps the softmax of this one
        if (j + 1 < n_tiles && !issue_s(j + 1)) break;
        const int b = j & 1;
        if (!mbar_wait(&p_full[b], (j >> 1) & 1, p.err)) break;
        tc_fence_after();
        const uint32_t a_p = smem_u32(s_p + b * 2 * kAttnTile);
        const uint32_t a_v = smem_u32(s_kv + b * 4 * kAttnTile + 2 * kAttnTile);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * kAttnTile;
          umma_bf16(tmem_base, sdesc_sw128(a_p + off) + 2 * (k & 3),
                    sdesc_sw128(a_v + off) + 2 * (k & 3), idesc, (j > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&pv_done[b]);
        umma_commit(&kv_empty[b]);
      }
    }
  } else {
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane_id();
    const int tok = tok0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const int key_lim =
        p.causal_prefix >= 0 ? min(p.n_keys, p.causal_prefix + tok + 1) : p.n_keys;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles && ok; ++j) {
      const int st = j & 1;
      if (!mbar_wait(&s_full[st], (j >> 1) & 1, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int key0 = (tile0 + j) * 128;
      const uint32_t s_addr = tmem_base + 128 + st * 128 + lane_off;
      // pass 1: row maximum of this tile (scaled, log2 units)
      float m_tile = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(s_addr + c * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (key0 + c * 32 + i < key_lim) m_tile = fmaxf(m_tile, v[i] * p.scale_log2);
      }
      // move the reference maximum only when it grows by more than 8 (factor 256)
      float alpha = 1.0f;
      bool rescale = false;
      if (m_tile > m_run + 8.0f || (m_run == -INFINITY && m_tile > -INFINITY)) {
        if (m_run != -INFINITY) {
          alpha = exp2f(m_run - m_tile);
          rescale = true;
        }
        m_run = m_tile;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // O must hold every earlier P V before it is rescaled
        if (j > 0 && !mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(tmem_base + lane_off + c * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= alpha;
          tmem_st32(tmem_base + lane_off + c * 32, v);
        }
      }
      // the P buffer of this tile was last read by P V of tile j - 2
      const int b = j & 1;
      if (j >= 2 && !mbar_wait(&pv_done[b], ((j - 2) >> 1) & 1, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // pass 2: probabilities (bf16) into the swizzled K-major layout: slab key / 64; the
      // 16-byte unit u of row r's 128-byte line lands at unit u ^ (r % 8)
      uint8_t* pb = s_p + b * 2 * kAttnTile + (r >> 3) * 1024 + (r & 7) * 128;
      float rowsum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(s_addr + c * 32, v);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int k0 = key0 + c * 32 + 2 * i;
          const float e0 = (k0 < key_lim) ? exp2f(v[2 * i] * p.scale_log2 - m_run) : 0.f;
          const float e1 = (k0 + 1 < key_lim) ? exp2f(v[2 * i + 1] * p.scale_log2 - m_run) : 0.f;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(e0, e1);
          // the denominator sums exactly the probabilities P V uses
          rowsum += __low2float(h2) + __high2float(h2);
          pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int unit = c * 4 + q;  // 16-byte unit of the 256-byte row (0..15)
          const int slab = unit >> 3, u = unit & 7;
          *reinterpret_cast<uint4*>(pb + slab * kAttnTile + ((u ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      l_run = l_run * alpha + rowsum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    const long long row = (static_cast<long long>(split) * p.n_heads + head) * p.tq + tok;
    float4* dst = reinterpret_cast<float4*>(p.o_part + row * 128);
    const bool have_o = ok && n_tiles > 0 &&
                        mbar_wait(&pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, p.err);
    if (have_o) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(tmem_base + lane_off + c * 32, v);
        if (tok < p.n_queries) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[c * 8 + i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
    } else if (tok < p.n_queries) {
      for (int i = 0; i < 32; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      m_run = -INFINITY;
      l_run = 0.f;
    }
    if (tok < p.n_queries) p.ml_part[row] = make_float2(m_run, l_run);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// Merge the key splits: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, stored bf16 into
// o [T, Hq * 128] (token-major, ready to be the O-projection's token operand).
template <typename TA>
__global__ void attn_combine_kernel(const float* __restrict__ o_part,
                                    const float2* __restrict__ ml_part, int n_splits, int n_heads,
                                    int tq, int n_queries, TA* __restrict__ o, const int* done) {
  if (block_done(done)) return;
  const int tok = blockIdx.x, head = blockIdx.y, d = threadIdx.x;
  if (tok >= n_queries) return;
  float mmax = -INFINITY;
  for (int s = 0; s < n_splits; ++s)
    mmax = fmaxf(mmax, ml_part[(static_cast<long long>(s) * n_heads + head) * tq + tok].x);
  float num = 0.f, den = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const long long row = (static_cast<long long>(s) * n_heads + head) * tq + tok;
    const float2 ml = ml_part[row];
    if (ml.y == 0.f) continue;
    const float w = exp2f(ml.x - mmax);
    num += w * o_part[row * 128 + d];
    den += w * ml.y;
  }
  o[static_cast<long long>(tok) * n_heads * 128 + head * 128 + d] = store_from_f32<TA>(num / den);
}

}  // namespace dg
