// layer.cuh -- the non-GEMM kernels of one decoder layer (bandwidth-bound, one pass each).
//
//   embed_norm        x = E[ids] (fp32 residual), xn = rmsnorm(x) * w        (a1, a2)
//   qkv_finalize      (all-fp32 path) sum of partials; rotate-half RoPE at absolute positions
//                     for q and k heads (Q [Hq, Tq, hd], K cache slots P..P+n-1); V stored
//                     transposed into V^T [hd, cap]                            (a3)
//   residual_norm     x += partials (none on the bf16 path, whose O projection adds into x
//                     itself); xn2 = rmsnorm(x) * w                             (a5, a2)
//   router_topk_*     router logits -> top-k ids (lowest index on ties) and the softmax of
//                     the selected logits (= renormalised full-softmax probabilities) (a6)
//   route_canvas      per-expert token bitmasks -> offsets, stable slot order, the token-chunk
//                     list of the grouped GEMMs, the route weights in permuted order (run by
//                     the router kernel's last CTA); the bf16 / e4m3 gate/up GEMM then copies
//                     each routed row's token itself (64-token chunks)                  (a7)
//   gather_rows       x_perm[p] = xn[perm[p] / k] for the wide-chunk passes           (a7)
//   moe_combine_norm  x += sum over slots in order of y_slot + y_shared; xn = rmsnorm(x) * w
//                     for the next layer (or the final norm)                  (a9, a2)
// RMSNorm is x / sqrt(mean(x^2) + eps) * w (pre-norm, the Gemma-style plain reading).
#pragma once
#include "dg_common.cuh"

namespace dg {

// block-wide sum for 256 threads
DG_DEV float block_sum_256(float v, float* sm) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane_id() == 0) sm[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) t += sm[w];
  __syncthreads();
  return t;
}

DG_DEV float block_max_256(float v, float* sm) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane_id() == 0) sm[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = sm[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) t = fmaxf(t, sm[w]);
  __syncthreads();
  return t;
}

template <typename TW, typename TA>
__global__ void __launch_bounds__(256) embed_norm_kernel(const int32_t* __restrict__ ids,
                                                         const TW* __restrict__ embed, int d,
                                                         int vocab,
                                                         const float* __restrict__ w, float eps,
                                                         float* __restrict__ x,
                                                         TA* __restrict__ xn, const int* done,
                                                         int* err) {
  pdl_enter();
  if (block_done(done)) return;
  __shared__ float sm[8];
  const int t = blockIdx.x;
  int id = ids[t];
  if (id < 0 || id >= vocab) {  // never read outside the table: record the error, use row 0
    if (threadIdx.x == 0) atomicExch(err, kDevErrBadId);
    id = 0;
  }
  const TW* e = embed + static_cast<long long>(id) * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += 256) {
    const float v = load_as_f32<TW>(e, i);
    x[static_cast<long long>(t) * d + i] = v;
    ss += v * v;
  }
  const float inv = rsqrtf(block_sum_256(ss, sm) / d + eps);
  for (int i = threadIdx.x; i < d; i += 256)
    xn[static_cast<long long>(t) * d + i] =
        store_from_f32<TA>(x[static_cast<long long>(t) * d + i] * inv * w[i]);
}

// Sum of up to kMaxSplits split-K partials of one float4 column block (independent loads).
constexpr int kMaxSplits = 16;
DG_DEV float4 sum_splits4(const float* part, int splits, long long split_stride, long long off) {
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) {
    if (s < splits) {
      const float4 v = *reinterpret_cast<const float4*>(part + s * split_stride + off);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
  }
  return acc;
}

template <typename TA>
DG_DEV void store4(TA* dst, float4 v);
template <>
DG_DEV void store4<float>(float* dst, float4 v) {
  *reinterpret_cast<float4*>(dst) = v;
}
template <>
DG_DEV void store4<__nv_bfloat16>(__nv_bfloat16* dst, float4 v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  const __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&a);
  u.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(dst) = u;
}

// QKV finalize: sum the split-K partials of 16 tokens for one head and store them.
//  q / k heads: rotate-half RoPE at absolute positions pos0 + t (cos/sin table in fp32 computed
//               in fp64), stored to Q [Hq, tq, hd] or to the K cache slots pos0 + t;
//  v heads:     stored transposed into V^T [hd, cap] at columns pos0 + t.
// grid (ceil(n / 16), Hq + 2 Hkv), 128 threads.  Phase 1 sums the [16, hd] block of every split
// with independent float4 loads into shared memory; phase 2 rotates or transposes from there.
// hd % 4 == 0, hd <= 128.
constexpr int kQkvTok = 16;
template <typename TA>
__global__ void __launch_bounds__(128) qkv_finalize_kernel(
    const float* __restrict__ part, int splits, long long split_stride, int ld, int hd,
    int n_heads, int n_kv_heads, const float2* __restrict__ rope_tab, int n, int pos0,
    TA* __restrict__ q, int tq, TA* __restrict__ k_cache, TA* __restrict__ vt_cache, int ldk,
    const int* done) {
  pdl_enter();
  if (block_done(done)) return;
  __shared__ float blk[kQkvTok][128 + 4];
  const int t0 = blockIdx.x * kQkvTok, h = blockIdx.y, tid = threadIdx.x;
  const int nt = min(kQkvTok, n - t0);
  const int hv = hd >> 2;  // float4 per token row
  for (int e = tid; e < kQkvTok * hv; e += 128) {
    const int tt = e / hv, c4 = e % hv;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tt < nt)
      acc = sum_splits4(part, splits, split_stride,
                        static_cast<long long>(t0 + tt) * ld + h * hd + 4 * c4);
    *reinterpret_cast<float4*>(&blk[tt][4 * c4]) = acc;
  }
  __syncthreads();
  const int half = hd >> 1;
  if (h < n_heads + n_kv_heads) {
    for (int e = tid; e < nt * half; e += 128) {
      const int tt = e / half, i = e % half;
      const int t = t0 + tt;
      const float a = blk[tt][i], b = blk[tt][i + half];
      const float2 cs = rope_tab[static_cast<long long>(pos0 + t) * half + i];  // (cos, sin)
      TA* dst = (h < n_heads) ? q + (static_cast<long long>(h) * tq + t) * hd
                              : k_cache + (static_cast<long long>(h - n_heads) * ldk + pos0 + t) * hd;
      dst[i] = store_from_f32<TA>(a * cs.x - b * cs.y);
      dst[i + half] = store_from_f32<TA>(b * cs.x + a * cs.y);
    }
  } else {
    const int g = h - n_heads - n_kv_heads;
    for (int dd = tid; dd < hd; dd += 128) {
      TA* dst = vt_cache + (static_cast<long long>(g) * hd + dd) * ldk + pos0 + t0;
      for (int tt = 0; tt < nt; ++tt) dst[tt] = store_from_f32<TA>(blk[tt][dd]);
    }
  }
}

// x += sum of split partials (0 splits: x unchanged); xn = rmsnorm(x) * w.  One CTA per token,
// float4 columns, d % 4 == 0 and d <= 4 * 256 * kNormVec.
constexpr int kNormVec = 4;
template <typename TA, bool kQ8 = false>
__global__ void __launch_bounds__(256) residual_norm_kernel(float* __restrict__ x,
                                                            const float* __restrict__ part,
                                                            int splits, long long split_stride,
                                                            int d, const float* __restrict__ w,
                                                            float eps, TA* __restrict__ xn,
                                                            uint8_t* __restrict__ q_codes,
                                                            int q_pitch, float* __restrict__ q_scale,
                                                            const int* done) {
  pdl_enter();
  if (block_done(done)) return;
  __shared__ float sm[8];
  const int t = blockIdx.x;
  const int nv = d >> 2;
  float* xr = x + static_cast<long long>(t) * d;
  float4 v[kNormVec];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < kNormVec; ++j) {
    const int i = threadIdx.x + j * 256;
    if (i < nv) {
      float4 a = reinterpret_cast<const float4*>(xr)[i];
      const float4 p = sum_splits4(part, splits, split_stride, static_cast<long long>(t) * d + 4 * i);
      a.x += p.x;
      a.y += p.y;
      a.z += p.z;
      a.w += p.w;
      v[j] = a;
      if (splits > 0) reinterpret_cast<float4*>(xr)[i] = a;
      ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
    }
  }
  const float inv = rsqrtf(block_sum_256(ss, sm) / d + eps);
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < kNormVec; ++j) {
    const int i = threadIdx.x + j * 256;
    if (i < nv) {
      const float4 g = reinterpret_cast<const float4*>(w)[i];
      float4 y = make_float4(v[j].x * inv * g.x, v[j].y * inv * g.y, v[j].z * inv * g.z,
                             v[j].w * inv * g.w);
      store4<TA>(xn + static_cast<long long>(t) * d + 4 * i, y);
      if constexpr (kQ8) {  // the stored (bf16-rounded) values are the ones quantised
        y = make_float4(__bfloat162float(__float2bfloat16_rn(y.x)),
                        __bfloat162float(__float2bfloat16_rn(y.y)),
                        __bfloat162float(__float2bfloat16_rn(y.z)),
                        __bfloat162float(__float2bfloat16_rn(y.w)));
        amax = fmaxf(fmaxf(amax, fmaxf(fabsf(y.x), fabsf(y.y))), fmaxf(fabsf(y.z), fabsf(y.w)));
      }
      v[j] = y;
    }
  }
  if constexpr (!kQ8) return;
  // e4m3 codes of the row as quant_rows_kernel makes them: scale = max|row| / 448 (IEEE division),
  // codes = e4m3_rn_satfinite(x / scale), all zero for a zero row; the row's pitch padding zero
  const float sc = __fdiv_rn(block_max_256(amax, sm), kE4m3Max);
  if (threadIdx.x == 0) q_scale[t] = sc;
  uint8_t* qr = q_codes + static_cast<long long>(t) * q_pitch;
#pragma unroll
  for (int j = 0; j < kNormVec; ++j) {
    const int i = threadIdx.x + j * 256;
    if (i < nv) {
      const uint32_t c =
          sc > 0.f ? e4m3x2(__fdiv_rn(v[j].x, sc), __fdiv_rn(v[j].y, sc)) |
                         (e4m3x2(__fdiv_rn(v[j].z, sc), __fdiv_rn(v[j].w, sc)) << 16)
                   : 0u;
      reinterpret_cast<uint32_t*>(qr)[i] = c;
    }
  }
  for (int i = nv + threadIdx.x; i < (q_pitch >> 2); i += 256) reinterpret_cast<uint32_t*>(qr)[i] = 0u;
}

// Top-k of one token's router logits held by one warp; E <= 256 and E % 4 == 0, k <= 8.  Lane
// l holds experts 4l..4l+3 in v[0..3] and 128+4l..128+4l+3 in v[4..7] (-inf where e >= E).
// Top-k by repeated warp argmax (largest logit, lowest index on ties); the weights are the
// softmax of the selected logits.  Lane 0 writes ids_t[0..k) and wts_t[0..k).
DG_DEV void router_topk_select(float (&v)[8], int n_experts, int top_k, int32_t* ids_t,
                               float* wts_t) {
  const int lane = lane_id();
  // a NaN logit ranks as -inf, so every selection below names a valid expert (top_k <= E)
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (v[j] != v[j]) v[j] = -INFINITY;
  float sel_v[8];
  int sel_i[8];
  for (int kk = 0; kk < top_k; ++kk) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = 128 * (j >> 2) + 4 * lane + (j & 3);
      if (e < n_experts && (v[j] > bv || (v[j] == bv && e < bi))) {
        bv = v[j];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    sel_v[kk] = bv;
    sel_i[kk] = bi;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (128 * (j >> 2) + 4 * lane + (j & 3) == bi) v[j] = -INFINITY;
  }
  if (lane == 0) {
    float den = 0.f;
    for (int kk = 0; kk < top_k; ++kk) den += expf(sel_v[kk] - sel_v[0]);
    for (int kk = 0; kk < top_k; ++kk) {
      ids_t[kk] = sel_i[kk];
      wts_t[kk] = expf(sel_v[kk] - sel_v[0]) / den;
    }
  }
}

// Top-k of token t from split-K partials of its router logits (summed in split order).
DG_DEV void router_topk_token(const float* __restrict__ part, int splits, long long split_stride,
                              int t, int n_experts, int top_k, float* __restrict__ logits_out,
                              int32_t* __restrict__ ids, float* __restrict__ wts) {
  const int lane = lane_id();
  float v[8];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int e0 = 128 * h + 4 * lane;
    float4 a = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    if (e0 < n_experts) {
      a = sum_splits4(part, splits, split_stride, static_cast<long long>(t) * n_experts + e0);
      if (logits_out)
        *reinterpret_cast<float4*>(logits_out + static_cast<long long>(t) * n_experts + e0) = a;
    }
    v[4 * h] = a.x;
    v[4 * h + 1] = a.y;
    v[4 * h + 2] = a.z;
    v[4 * h + 3] = a.w;
  }
  router_topk_select(v, n_experts, top_k, ids + static_cast<long long>(t) * top_k,
                     wts + static_cast<long long>(t) * top_k);
}

// One warp per token (the all-fp32 path, which needs no permutation).
__global__ void router_topk_kernel(const float* __restrict__ part, int splits,
                                   long long split_stride, int n_tokens, int n_experts, int top_k,
                                   float* __restrict__ logits_out, int32_t* __restrict__ ids,
                                   float* __restrict__ wts, const int* done) {
  pdl_enter();
  if (block_done(done)) return;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n_tokens) return;
  router_topk_token(part, splits, split_stride, t, n_experts, top_k, logits_out, ids, wts);
}

struct RouteArgs {
  const int32_t* ids;  // [n_tokens * top_k] expert of slot (token * k + j)
  int n_tokens, top_k, n_experts;
  int n_chunk;         // tokens per grouped-GEMM chunk
  int32_t* offsets;    // [E + 1] first permuted row of each expert
  int32_t* perm;       // [n_slots] permuted row -> slot
  int4* chunks;        // [max chunks] (expert, first permuted row, tokens, 0) in expert order
  int32_t* n_chunks;   // [1] chunks in use
  const float* wts;    // optional: route weights by slot, written to w_perm by permuted row
  float* w_perm;
};

constexpr int kRouteMaxTokens = 4096;
// Shared memory the routing needs (ints) for E experts and n tokens.
__host__ __device__ constexpr int route_smem_ints(int n_experts, int n_tokens) {
  return 2 * n_experts * ((n_tokens + 31) / 32) + 4 * (n_experts + 1);
}

// Exclusive scan of up to 256 values by one warp (8 per lane); returns the total to all lanes.
DG_DEV int warp_exclusive_scan_256(const int* in, int* out, int n) {
  const int lane = lane_id();
  int v[8], s = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane * 8 + j;
    v[j] = e < n ? in[e] : 0;
    s += v[j];
  }
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int run = incl - s;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane * 8 + j;
    if (e < n) out[e] = run;
    run += v[j];
  }
  return __shfl_sync(0xffffffffu, incl, 31);
}

// Expert permutation of the canvas by one CTA (any multiple of 32 threads), from the top-k ids
// (read through L2: other CTAs wrote them).  A token picks an expert at most once, so with
// mask[e] the bit set of tokens that picked e, the rank of slot (t, j) inside its expert is the
// number of earlier tokens in mask[e]: prefix[e][t / 32] + popc(mask[e][t / 32] below bit t % 32).
// perm[offsets[e] + rank] = slot keeps slot order inside each expert; every expert's rows are
// then cut into chunks of n_chunk tokens (the grouped GEMMs' token tiles).  sm holds
// route_smem_ints(E, n_tokens) ints; E <= 256, n_tokens <= kRouteMaxTokens.
DG_DEV void route_canvas(const RouteArgs& a, int* sm) {
  const int E = a.n_experts, words = (a.n_tokens + 31) >> 5, n_slots = a.n_tokens * a.top_k;
  const int tid = threadIdx.x, nth = blockDim.x;
  uint32_t* mask = reinterpret_cast<uint32_t*>(sm);  // [E][words]
  int* prefix = sm + E * words;                      // [E][words]
  int* count_s = prefix + E * words;                 // [E + 1]
  int* off_s = count_s + (E + 1);
  int* nch_s = off_s + (E + 1);
  int* cbase_s = nch_s + (E + 1);
  for (int i = tid; i < E * words; i += nth) mask[i] = 0u;
  __syncthreads();
  // the ids are read in batches of kIdBatch per thread, all loads issued before their use
  constexpr int kIdBatch = 8;
  for (int s0 = 0; s0 < n_slots; s0 += nth * kIdBatch) {
    int e[kIdBatch];
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const int s = s0 + b * nth + tid;
      e[b] = s < n_slots ? __ldcg(a.ids + s) : -1;
    }
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const int t = (s0 + b * nth + tid) / a.top_k;
      if (e[b] >= 0) atomicOr(&mask[e[b] * words + (t >> 5)], 1u << (t & 31));
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += nth) {
    int run = 0;
    for (int w = 0; w < words; ++w) {
      prefix[e * words + w] = run;
      run += __popc(mask[e * words + w]);
    }
    count_s[e] = run;
    nch_s[e] = (run + a.n_chunk - 1) / a.n_chunk;
  }
  __syncthreads();
  if (tid < 32) {
    const int total = warp_exclusive_scan_256(count_s, off_s, E);
    const int chunks = warp_exclusive_scan_256(nch_s, cbase_s, E);
    if (tid == 0) {
      off_s[E] = total;
      *a.n_chunks = chunks;
    }
  }
  __syncthreads();
  for (int e = tid; e <= E; e += nth) a.offsets[e] = off_s[e];
  for (int s0 = 0; s0 < n_slots; s0 += nth * kIdBatch) {
    int e[kIdBatch];
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const int s = s0 + b * nth + tid;
      e[b] = s < n_slots ? __ldcg(a.ids + s) : -1;
    }
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const int s = s0 + b * nth + tid, t = s / a.top_k, w = t >> 5;
      if (e[b] >= 0) {
        const int rank = prefix[e[b] * words + w] +
                         __popc(mask[e[b] * words + w] & ((1u << (t & 31)) - 1u));
        a.perm[off_s[e[b]] + rank] = s;
        if (a.w_perm) a.w_perm[off_s[e[b]] + rank] = __ldcg(a.wts + s);
      }
    }
  }
  for (int e = tid; e < E; e += nth)
    for (int c = 0; c < nch_s[e]; ++c)
      a.chunks[cbase_s[e] + c] = make_int4(e, off_s[e] + c * a.n_chunk,
                                           min(a.n_chunk, count_s[e] - c * a.n_chunk), 0);
}

// Weights of the first routed chunks' experts, prefetched into L2 by the NVFP4 quantiser of the
// routed rows (the grouped GEMM reads them first): chunk c < n_first of the chunk list,
// `expert_bytes` per expert at w.
struct ExpertPrefetch {
  const int4* chunks;
  const int* n_chunks;
  int n_first;
  const void* w;
  long long expert_bytes;
};

// x_perm[p] = xn[perm[p] / k]: the routed rows in permuted order for the passes whose grouped
// GEMM reads them by TMA boxes (wide token chunks); 64 threads per row, 4 rows per CTA, 16-byte
// copies.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __nv_bfloat16* __restrict__ xn,
                                                          const int32_t* __restrict__ perm,
                                                          int top_k, int d, int n_rows,
                                                          __nv_bfloat16* __restrict__ x_perm,
                                                          const int* done) {
  pdl_enter();
  if (block_done(done)) return;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 6);
  if (row >= n_rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(xn + static_cast<long long>(perm[row] / top_k) * d);
  uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<long long>(row) * d);
  for (int i = threadIdx.x & 63; i < d / 8; i += 64) dst[i] = src[i];
}

// x += sum over slots s = 0..k-1 (in order) of y_slot[t*k + s] + y_shared[t]; then, when w is
// given, xn = rmsnorm(x) * w for the next layer (or the final norm).  One CTA per token.
template <typename TA>
__global__ void __launch_bounds__(256) moe_combine_norm_kernel(
    float* __restrict__ x, const float* __restrict__ y_slot, int top_k,
    const float* __restrict__ y_shared, int d, const float* __restrict__ w, float eps,
    TA* __restrict__ xn, const int* done) {
  pdl_enter();
  if (block_done(done)) return;
  __shared__ float sm[8];
  const int t = blockIdx.x;
  const int nv = d >> 2;
  float* xr = x + static_cast<long long>(t) * d;
  float4 v[kNormVec];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < kNormVec; ++j) {
    const int i = threadIdx.x + j * 256;
    if (i < nv) {
      float4 y[8];
#pragma unroll
      for (int s = 0; s < 8; ++s)
        if (s < top_k)
          y[s] = reinterpret_cast<const float4*>(
              y_slot + (static_cast<long long>(t) * top_k + s) * d)[i];
      float4 a = reinterpret_cast<const float4*>(xr)[i];
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int s = 0; s < 8; ++s)
        if (s < top_k) {
          acc.x += y[s].x;
          acc.y += y[s].y;
          acc.z += y[s].z;
          acc.w += y[s].w;
        }
      if (y_shared) {
        const float4 b = reinterpret_cast<const float4*>(y_shared + static_cast<long long>(t) * d)[i];
        acc.x += b.x;
        acc.y += b.y;
        acc.z += b.z;
        acc.w += b.w;
      }
      a.x += acc.x;
      a.y += acc.y;
      a.z += acc.z;
      a.w += acc.w;
      v[j] = a;
      reinterpret_cast<float4*>(xr)[i] = a;
      ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
    }
  }
  if (w == nullptr) return;  // standalone MoE: no following norm
  const float inv = rsqrtf(block_sum_256(ss, sm) / d + eps);
#pragma unroll
  for (int j = 0; j < kNormVec; ++j) {
    const int i = threadIdx.x + j * 256;
    if (i < nv) {
      const float4 g = reinterpret_cast<const float4*>(w)[i];
      store4<TA>(xn + static_cast<long long>(t) * d + 4 * i,
                 make_float4(v[j].x * inv * g.x, v[j].y * inv * g.y, v[j].z * inv * g.z,
                             v[j].w * inv * g.w));
    }
  }
}

// RoPE table: (cos, sin) of pos * theta^(-2i/hd) for pos < n_pos, i < hd/2, computed in fp64.
__global__ void rope_table_kernel(float2* tab, int n_pos, int half, double theta) {
  pdl_enter();
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(n_pos) * half) return;
  const int pos = static_cast<int>(idx / half), i = static_cast<int>(idx % half);
  const double ang = pos * pow(theta, -2.0 * i / (2.0 * half));
  tab[idx] = make_float2(static_cast<float>(cos(ang)), static_cast<float>(sin(ang)));
}

}  // namespace dg
