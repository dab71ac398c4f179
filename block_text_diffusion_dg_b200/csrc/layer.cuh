// layer.cuh -- the non-GEMM kernels of one decoder layer (bandwidth-bound, one pass each).
//
//   embed_norm        x = E[ids] (fp32 residual), xn = rmsnorm(x) * w        (a1, a2)
//   rope_qk           sum split-K partials, rotate-half RoPE at absolute positions, store
//                     Q [Hq, Tq, hd] and K into the cache slots P..P+n-1       (a3)
//   v_store           sum partials, store V transposed into V^T [hd, cap]      (a3)
//   residual_norm     x += O-projection partials; xn2 = rmsnorm(x) * w         (a5, a2)
//   router_topk       router logits -> top-k ids (lowest index on ties) and the softmax of
//                     the selected logits (= renormalised full-softmax probabilities) (a6)
//   moe_route         per-expert counts, offsets, stable slot order, grouped GEMM item lists (a7)
//   gather_rows       x_perm[p] = xn2[token of slot perm[p]]                   (a7)
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

template <typename TW, typename TA>
__global__ void __launch_bounds__(256) embed_norm_kernel(const int32_t* __restrict__ ids,
                                                         const TW* __restrict__ embed, int d,
                                                         const float* __restrict__ w, float eps,
                                                         float* __restrict__ x,
                                                         TA* __restrict__ xn, const int* done) {
  if (block_done(done)) return;
  __shared__ float sm[8];
  const int t = blockIdx.x;
  const TW* e = embed + static_cast<long long>(ids[t]) * d;
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

// grid (n tokens, Hq + Hkv); threads = hd / 2; thread i rotates dims (i, i + hd/2).
template <typename TA>
__global__ void rope_qk_kernel(const float* __restrict__ part, int splits, long long split_stride,
                               int ld, int hd, int n_heads, const float2* __restrict__ rope_tab,
                               int pos0, TA* __restrict__ q, int tq, TA* __restrict__ k_cache,
                               int ldk, const int* done) {
  if (block_done(done)) return;
  const int t = blockIdx.x, h = blockIdx.y, i = threadIdx.x, half = hd >> 1;
  const int col = h * hd + i;
  float a = 0.f, b = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float* src = part + s * split_stride + static_cast<long long>(t) * ld + col;
    a += src[0];
    b += src[half];
  }
  const float2 cs = rope_tab[static_cast<long long>(pos0 + t) * half + i];  // (cos, sin)
  const float ra = a * cs.x - b * cs.y;
  const float rb = b * cs.x + a * cs.y;
  TA* dst;
  if (h < n_heads) {
    dst = q + (static_cast<long long>(h) * tq + t) * hd;
  } else {
    dst = k_cache + (static_cast<long long>(h - n_heads) * ldk + pos0 + t) * hd;
  }
  dst[i] = store_from_f32<TA>(ra);
  dst[i + half] = store_from_f32<TA>(rb);
}

// V heads: transpose [token, dim] partial sums into V^T [hd, cap] at columns pos0 + t.
// grid (ceil(n / 32), Hkv); block (32, 8).
template <typename TA>
__global__ void v_store_kernel(const float* __restrict__ part, int splits, long long split_stride,
                               int ld, int hd, int v_col0, int n, int pos0,
                               TA* __restrict__ vt_cache, int ldk, const int* done) {
  if (block_done(done)) return;
  __shared__ float tile[128][33];
  const int t0 = blockIdx.x * 32, g = blockIdx.y;
  for (int tt = threadIdx.y; tt < 32; tt += 8) {
    const int t = t0 + tt;
    for (int dd = threadIdx.x; dd < hd; dd += 32) {
      float v = 0.f;
      if (t < n)
        for (int s = 0; s < splits; ++s)
          v += part[s * split_stride + static_cast<long long>(t) * ld + v_col0 + g * hd + dd];
      tile[dd][tt] = v;
    }
  }
  __syncthreads();
  const int t = t0 + threadIdx.x;
  if (t < n)
    for (int dd = threadIdx.y; dd < hd; dd += 8)
      vt_cache[(static_cast<long long>(g) * hd + dd) * ldk + pos0 + t] =
          store_from_f32<TA>(tile[dd][threadIdx.x]);
}

template <typename TA>
__global__ void __launch_bounds__(256) residual_norm_kernel(float* __restrict__ x,
                                                            const float* __restrict__ part,
                                                            int splits, long long split_stride,
                                                            int d, const float* __restrict__ w,
                                                            float eps, TA* __restrict__ xn,
                                                            const int* done) {
  if (block_done(done)) return;
  __shared__ float sm[8];
  const int t = blockIdx.x;
  float* xr = x + static_cast<long long>(t) * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += 256) {
    float v = xr[i];
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc += part[s * split_stride + static_cast<long long>(t) * d + i];
    v += acc;
    xr[i] = v;
    ss += v * v;
  }
  const float inv = rsqrtf(block_sum_256(ss, sm) / d + eps);
  for (int i = threadIdx.x; i < d; i += 256)
    xn[static_cast<long long>(t) * d + i] = store_from_f32<TA>(xr[i] * inv * w[i]);
}

// one warp per token; E <= 256, k <= 8.
__global__ void router_topk_kernel(const float* __restrict__ part, int splits,
                                   long long split_stride, int n_tokens, int n_experts, int top_k,
                                   float* __restrict__ logits_out, int32_t* __restrict__ ids,
                                   float* __restrict__ wts, const int* done) {
  if (block_done(done)) return;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n_tokens) return;
  const int lane = lane_id();
  float v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    float acc = -INFINITY;
    if (e < n_experts) {
      acc = 0.f;
      for (int s = 0; s < splits; ++s)
        acc += part[s * split_stride + static_cast<long long>(t) * n_experts + e];
      if (logits_out) logits_out[static_cast<long long>(t) * n_experts + e] = acc;
    }
    v[j] = acc;
  }
  float sel_v[8];
  int sel_i[8];
  for (int kk = 0; kk < top_k; ++kk) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
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
      if (lane + 32 * j == bi) v[j] = -INFINITY;
  }
  if (lane == 0) {
    float den = 0.f;
    for (int kk = 0; kk < top_k; ++kk) den += expf(sel_v[kk] - sel_v[0]);
    for (int kk = 0; kk < top_k; ++kk) {
      ids[t * top_k + kk] = sel_i[kk];
      wts[t * top_k + kk] = expf(sel_v[kk] - sel_v[0]) / den;
    }
  }
}

struct RouteArgs {
  const int32_t* ids;  // [n_slots] expert of slot (token * k + s)
  int n_slots, n_experts;
  int32_t* offsets;  // [E + 1]
  int32_t* perm;     // [n_slots] permuted row -> slot
  int4* items_gu;    // grouped items for gate/up
  int4* items_d;     // grouped items for down
  int32_t* counts;   // [2]: item counts (gate/up, down)
  int m_tiles_gu, m_tiles_d, n_chunk;
  const int* done;
};

// Single CTA of 1024 threads: counts, exclusive scan, stable (slot-order) placement via
// warp match + per-warp counts, and the grouped item lists.
__global__ void __launch_bounds__(1024) moe_route_kernel(RouteArgs a) {
  if (block_done(a.done)) return;
  __shared__ int cnt[32][257];  // per-warp counts in the current round, per expert
  __shared__ int off_s[257];
  __shared__ int base_s[256];
  const int tid = threadIdx.x, warp = tid >> 5, lane = lane_id();
  const int E = a.n_experts;
  // counts and offsets
  for (int e = tid; e < E; e += 1024) base_s[e] = 0;
  __syncthreads();
  for (int s = tid; s < a.n_slots; s += 1024) atomicAdd(&base_s[a.ids[s]], 1);
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    int n_gu = 0, n_d = 0;
    for (int e = 0; e < E; ++e) {
      off_s[e] = acc;
      const int c = base_s[e];
      const int chunks = (c + a.n_chunk - 1) / a.n_chunk;
      // items are written below by one thread per expert; here only the totals
      n_gu += chunks * a.m_tiles_gu;
      n_d += chunks * a.m_tiles_d;
      acc += c;
    }
    off_s[E] = acc;
    a.counts[0] = n_gu;
    a.counts[1] = n_d;
  }
  __syncthreads();
  for (int e = tid; e <= E; e += 1024) a.offsets[e] = off_s[e];
  // grouped items: thread e writes its expert's items (expert order, then m tile, then chunk)
  for (int e = tid; e < E; e += 1024) {
    const int c = base_s[e];
    const int chunks = (c + a.n_chunk - 1) / a.n_chunk;
    int before = 0;  // chunks of experts < e
    for (int f = 0; f < e; ++f) before += (base_s[f] + a.n_chunk - 1) / a.n_chunk;
    for (int ch = 0; ch < chunks; ++ch) {
      const int tok0 = off_s[e] + ch * a.n_chunk;
      const int n = min(a.n_chunk, c - ch * a.n_chunk);
      for (int m = 0; m < a.m_tiles_gu; ++m)
        a.items_gu[(before + ch) * a.m_tiles_gu + m] = make_int4(e, m, tok0, n);
      for (int m = 0; m < a.m_tiles_d; ++m)
        a.items_d[(before + ch) * a.m_tiles_d + m] = make_int4(e, m, tok0, n);
    }
  }
  __syncthreads();
  // stable placement, 1024 slots per round
  for (int e = tid; e < E; e += 1024) base_s[e] = off_s[e];
  for (int r0 = 0; r0 < a.n_slots; r0 += 1024) {
    for (int i = tid; i < 32 * 257; i += 1024) (&cnt[0][0])[i] = 0;
    __syncthreads();
    const int s = r0 + tid;
    const bool valid = s < a.n_slots;
    const int e = valid ? a.ids[s] : -1 - lane;  // distinct dummies never match real experts
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank == 0) cnt[warp][e] = __popc(peers);
    __syncthreads();
    if (valid) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += cnt[w][e];
      a.perm[base_s[e] + before + rank] = s;
    }
    __syncthreads();
    for (int f = tid; f < E; f += 1024) {
      int tot = 0;
      for (int w = 0; w < 32; ++w) tot += cnt[w][f];
      base_s[f] += tot;
    }
    __syncthreads();
  }
}

// x_perm[p] = xn[perm[p] / k]; one CTA per permuted row, 16-byte copies.
__global__ void gather_rows_kernel(const __nv_bfloat16* __restrict__ xn,
                                   const int32_t* __restrict__ perm, int top_k, int d,
                                   __nv_bfloat16* __restrict__ x_perm, const int* done) {
  if (block_done(done)) return;
  const int p = blockIdx.x;
  const int t = perm[p] / top_k;
  const uint4* src = reinterpret_cast<const uint4*>(xn + static_cast<long long>(t) * d);
  uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<long long>(p) * d);
  for (int i = threadIdx.x; i < d / 8; i += blockDim.x) dst[i] = src[i];
}

template <typename TA>
__global__ void __launch_bounds__(256) moe_combine_norm_kernel(
    float* __restrict__ x, const float* __restrict__ y_slot, int top_k,
    const float* __restrict__ y_shared, int d, const float* __restrict__ w, float eps,
    TA* __restrict__ xn, const int* done) {
  if (block_done(done)) return;
  __shared__ float sm[8];
  const int t = blockIdx.x;
  float* xr = x + static_cast<long long>(t) * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += 256) {
    float y = 0.f;
    for (int s = 0; s < top_k; ++s) y += y_slot[(static_cast<long long>(t) * top_k + s) * d + i];
    if (y_shared) y += y_shared[static_cast<long long>(t) * d + i];
    const float v = xr[i] + y;
    xr[i] = v;
    ss += v * v;
  }
  if (w == nullptr) return;  // standalone MoE: no following norm
  const float inv = rsqrtf(block_sum_256(ss, sm) / d + eps);
  for (int i = threadIdx.x; i < d; i += 256)
    xn[static_cast<long long>(t) * d + i] = store_from_f32<TA>(xr[i] * inv * w[i]);
}

// RoPE table: (cos, sin) of pos * theta^(-2i/hd) for pos < n_pos, i < hd/2, computed in fp64.
__global__ void rope_table_kernel(float2* tab, int n_pos, int half, double theta) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(n_pos) * half) return;
  const int pos = static_cast<int>(idx / half), i = static_cast<int>(idx % half);
  const double ang = pos * pow(theta, -2.0 * i / (2.0 * half));
  tab[idx] = make_float2(static_cast<float>(cos(ang)), static_cast<float>(sin(ang)));
}

}  // namespace dg
