// fp32_path.cuh -- the all-fp32 variants of the contraction kernels (the small correctness
// model stores everything in fp32, where bf16 or tf32 tensor-core inputs would be too coarse
// for a 1e-4 tolerance).  Plain SIMT fp32, sequential accumulation order.
#pragma once
#include "dg_common.cuh"

namespace dg {

// out[m * ld + n] = sum_k X[m, k] * W[n, k]   (X [M, K], W [N, K], both row-major)
__global__ void __launch_bounds__(256) gemm_f32_nt_kernel(const float* __restrict__ X,
                                                          const float* __restrict__ W, int M, int N,
                                                          int K, float* __restrict__ out,
                                                          long long ld, const int* done) {
  pdl_enter();
  if (block_done(done)) return;
  __shared__ float xs[16][65];
  __shared__ float ws[16][65];
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      const int r = i >> 4, c = i & 15;
      xs[c][r] = (m0 + r < M && k0 + c < K) ? X[static_cast<long long>(m0 + r) * K + k0 + c] : 0.f;
      ws[c][r] = (n0 + r < N && k0 + c < K) ? W[static_cast<long long>(n0 + r) * K + k0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = xs[c][ty * 4 + i];
        b[i] = ws[c][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) out[static_cast<long long>(m) * ld + n] = acc[i][j];
    }
}

// One CTA per (token, head); scores for every visible key in shared memory, exact softmax.
// q [Hq, tq, hd], k [Hkv, ldk, hd], vt [Hkv, hd, ldk]; o [T, Hq * hd].
__global__ void __launch_bounds__(128) attention_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ vt,
    float* __restrict__ o, int n_heads, int group, int tq, int hd, int ldk, int n_keys,
    int causal_prefix, float scale, const int* done) {
  pdl_enter();
  if (block_done(done)) return;
  extern __shared__ float sc[];  // [n_keys] scores, then [hd] query
  float* qs = sc + n_keys;
  __shared__ float red[4];
  const int t = blockIdx.x, h = blockIdx.y, g = h / group;
  const int lim = causal_prefix >= 0 ? min(n_keys, causal_prefix + t + 1) : n_keys;
  for (int i = threadIdx.x; i < hd; i += blockDim.x)
    qs[i] = q[(static_cast<long long>(h) * tq + t) * hd + i];
  __syncthreads();
  float mx = -INFINITY;
  for (int n = threadIdx.x; n < lim; n += blockDim.x) {
    const float* kr = k + (static_cast<long long>(g) * ldk + n) * hd;
    float s = 0.f;
    for (int i = 0; i < hd; ++i) s = fmaf(qs[i], kr[i], s);
    s *= scale;
    sc[n] = s;
    mx = fmaxf(mx, s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane_id() == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float sum = 0.f;
  for (int n = threadIdx.x; n < lim; n += blockDim.x) {
    const float e = expf(sc[n] - mx);
    sc[n] = e;
    sum += e;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane_id() == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  sum = red[0] + red[1] + red[2] + red[3];
  for (int i = threadIdx.x; i < hd; i += blockDim.x) {
    const float* vr = vt + (static_cast<long long>(g) * hd + i) * ldk;
    float acc = 0.f;
    for (int n = 0; n < lim; ++n) acc = fmaf(sc[n], vr[n], acc);
    o[static_cast<long long>(t) * n_heads * hd + h * hd + i] = acc / sum;
  }
}

// One CTA per routed slot (token t, slot s) -- or per token for the shared expert
// (ids == nullptr): h = silu(x W_g^T) * (x W_u^T), y = h W_d^T, scaled by the router weight.
__global__ void __launch_bounds__(256) moe_expert_f32_kernel(
    const float* __restrict__ xn, const int32_t* __restrict__ ids, const float* __restrict__ wts,
    int top_k, const float* __restrict__ w_gu, const float* __restrict__ w_d, int d, int hidden,
    float* __restrict__ y, const int* done) {
  pdl_enter();
  if (block_done(done)) return;
  extern __shared__ float sm[];  // [d] x, then [hidden] h
  float* xs = sm;
  float* hs = sm + d;
  const int slot = blockIdx.x;
  const int t = ids ? slot / top_k : slot;
  const int e = ids ? ids[slot] : 0;
  const float scale = ids ? wts[slot] : 1.0f;
  const float* gu = w_gu + static_cast<long long>(e) * 2 * hidden * d;
  const float* dn = w_d + static_cast<long long>(e) * d * hidden;
  for (int i = threadIdx.x; i < d; i += 256) xs[i] = xn[static_cast<long long>(t) * d + i];
  __syncthreads();
  for (int j = threadIdx.x; j < hidden; j += 256) {
    const float* rg = gu + static_cast<long long>(2 * j) * d;
    const float* ru = rg + d;
    float g = 0.f, u = 0.f;
    for (int i = 0; i < d; ++i) {
      g = fmaf(xs[i], rg[i], g);
      u = fmaf(xs[i], ru[i], u);
    }
    hs[j] = g / (1.0f + expf(-g)) * u;
  }
  __syncthreads();
  for (int f = threadIdx.x; f < d; f += 256) {
    const float* rd = dn + static_cast<long long>(f) * hidden;
    float acc = 0.f;
    for (int j = 0; j < hidden; ++j) acc = fmaf(hs[j], rd[j], acc);
    y[static_cast<long long>(slot) * d + f] = acc * scale;
  }
}

}  // namespace dg
