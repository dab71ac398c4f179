// sampler.cuh -- canvas sampler kernels: Philox canvas fill, per-chunk softmax statistics
// of logits, and the merge + lock/re-noise + adaptive-stop kernel.
//
// Statistics of one row x over a vocabulary slice, relative to the slice maximum m:
//   S = sum exp(x - m),  U = sum exp(x - m) (x - m),  a = lowest index with x = m.
// Slices merge exactly: with M = max m_s,  S = sum e^(m_s - M) S_s,
//   U = sum e^(m_s - M) (U_s + (m_s - M) S_s).  Then conf = max prob = 1 / S and the
// entropy is H = ln S - U / S (nats).  The decision rules follow the canvas description:
// lock when conf >= tau, otherwise re-noise with the Philox draw of (position, step,
// block, tag 1); stop after step t >= 2 when mean H < h_bound and the argmax vector equals
// the previous step's.
#pragma once
#include "dg_common.cuh"
#include "philox.cuh"

namespace dg {

// Layout of the device state words (mirrors DG_STATE_* in dg.h).
enum : int {
  kStDone = 0,
  kStStopStep = 1,
  kStWouldStop = 2,
  kStStepsRun = 3,
  kStLocked = 4,
  kStError = 5,
  kStWords = 16
};

struct StatPartial {  // 16 bytes: m, S, U, argmax (int bits)
  float m, s, u;
  int a;
};

// Merge two statistics; on equal maxima the lower argmax wins (lowest-index rule).
struct StatD {
  double m, s, u;
  int a;
};
DG_DEV StatD stat_merge(const StatD& x, const StatD& y) {
  if (y.s == 0.0) return x;
  if (x.s == 0.0) return y;
  StatD r;
  if (x.m > y.m || (x.m == y.m && x.a < y.a)) {
    r.m = x.m;
    r.a = x.a;
  } else {
    r.m = y.m;
    r.a = y.a;
  }
  const double ex = exp(x.m - r.m), ey = exp(y.m - r.m);
  r.s = ex * x.s + ey * y.s;
  r.u = ex * (x.u + (x.m - r.m) * x.s) + ey * (y.u + (y.m - r.m) * y.s);
  return r;
}

__global__ void canvas_init_kernel(int32_t* canvas, int32_t t, int32_t vocab, uint64_t seed,
                                   uint32_t block, int32_t* state, int32_t* ticket) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < t) canvas[i] = canvas_uniform_id(seed, block, 0u, static_cast<uint32_t>(i), 0u,
                                           static_cast<uint32_t>(vocab));
  if (blockIdx.x == 0 && threadIdx.x < kStWords) {
    state[threadIdx.x] = 0;
    if (threadIdx.x == 0) *ticket = 0;
  }
}

// Partial statistics of one row slice.  grid = (chunks, rows), 256 threads; each thread
// holds up to kPerThread values in registers.  Partial index = row * chunks + chunk.
template <typename T, int kPerThread>
__global__ void __launch_bounds__(256) logits_stats_kernel(const T* __restrict__ logits,
                                                           int32_t vocab, int32_t chunk,
                                                           StatPartial* __restrict__ out,
                                                           const int* done) {
  if (block_done(done)) return;
  constexpr int kVec = 16 / sizeof(T);
  constexpr int kLoads = kPerThread / kVec;
  const int row = blockIdx.y;
  const int c0 = blockIdx.x * chunk;
  const int c1 = min(c0 + chunk, vocab);
  const T* base = logits + static_cast<size_t>(row) * vocab;
  float v[kPerThread];
  float m = -INFINITY;
  int a = 0x7fffffff;
#pragma unroll
  for (int l = 0; l < kLoads; ++l) {
    const int col = c0 + (l * blockDim.x + threadIdx.x) * kVec;
    if (col < c1) {
      const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(base + col));
      const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int j = 0; j < kVec; ++j) {
        const float x = load_as_f32<T>(e, j);
        v[l * kVec + j] = x;
        if (x > m) {
          m = x;
          a = col + j;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < kVec; ++j) v[l * kVec + j] = -INFINITY;
    }
  }
  // block max with lowest index
  __shared__ float sm_m[8];
  __shared__ int sm_a[8];
  __shared__ float sm_s[8], sm_u[8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, o);
    const int oa = __shfl_xor_sync(0xffffffffu, a, o);
    if (om > m || (om == m && oa < a)) {
      m = om;
      a = oa;
    }
  }
  const int warp = threadIdx.x >> 5;
  if (lane_id() == 0) {
    sm_m[warp] = m;
    sm_a[warp] = a;
  }
  __syncthreads();
  float bm = sm_m[0];
  int ba = sm_a[0];
  for (int w = 1; w < 8; ++w) {
    if (sm_m[w] > bm || (sm_m[w] == bm && sm_a[w] < ba)) {
      bm = sm_m[w];
      ba = sm_a[w];
    }
  }
  float s = 0.f, u = 0.f;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const float d = v[i] - bm;
    const float e = __expf(d);  // exp(-inf) = 0 for padding
    s += e;
    u += (d > -INFINITY) ? e * d : 0.f;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    u += __shfl_xor_sync(0xffffffffu, u, o);
  }
  if (lane_id() == 0) {
    sm_s[warp] = s;
    sm_u[warp] = u;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float ts = 0.f, tu = 0.f;
    for (int w = 0; w < 8; ++w) {
      ts += sm_s[w];
      tu += sm_u[w];
    }
    out[static_cast<size_t>(row) * gridDim.x + blockIdx.x] = StatPartial{bm, ts, tu, ba};
  }
}

struct SamplerArgs {
  const StatPartial* partials;  // [rows, nsplit]
  int32_t nsplit;
  int32_t rows;
  int32_t vocab;
  uint64_t seed;
  uint32_t block;
  uint32_t step;
  float tau;
  float h_bound;
  int32_t max_steps;
  int32_t fixed_steps;
  int32_t* canvas;
  int32_t* argmax;
  int32_t* prev_argmax;
  float* entropy;
  float* conf;
  double* row_h;
  int32_t* locked;
  int32_t* state;
  int32_t* ticket;
};

// One CTA per row: merge the row's partials, decide lock / re-noise; the last CTA to finish
// evaluates the stop rule for the whole canvas (no CTA ever waits on another).
__global__ void __launch_bounds__(256) sampler_merge_kernel(SamplerArgs p) {
  if (block_done(p.state + kStDone)) return;
  const int row = blockIdx.x;
  StatD acc{0.0, 0.0, 0.0, 0x7fffffff};
  for (int i = threadIdx.x; i < p.nsplit; i += blockDim.x) {
    const StatPartial q = p.partials[static_cast<size_t>(row) * p.nsplit + i];
    acc = stat_merge(acc, StatD{q.m, q.s, q.u, q.a});
  }
  __shared__ StatD red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] = stat_merge(red[threadIdx.x], red[threadIdx.x + o]);
    __syncthreads();
  }
  __shared__ int is_last;
  if (threadIdx.x == 0) {
    const StatD r = red[0];
    const double conf = 1.0 / r.s;
    const double h = log(r.s) - r.u / r.s;
    p.conf[row] = static_cast<float>(conf);
    p.entropy[row] = static_cast<float>(h);
    p.row_h[row] = h;
    const bool lock = conf >= static_cast<double>(p.tau);
    p.argmax[row] = r.a;
    p.locked[row] = lock ? 1 : 0;
    p.canvas[row] = lock ? r.a
                         : canvas_uniform_id(p.seed, p.block, p.step, static_cast<uint32_t>(row),
                                             1u, static_cast<uint32_t>(p.vocab));
    __threadfence();
    is_last = (atomicAdd(p.ticket, 1) == p.rows - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // --- last CTA: stop test over the whole canvas -------------------------------------
  __shared__ int n_diff, n_locked;
  if (threadIdx.x == 0) {
    n_diff = 0;
    n_locked = 0;
  }
  __syncthreads();
  int my_diff = 0, my_locked = 0;
  for (int i = threadIdx.x; i < p.rows; i += blockDim.x) {
    my_diff += (*reinterpret_cast<volatile int32_t*>(p.argmax + i) != p.prev_argmax[i]);
    my_locked += *reinterpret_cast<volatile int32_t*>(p.locked + i);
  }
  atomicAdd(&n_diff, my_diff);
  atomicAdd(&n_locked, my_locked);
  __syncthreads();
  if (threadIdx.x == 0) {
    double hsum = 0.0;
    for (int i = 0; i < p.rows; ++i)  // fixed order: deterministic mean
      hsum += *reinterpret_cast<volatile double*>(p.row_h + i);
    const double hbar = hsum / p.rows;
    const int step = static_cast<int>(p.step);
    const bool stop_now = step >= 2 && hbar < static_cast<double>(p.h_bound) && n_diff == 0;
    int32_t* st = p.state;
    st[kStStepsRun] = step;
    st[kStLocked] = n_locked;
    if (stop_now && st[kStWouldStop] == 0) st[kStWouldStop] = step;
    const bool done = (p.fixed_steps > 0) ? (step >= p.fixed_steps)
                                          : (stop_now || step >= p.max_steps);
    if (done) {
      st[kStStopStep] = step;
      st[kStDone] = 1;
    }
    *p.ticket = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < p.rows; i += blockDim.x)
    p.prev_argmax[i] = *reinterpret_cast<volatile int32_t*>(p.argmax + i);
}

}  // namespace dg
