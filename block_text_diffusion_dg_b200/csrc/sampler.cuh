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
// the previous step's.  Variants: lock when H <= entropy_lock instead (the recipe's
// "entropy_bound" sampler), and sticky locks (a locked position keeps its token for the rest
// of the block instead of being re-decided every step).
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

// Canvas fill of n_seq canvases of t positions: canvas b takes the Philox stream keyed by seed + b
// ([canvas] step 2: ids uniform over the vocabulary), with counter (position, 0, block, 0).  The
// decode state of every canvas is reset (state words [n_seq][kStWords], completion tickets
// [n_seq], lock flags) and so are the all-canvases-done words (all_done[0] flag, all_done[1]
// count; may be null).
__global__ void canvas_init_kernel(int32_t* canvas, int32_t t, int32_t n_seq, int32_t vocab,
                                   uint64_t seed, uint32_t block, int32_t* state, int32_t* ticket,
                                   int32_t* locked, int32_t* all_done) {
  pdl_enter();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < t * n_seq) {
    const int b = i / t;
    canvas[i] = canvas_uniform_id(seed + static_cast<uint64_t>(b), block, 0u,
                                  static_cast<uint32_t>(i - b * t), 0u, static_cast<uint32_t>(vocab));
    if (locked) locked[i] = 0;
  }
  if (blockIdx.x == 0) {
    for (int w = threadIdx.x; w < n_seq * kStWords; w += blockDim.x) state[w] = 0;
    if (threadIdx.x < n_seq) ticket[threadIdx.x] = 0;
    if (all_done && threadIdx.x < 2) all_done[threadIdx.x] = 0;
  }
}

// Floor of x - m in the exponent sums.  Logits may hold -inf (masked vocabulary entries) as long
// as every row has a finite value: such an entry has x - m = -inf, and e^(x - m) (x - m) would be
// 0 * -inf = NaN, which would make the row's entropy, the mean entropy and hence the stop test NaN.
// Clamping x - m at -1e30 makes its term exactly 0 (2^(-1e30 log2 e) = 0, 0 * -1e30 = 0).
constexpr float kMaskedDelta = -1e30f;

// Fresh decode state for a block: state words, completion tickets and all-done words zeroed, lock
// flags of the n_seq * t canvas positions cleared; the canvases themselves are kept
// (dg_reset_block).
__global__ void block_reset_kernel(int32_t* state, int32_t* ticket, int32_t* locked, int32_t t,
                                   int32_t n_seq, int32_t* all_done) {
  pdl_enter();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < t * n_seq) locked[i] = 0;
  if (blockIdx.x == 0) {
    for (int w = threadIdx.x; w < n_seq * kStWords; w += blockDim.x) state[w] = 0;
    if (threadIdx.x < n_seq) ticket[threadIdx.x] = 0;
    if (all_done && threadIdx.x < 2) all_done[threadIdx.x] = 0;
  }
}

// Statistics (m, S, U, argmax) of one row slice held in registers by a 256-thread CTA: pass 1
// takes the maximum (only threads holding it then look for its lowest column), pass 2
// accumulates e = 2^((x - m) log2 e), S += e, U += e (x - m).  Value i of a thread sits at column
// c0 + ((i / kVec) * 256 + tid) * kVec + i % kVec; values past the row end are -inf (`full` = no
// such padding in this slice, uniform over the CTA).
// With a temperature T (inv_t = 1 / T) the statistics are those of x / T: d = (x - m) / T and
// the slice maximum is returned as m / T; the argmax does not depend on T.
template <int kPerThread, int kVec>
DG_DEV StatPartial slice_stats(const float (&v)[kPerThread], int c0, bool full, float* sm_f,
                               int* sm_i, float inv_t = 1.0f) {
  const int warp = threadIdx.x >> 5;
  float tm = v[0];
#pragma unroll
  for (int i = 1; i < kPerThread; ++i) tm = fmaxf(tm, v[i]);
  float m = tm;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane_id() == 0) sm_f[warp] = m;
  __syncthreads();
  float bm = sm_f[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) bm = fmaxf(bm, sm_f[w]);
  int a = 0x7fffffff;
  if (tm == bm) {  // rare: this thread holds the slice maximum; values are in column order
#pragma unroll
    for (int i = kPerThread - 1; i >= 0; --i)
      if (v[i] == bm) a = c0 + ((i / kVec) * 256 + static_cast<int>(threadIdx.x)) * kVec + i % kVec;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
  constexpr float kLog2e = 1.4426950408889634f;
  float s4[4] = {0.f, 0.f, 0.f, 0.f}, u4[4] = {0.f, 0.f, 0.f, 0.f};
  if (full) {
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      // a -inf logit (masked vocabulary entry) gives d = -1e30: e = 0 and e * d = 0, not NaN
      const float d = fmaxf((v[i] - bm) * inv_t, kMaskedDelta);
      const float e = fast_exp2(d * kLog2e);
      s4[i & 3] += e;
      u4[i & 3] = fmaf(e, d, u4[i & 3]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      if (v[i] != -INFINITY) {
        const float d = (v[i] - bm) * inv_t;
        const float e = fast_exp2(d * kLog2e);
        s4[i & 3] += e;
        u4[i & 3] = fmaf(e, d, u4[i & 3]);
      }
    }
  }
  float s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
  float u = (u4[0] + u4[1]) + (u4[2] + u4[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    u += __shfl_xor_sync(0xffffffffu, u, o);
  }
  __syncthreads();  // sm_f is reused below
  if (lane_id() == 0) {
    sm_f[warp] = s;
    sm_f[8 + warp] = u;
    sm_i[warp] = a;
  }
  __syncthreads();
  StatPartial r{bm * inv_t, 0.f, 0.f, 0x7fffffff};
  if (threadIdx.x == 0) {
    for (int w = 0; w < 8; ++w) {
      r.s += sm_f[w];
      r.u += sm_f[8 + w];
      r.a = min(r.a, sm_i[w]);
    }
  }
  return r;  // valid in thread 0
}

// Load this CTA's slice of one row (layout as above); returns whether it has no padding.
template <typename T, int kPerThread>
DG_DEV bool load_slice(const T* base, int c0, int c1, float (&v)[kPerThread]) {
  constexpr int kVec = 16 / sizeof(T);
  constexpr int kLoads = kPerThread / kVec;
  const bool full = c0 + kPerThread * 256 <= c1;
#pragma unroll
  for (int l = 0; l < kLoads; ++l) {
    const int c = c0 + (l * 256 + threadIdx.x) * kVec;
    if (full || c < c1) {
      const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(base + c));
      const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int j = 0; j < kVec; ++j) v[l * kVec + j] = load_as_f32<T>(e, j);
    } else {
#pragma unroll
      for (int j = 0; j < kVec; ++j) v[l * kVec + j] = -INFINITY;
    }
  }
  return full;
}

// Partial statistics of one row slice.  grid = (chunks, rows), 256 threads, chunk =
// 256 * kPerThread columns.  Partial index = row * chunks + chunk.
template <typename T, int kPerThread>
__global__ void __launch_bounds__(256) logits_stats_kernel(const T* __restrict__ logits,
                                                           int32_t vocab, int32_t chunk,
                                                           StatPartial* __restrict__ out,
                                                           const int* done,
                                                           float inv_t = 1.0f) {
  pdl_enter();
  if (block_done(done)) return;
  __shared__ float sm_f[16];
  __shared__ int sm_i[8];
  const int row = blockIdx.y;
  const int c0 = blockIdx.x * chunk;
  float v[kPerThread];
  const bool full = load_slice<T, kPerThread>(logits + static_cast<size_t>(row) * vocab, c0,
                                              min(c0 + chunk, vocab), v);
  const StatPartial r = slice_stats<kPerThread, 16 / sizeof(T)>(v, c0, full, sm_f, sm_i, inv_t);
  if (threadIdx.x == 0) out[static_cast<size_t>(row) * gridDim.x + blockIdx.x] = r;
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
  int32_t lock_rule;   // 0: lock when conf >= tau; 1: lock when H <= entropy_lock
  float entropy_lock;
  int32_t sticky;      // nonzero: a locked position keeps its token (locked[] persists)
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
  // Batched canvases: n_seq canvases of `rows` positions each, stored one after another in every
  // per-row array (partials too); canvas b keys its Philox stream with seed + b and has its own
  // state words (state + b * kStWords) and ticket (ticket + b).  all_done (may be null): [0] is
  // set once every canvas has stopped, [1] counts the stopped canvases.
  int32_t n_seq;
  int32_t* all_done;
};

// The arguments of canvas b alone.
DG_DEV SamplerArgs seq_view(const SamplerArgs& p, int b) {
  SamplerArgs q = p;
  const long long r0 = static_cast<long long>(b) * p.rows;
  q.partials = p.partials + r0 * p.nsplit;
  q.seed = p.seed + static_cast<uint64_t>(b);
  q.canvas = p.canvas + r0;
  q.argmax = p.argmax + r0;
  q.prev_argmax = p.prev_argmax + r0;
  q.entropy = p.entropy + r0;
  q.conf = p.conf + r0;
  q.row_h = p.row_h + r0;
  q.locked = p.locked + r0;
  q.state = p.state + b * kStWords;
  q.ticket = p.ticket + b;
  return q;
}

// Decide lock / re-noise for one row from its merged statistics and write the row's outputs;
// returns (in every thread) whether this CTA is the last row to finish the step.
DG_DEV bool sampler_row_finish(const SamplerArgs& p, int row, const StatD& r) {
  __shared__ int is_last;
  if (threadIdx.x == 0) {
    const double conf = 1.0 / r.s;
    const double h = log(r.s) - r.u / r.s;
    p.conf[row] = static_cast<float>(conf);
    p.entropy[row] = static_cast<float>(h);
    p.row_h[row] = h;
    const bool lock = p.lock_rule == 0 ? conf >= static_cast<double>(p.tau)
                                        : h <= static_cast<double>(p.entropy_lock);
    const bool kept = p.sticky != 0 && p.locked[row] != 0;
    p.argmax[row] = r.a;
    p.locked[row] = (lock || kept) ? 1 : 0;
    if (!kept)
      p.canvas[row] = lock ? r.a
                           : canvas_uniform_id(p.seed, p.block, p.step, static_cast<uint32_t>(row),
                                               1u, static_cast<uint32_t>(p.vocab));
    __threadfence();
    is_last = (atomicAdd(p.ticket, 1) == p.rows - 1);
  }
  __syncthreads();
  return is_last;
}

// Committed ids with sticky locks: a locked position's canvas token, otherwise the argmax.
__global__ void commit_ids_kernel(const int32_t* canvas, const int32_t* argmax,
                                  const int32_t* locked, int32_t* out, int n) {
  pdl_enter();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = locked[i] ? canvas[i] : argmax[i];
}

// Merge one row's nsplit partials (block-wide, fp64 tree) and finish the row.
DG_DEV bool sampler_row(const SamplerArgs& p, int row) {
  StatD acc{0.0, 0.0, 0.0, 0x7fffffff};
  for (int i = threadIdx.x; i < p.nsplit; i += blockDim.x) {
    const float4 q4 = __ldcg(reinterpret_cast<const float4*>(p.partials) +
                             static_cast<size_t>(row) * p.nsplit + i);
    acc = stat_merge(acc, StatD{q4.x, q4.y, q4.z, __float_as_int(q4.w)});
  }
  __shared__ StatD red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] = stat_merge(red[threadIdx.x], red[threadIdx.x + o]);
    __syncthreads();
  }
  return sampler_row_finish(p, row, red[0]);
}

// Merge one row's pieces in column order: the piece starting at segment s keeps its partial at
// slot row * segs + s and its length in segments at the same slot of piece_len.
DG_DEV bool sampler_row_pieces(const SamplerArgs& p, int row, int segs,
                               const int32_t* piece_len) {
  // every slot of the row in one parallel round trip (slots that start no piece hold stale
  // values and are never visited), then thread 0 follows the chain from segment 0
  constexpr int kMaxSegs = 256;
  __shared__ float4 sp[kMaxSegs];
  __shared__ int sl[kMaxSegs];
  __shared__ StatD merged;
  for (int i = threadIdx.x; i < segs && i < kMaxSegs; i += blockDim.x) {
    const size_t slot = static_cast<size_t>(row) * segs + i;
    sp[i] = __ldcg(reinterpret_cast<const float4*>(p.partials) + slot);
    sl[i] = __ldcg(piece_len + slot);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    StatD acc{0.0, 0.0, 0.0, 0x7fffffff};
    for (int s = 0; s < segs;) {
      float4 q4;
      int len;
      if (s < kMaxSegs) {
        q4 = sp[s];
        len = sl[s];
      } else {
        const size_t slot = static_cast<size_t>(row) * segs + s;
        q4 = __ldcg(reinterpret_cast<const float4*>(p.partials) + slot);
        len = __ldcg(piece_len + slot);
      }
      acc = stat_merge(acc, StatD{q4.x, q4.y, q4.z, __float_as_int(q4.w)});
      s += max(1, len);
    }
    merged = acc;
  }
  __syncthreads();
  return sampler_row_finish(p, row, merged);
}

// The stop test over the whole canvas, run by the last row's CTA (after a fence).  Rows written
// by other CTAs are read through L2 (ld.global.cg); the mean entropy is a fixed-shape fp64 tree
// over the rows, so it does not depend on timing.  rows <= 1024.
DG_DEV void sampler_stop_test(const SamplerArgs& p) {
  __threadfence();
  __shared__ double hs[256];
  __shared__ int n_diff, n_locked;
  if (threadIdx.x == 0) {
    n_diff = 0;
    n_locked = 0;
  }
  double h_part = 0.0;
  int my_diff = 0, my_locked = 0;
  for (int i = threadIdx.x; i < p.rows; i += blockDim.x) {
    my_diff += (__ldcg(p.argmax + i) != p.prev_argmax[i]);
    my_locked += __ldcg(p.locked + i);
    h_part += __ldcg(p.row_h + i);
  }
  hs[threadIdx.x] = h_part;
  __syncthreads();
  atomicAdd(&n_diff, my_diff);
  atomicAdd(&n_locked, my_locked);
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) hs[threadIdx.x] += hs[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double hbar = hs[0] / p.rows;
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
      if (p.all_done && atomicAdd(p.all_done + 1, 1) == p.n_seq - 1) p.all_done[0] = 1;
    }
    *p.ticket = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < p.rows; i += blockDim.x) p.prev_argmax[i] = __ldcg(p.argmax + i);
}

// One CTA per row of the n_seq canvases: merge the row's partials, decide lock / re-noise; the
// last CTA of a canvas to finish evaluates the stop rule for that canvas (no CTA ever waits on
// another).  A canvas that has stopped is left as it is while the others go on.
__global__ void __launch_bounds__(256) sampler_merge_kernel(SamplerArgs p) {
  pdl_enter();
  const int b = blockIdx.x / p.rows;
  const SamplerArgs q = seq_view(p, b);
  if (block_done(q.state + kStDone)) return;
  if (sampler_row(q, blockIdx.x - b * p.rows)) sampler_stop_test(q);
}

// (m, S, U, a) <- merge with (m2, S2, U2, a2) in fp32 (2^x on the special-function unit); an
// empty side (S = 0) is ignored; equal maxima keep the lower argmax.
DG_DEV void stat_merge_f32(float& m, float& s, float& u, int& a, float m2, float s2, float u2,
                           int a2) {
  constexpr float kLog2e = 1.4426950408889634f;
  if (s2 == 0.f) return;
  if (s == 0.f) {
    m = m2;
    s = s2;
    u = u2;
    a = a2;
    return;
  }
  const float mm = fmaxf(m, m2);
  const int aa = (m > m2 || (m == m2 && a < a2)) ? a : a2;
  const float d1 = m - mm, d2 = m2 - mm;
  const float e1 = fast_exp2(d1 * kLog2e), e2 = fast_exp2(d2 * kLog2e);
  u = e1 * (u + d1 * s) + e2 * (u2 + d2 * s2);
  s = e1 * s + e2 * s2;
  m = mm;
  a = aa;
}

// Streaming statistics of one row slice for a 256-thread CTA.  Every thread walks its columns in
// groups of kLoads 16-byte vectors (column c0 + ((g * kLoads + l) * 256 + tid) * kVec + j,
// increasing in (g, l, j)) keeping running (m, S, T, a) with T = sum e t, t = (x - m) log2 e,
// e = 2^t (so U = T / log2 e) and a the first column holding m; S and T are rescaled only when a
// group raises the maximum, which is also the only time the group is searched for its first
// maximal column.  The CTA merge rescales every thread's sums once to the CTA maximum and adds
// them up; the argmax is the lowest column among the threads holding that maximum.  Thread 0
// returns the result.
template <typename T> DG_DEV void to_f32x8(const uint4& raw, float (&v)[16 / sizeof(T)]);
template <> DG_DEV void to_f32x8<__nv_bfloat16>(const uint4& raw, float (&v)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    v[2 * q] = __uint_as_float(w[q] << 16);
    v[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
  }
}
template <> DG_DEV void to_f32x8<float>(const uint4& raw, float (&v)[4]) {
  v[0] = __uint_as_float(raw.x);
  v[1] = __uint_as_float(raw.y);
  v[2] = __uint_as_float(raw.z);
  v[3] = __uint_as_float(raw.w);
}

template <typename T, int kLoads>
DG_DEV StatPartial stream_slice_stats(const T* base, int c0, int c1) {
  constexpr int kVec = 16 / sizeof(T);
  constexpr int kSpan = kLoads * 256 * kVec;  // columns per group over the CTA
  constexpr float kLog2e = 1.4426950408889634f;
  const int tid = threadIdx.x;
  float m = -INFINITY;
  float2 s2 = make_float2(0.f, 0.f), t2 = make_float2(0.f, 0.f);
  int a = 0x7fffffff;
  for (int g0 = c0; g0 < c1; g0 += kSpan) {
    const bool full = g0 + kSpan <= c1;
    uint4 raw[kLoads];
#pragma unroll
    for (int l = 0; l < kLoads; ++l) {
      const int c = g0 + (l * 256 + tid) * kVec;
      if (full || c < c1) {
        raw[l] = __ldcs(reinterpret_cast<const uint4*>(base + c));
      } else if constexpr (sizeof(T) == 2) {
        raw[l] = make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);  // bf16 -inf
      } else {
        raw[l] = make_uint4(0xff800000u, 0xff800000u, 0xff800000u, 0xff800000u);  // fp32 -inf
      }
    }
    // group maximum (packed bf16 pairs for bf16 input); -inf padding never wins
    float gm;
    if constexpr (sizeof(T) == 2) {
      __nv_bfloat162 mx = *reinterpret_cast<const __nv_bfloat162*>(&raw[0].x);
#pragma unroll
      for (int l = 0; l < kLoads; ++l) {
        const uint32_t w[4] = {raw[l].x, raw[l].y, raw[l].z, raw[l].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) mx = __hmax2(mx, *reinterpret_cast<const __nv_bfloat162*>(&w[q]));
      }
      gm = fmaxf(__low2float(mx), __high2float(mx));
    } else {
      gm = -INFINITY;
#pragma unroll
      for (int l = 0; l < kLoads; ++l)
        gm = fmaxf(fmaxf(__uint_as_float(raw[l].x), __uint_as_float(raw[l].y)),
                   fmaxf(fmaxf(__uint_as_float(raw[l].z), __uint_as_float(raw[l].w)), gm));
    }
    if (gm > m) {  // strict: an earlier group keeps an equal maximum
      if (m != -INFINITY) {
        const float dt = (m - gm) * kLog2e;  // t shifts by dt for every earlier term
        const float sc = fast_exp2(dt);
        t2 = make_float2(sc * (t2.x + dt * s2.x), sc * (t2.y + dt * s2.y));
        s2 = make_float2(sc * s2.x, sc * s2.y);
      }
      m = gm;
      // first column of this group holding the new maximum (columns increase with l, then j)
      int found = 0x7fffffff;
#pragma unroll
      for (int l = kLoads - 1; l >= 0; --l) {
        float v[kVec];
        to_f32x8<T>(raw[l], v);
#pragma unroll
        for (int j = kVec - 1; j >= 0; --j)
          if (v[j] == gm) found = g0 + (l * 256 + tid) * kVec + j;
      }
      a = found;
    }
    // t = (x - m) log2 e with the subtraction first, so the maximum's own term is exactly 2^0
    const float2 l2 = make_float2(kLog2e, kLog2e);
    const float2 nm2 = make_float2(-m, -m);
    if (full) {
#pragma unroll
      for (int l = 0; l < kLoads; ++l) {
        float v[kVec];
        to_f32x8<T>(raw[l], v);
#pragma unroll
        for (int j = 0; j < kVec; j += 2) {
          float2 t = fmul2(fadd2(make_float2(v[j], v[j + 1]), nm2), l2);
          // -inf logits: t = -inf (or NaN while m is still -inf) becomes -1e30, so e = 0 and
          // e * t = 0 instead of NaN
          t = make_float2(fmaxf(t.x, kMaskedDelta), fmaxf(t.y, kMaskedDelta));
          const float2 e = make_float2(fast_exp2(t.x), fast_exp2(t.y));
          s2 = fadd2(s2, e);
          t2 = ffma2(e, t, t2);
        }
      }
    } else {  // ragged end of the row: -inf padding contributes nothing (and no 0 * -inf)
#pragma unroll
      for (int l = 0; l < kLoads; ++l) {
        float v[kVec];
        to_f32x8<T>(raw[l], v);
#pragma unroll
        for (int j = 0; j < kVec; ++j)
          if (v[j] != -INFINITY) {
            const float t = (v[j] - m) * kLog2e;
            const float e = fast_exp2(t);
            s2.x += e;
            t2.x = fmaf(e, t, t2.x);
          }
      }
    }
  }
  float s = s2.x + s2.y, tt = t2.x + t2.y;
  // CTA maximum
  const int warp = tid >> 5;
  __shared__ float wmax[8];
  __shared__ float wsum[2][8];
  __shared__ int warg[8];
  float bm = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
  if (lane_id() == 0) wmax[warp] = bm;
  __syncthreads();
  bm = wmax[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) bm = fmaxf(bm, wmax[w]);
  // every thread's sums relative to the CTA maximum, then plain sums; argmax = lowest column
  // among the threads that hold the maximum
  if (m == -INFINITY || bm == -INFINITY) {
    s = 0.f;
    tt = 0.f;
  } else if (m != bm) {
    const float dt = (m - bm) * kLog2e;
    const float sc = fast_exp2(dt);
    tt = sc * (tt + dt * s);
    s *= sc;
  }
  int am = (m == bm) ? a : 0x7fffffff;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    tt += __shfl_xor_sync(0xffffffffu, tt, o);
    am = min(am, __shfl_xor_sync(0xffffffffu, am, o));
  }
  if (lane_id() == 0) {
    wsum[0][warp] = s;
    wsum[1][warp] = tt;
    warg[warp] = am;
  }
  __syncthreads();
  StatPartial r{-INFINITY, 0.f, 0.f, 0x7fffffff};
  if (tid == 0) {
    float rs = 0.f, rt = 0.f;
    int ra = 0x7fffffff;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      rs += wsum[0][w];
      rt += wsum[1][w];
      ra = min(ra, warg[w]);
    }
    r = StatPartial{bm, rs, rt * (1.0f / kLog2e), ra};
  }
  __syncthreads();  // the shared arrays are rewritten by the next slice
  return r;
}

// Statistics, merge and stop test in one launch on a balanced persistent grid.  The rows x segs
// units (one kSpan-column group each) are cut into gridDim.x contiguous runs of equal length; a
// CTA streams its run and writes one partial per row piece (a run covers a few rows at most),
// kept at the piece's first segment together with its length.  A per-row count of finished
// segments finds the CTA completing the row, which merges the pieces in column order; the last
// row runs the stop test.  No CTA waits on another; row_units [rows] starts and ends at zero.
template <typename T, int kLoads>
__global__ void __launch_bounds__(256, sizeof(T) == 2 ? 5 : 3)
    sampler_stream_kernel(const T* __restrict__ logits, int32_t segs, SamplerArgs p,
                          int32_t* __restrict__ row_units, int32_t* __restrict__ piece_len) {
  pdl_enter();
  if (block_done(p.state + kStDone)) return;
  constexpr int kSpan = kLoads * 256 * (16 / static_cast<int>(sizeof(T)));
  __shared__ int last_piece;
  const long long total = static_cast<long long>(p.rows) * segs;
  long long u = blockIdx.x * total / gridDim.x;
  const long long u_end = (blockIdx.x + 1) * total / gridDim.x;
  while (u < u_end) {
    const int row = static_cast<int>(u / segs);
    const int seg0 = static_cast<int>(u % segs);
    const int len = static_cast<int>(min(u_end, static_cast<long long>(row + 1) * segs) - u);
    const int c0 = seg0 * kSpan;
    const int c1 = min(p.vocab, (seg0 + len) * kSpan);
    const StatPartial r =
        stream_slice_stats<T, kLoads>(logits + static_cast<size_t>(row) * p.vocab, c0, c1);
    const size_t slot = static_cast<size_t>(row) * segs + seg0;
    if (threadIdx.x == 0) {
      const_cast<StatPartial*>(p.partials)[slot] = r;
      piece_len[slot] = len;
      __threadfence();
      last_piece = (atomicAdd(row_units + row, len) + len == segs);
    }
    __syncthreads();
    if (last_piece) {
      __threadfence();
      if (threadIdx.x == 0) row_units[row] = 0;
      if (sampler_row_pieces(p, row, segs, piece_len)) sampler_stop_test(p);
    }
    __syncthreads();  // last_piece is rewritten by the next piece
    u += len;
  }
}

}  // namespace dg
