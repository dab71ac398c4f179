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

// Merged statistics of a row in fp64 (relative to the row maximum m).
struct StatD {
  double m, s, u;
  int a;
};

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

// The id a re-noised position takes: the Philox draw of (position, step, block, tag 1).
DG_DEV int32_t renoise_id(const SamplerArgs& p, int row) {
  return canvas_uniform_id(p.seed, p.block, p.step, static_cast<uint32_t>(row), 1u,
                           static_cast<uint32_t>(p.vocab));
}

// Decide lock / re-noise for one row from its merged statistics (valid in lane 0) and write the
// row's outputs; returns (in every lane) whether this warp is the last row to finish the step.
// `noise` is the row's re-noise id when the caller drew it already (negative: drawn here).  The
// completion ticket is taken with one acquire-release atomic: this row's outputs are visible
// before it, and the last row sees every other row's outputs after it.
DG_DEV bool sampler_row_finish(const SamplerArgs& p, int row, const StatD& r, int32_t noise = -1) {
  int is_last = 0;
  if (lane_id() == 0) {
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
    if (!kept) p.canvas[row] = lock ? r.a : (noise >= 0 ? noise : renoise_id(p, row));
    is_last = (atomic_add_acq_rel(p.ticket, 1) == p.rows - 1);
  }
  is_last = __shfl_sync(0xffffffffu, is_last, 0);
  __syncwarp();
  return is_last != 0;
}

// Committed ids with sticky locks: a locked position's canvas token, otherwise the argmax.
__global__ void commit_ids_kernel(const int32_t* canvas, const int32_t* argmax,
                                  const int32_t* locked, int32_t* out, int n) {
  pdl_enter();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = locked[i] ? canvas[i] : argmax[i];
}

// Merge one row's nsplit partials with a 256-thread CTA, the row maximum M first (so the fp64
// exponentials are independent, with no dependent chain), then S = sum e^(m_i - M) S_i and
// U = sum e^(m_i - M) (U_i + (m_i - M) S_i); the argmax is the lowest index among the partials
// holding M.  Thread t takes partials t, t + 256, ...; the warps' maxima and then their sums
// combine through shared memory in warp order.  Valid in thread 0.
DG_DEV StatD sampler_row(const SamplerArgs& p, int row) {
  __shared__ float s_max[8];
  __shared__ double s_sum[2][8];
  __shared__ int s_arg[8];
  const float4* part = reinterpret_cast<const float4*>(p.partials) + static_cast<size_t>(row) * p.nsplit;
  const int tid = static_cast<int>(threadIdx.x), warp = tid >> 5;
  constexpr int kC = 4;  // partials per thread held in registers (nsplit <= 1024)
  float4 q[kC];
#pragma unroll
  for (int k = 0; k < kC; ++k) {
    const int i = tid + 256 * k;
    q[k] = i < p.nsplit ? __ldcg(part + i) : make_float4(-INFINITY, 0.f, 0.f, 0.f);
  }
  float m = -INFINITY;
#pragma unroll
  for (int k = 0; k < kC; ++k)
    if (q[k].y > 0.f) m = fmaxf(m, q[k].x);
  for (int i = tid + 256 * kC; i < p.nsplit; i += 256) {
    const float4 q4 = __ldcg(part + i);
    if (q4.y > 0.f) m = fmaxf(m, q4.x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane_id() == 0) s_max[warp] = m;
  __syncthreads();
  m = s_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, s_max[w]);
  double sum = 0.0, usum = 0.0;
  int a = 0x7fffffff;
  if (m != -INFINITY) {
    auto add = [&](const float4& q4) {
      if (q4.y > 0.f) {
        const double d = static_cast<double>(q4.x) - static_cast<double>(m);
        const double e = exp(d);
        sum += e * q4.y;
        usum += e * (static_cast<double>(q4.z) + d * q4.y);
        if (q4.x == m) a = min(a, __float_as_int(q4.w));
      }
    };
#pragma unroll
    for (int k = 0; k < kC; ++k) add(q[k]);
    for (int i = tid + 256 * kC; i < p.nsplit; i += 256) add(__ldcg(part + i));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    usum += __shfl_xor_sync(0xffffffffu, usum, o);
    a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
  }
  if (lane_id() == 0) {
    s_sum[0][warp] = sum;
    s_sum[1][warp] = usum;
    s_arg[warp] = a;
  }
  __syncthreads();
  StatD r{static_cast<double>(m), 0.0, 0.0, 0x7fffffff};
  if (tid == 0)
    for (int w = 0; w < 8; ++w) {
      r.s += s_sum[0][w];
      r.u += s_sum[1][w];
      r.a = min(r.a, s_arg[w]);
    }
  return r;
}

// The stop test over one canvas, run by the warp that finished its last row (after a fence).
// Rows written by other warps are read through L2 (ld.global.cg), eight rows per lane per batch so
// that the loads of a batch are in flight together; the mean entropy is a fixed-shape fp64 sum
// (per lane in row order, then a butterfly whose lane-0 result is used), so it does not depend on
// timing.  Each lane then stores its rows' argmax as the previous argmax of the next step.
DG_DEV void sampler_stop_test(const SamplerArgs& p) {
  __threadfence();
  constexpr int kBatch = 8;
  const int lane = static_cast<int>(lane_id());
  double h = 0.0;
  int n_diff = 0, n_locked = 0;
  for (int base = 0; base < p.rows; base += 32 * kBatch) {
    int am[kBatch], pv[kBatch], lk[kBatch];
    double hh[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int i = base + lane + 32 * k;
      if (i < p.rows) {
        am[k] = __ldcg(p.argmax + i);
        pv[k] = p.prev_argmax[i];
        lk[k] = __ldcg(p.locked + i);
        hh[k] = __ldcg(p.row_h + i);
      }
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int i = base + lane + 32 * k;
      if (i < p.rows) {
        n_diff += am[k] != pv[k];
        n_locked += lk[k];
        h += hh[k];
        p.prev_argmax[i] = am[k];
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) h += __shfl_xor_sync(0xffffffffu, h, o);
  n_diff = __reduce_add_sync(0xffffffffu, n_diff);
  n_locked = __reduce_add_sync(0xffffffffu, n_locked);
  if (lane == 0) {
    const double hbar = h / p.rows;
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
}

// One CTA per row of the n_seq canvases: merge the row's partials, decide lock / re-noise (warp 0);
// the last row of a canvas to finish evaluates the stop rule for that canvas (no CTA ever waits
// on another).  A canvas that has stopped is left as it is while the others go on.
__global__ void __launch_bounds__(256) sampler_merge_kernel(SamplerArgs p) {
  pdl_enter();
  const int b = blockIdx.x / p.rows;
  const SamplerArgs q = seq_view(p, b);
  if (block_done(q.state + kStDone)) return;
  const int row = blockIdx.x - b * p.rows;
  const StatD r = sampler_row(q, row);
  if (threadIdx.x < 32 && sampler_row_finish(q, row, r)) sampler_stop_test(q);
}

// ---- the standalone streaming sampler -------------------------------------------------------
// One warp streams a row slice in groups of kLoads 16-byte vectors per lane: column
// g + (l * 32 + lane) * kVec + j of the group starting at g (a group is a contiguous run of
// columns).  Per group a lane takes the group maximum first; when it exceeds the lane's running
// maximum m, the lane's S and U are rescaled to it and the group's start is remembered.  Then
//   d = x - m,  e = 2^(d log2 e),  S += e,  U += e d      (pairs in f32x2 arithmetic).
// The slice's maximum first occurs in the lowest of the remembered groups of the lanes holding
// it; the slice reports that group's start in place of a column, and the row's merge looks for
// the exact column in that one group.  A logit below -1e30 (a masked, -inf entry) is raised to
// -1e30 first, so e = 0 and e d = 0 instead of NaN; a row needs some logit above -1e30.
constexpr float kMaskedLogit = -1e30f;

template <typename T, int kLoads>
DG_DEV void warp_load_group(const T* base, int g, int c1, uint4 (&r)[kLoads]) {
  constexpr int kVec = 16 / static_cast<int>(sizeof(T));
  const int lane = static_cast<int>(lane_id());
#pragma unroll
  for (int l = 0; l < kLoads; ++l) {
    const int c = g + (l * 32 + lane) * kVec;
    if (c < c1)
      r[l] = __ldcs(reinterpret_cast<const uint4*>(base + c));
    else if constexpr (sizeof(T) == 2)
      r[l] = make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);  // bf16 -inf
    else
      r[l] = make_uint4(0xff800000u, 0xff800000u, 0xff800000u, 0xff800000u);  // fp32 -inf
  }
}

// value j (0 .. kVec-1) of a 16-byte vector as f32
template <typename T>
DG_DEV float vec_value(const uint4& v, int j) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if constexpr (sizeof(T) == 2)
    return __uint_as_float((j & 1) ? (w[j >> 1] & 0xffff0000u) : (w[j >> 1] << 16));
  else
    return __uint_as_float(w[j]);
}

template <typename T, int kLoads>
DG_DEV float group_max(const uint4 (&r)[kLoads]) {
  if constexpr (sizeof(T) == 2) {
    __nv_bfloat162 ml[kLoads];
#pragma unroll
    for (int l = 0; l < kLoads; ++l) {
      const __nv_bfloat162* w = reinterpret_cast<const __nv_bfloat162*>(&r[l]);
      ml[l] = __hmax2(__hmax2(w[0], w[1]), __hmax2(w[2], w[3]));
    }
#pragma unroll
    for (int st = 1; st < kLoads; st *= 2)
#pragma unroll
      for (int l = 0; l + st < kLoads; l += 2 * st) ml[l] = __hmax2(ml[l], ml[l + st]);
    return fmaxf(__low2float(ml[0]), __high2float(ml[0]));
  } else {
    float ml[kLoads];
#pragma unroll
    for (int l = 0; l < kLoads; ++l)
      ml[l] = fmaxf(fmaxf(__uint_as_float(r[l].x), __uint_as_float(r[l].y)),
                    fmaxf(__uint_as_float(r[l].z), __uint_as_float(r[l].w)));
#pragma unroll
    for (int st = 1; st < kLoads; st *= 2)
#pragma unroll
      for (int l = 0; l + st < kLoads; l += 2 * st) ml[l] = fmaxf(ml[l], ml[l + st]);
    return ml[0];
  }
}

template <typename T, int kLoads>
DG_DEV void group_accumulate(const uint4 (&r)[kLoads], float m, float2& s2, float2& u2) {
  constexpr float kLog2e = 1.4426950408889634f;
  const float2 nm2 = make_float2(-m, -m), l2 = make_float2(kLog2e, kLog2e);
#pragma unroll
  for (int l = 0; l < kLoads; ++l) {
    const uint32_t w4[4] = {r[l].x, r[l].y, r[l].z, r[l].w};
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat162 lo2 = __float2bfloat162_rn(kMaskedLogit);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 c = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&w4[q]), lo2);
        const uint32_t w = *reinterpret_cast<const uint32_t*>(&c);
        const float2 x = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
        const float2 d = __fadd2_rn(x, nm2);
        const float2 t = __fmul2_rn(d, l2);
        const float2 e = make_float2(fast_exp2(t.x), fast_exp2(t.y));
        s2 = __fadd2_rn(s2, e);
        u2 = __ffma2_rn(e, d, u2);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; q += 2) {
        const float2 x = make_float2(fmaxf(__uint_as_float(w4[q]), kMaskedLogit),
                                     fmaxf(__uint_as_float(w4[q + 1]), kMaskedLogit));
        const float2 d = __fadd2_rn(x, nm2);
        const float2 t = __fmul2_rn(d, l2);
        const float2 e = make_float2(fast_exp2(t.x), fast_exp2(t.y));
        s2 = __fadd2_rn(s2, e);
        u2 = __ffma2_rn(e, d, u2);
      }
    }
  }
}

// Statistics (m, S, U, g) of columns [c0, c1) of one row for one warp, g the start of the lowest
// group holding the maximum (every lane gets the same g; S and U are valid in lane 0).
template <typename T, int kLoads>
DG_DEV StatPartial warp_slice_stats(const T* base, int c0, int c1) {
  constexpr int kVec = 16 / static_cast<int>(sizeof(T));
  constexpr int kSpan = kLoads * 32 * kVec;
  constexpr float kLog2e = 1.4426950408889634f;
  float m = -INFINITY;
  float2 s2 = make_float2(0.f, 0.f), u2 = make_float2(0.f, 0.f);
  int gidx = c0;
  for (int g = c0; g < c1; g += kSpan) {
    uint4 r[kLoads];
    warp_load_group<T, kLoads>(base, g, c1, r);
    const float gm = group_max<T, kLoads>(r);
    if (gm > m) {  // strict: an earlier group keeps an equal maximum
      gidx = g;
      if (m != -INFINITY) {
        const float d = m - gm;
        const float sc = fast_exp2(d * kLog2e);
        u2 = make_float2(sc * (u2.x + d * s2.x), sc * (u2.y + d * s2.y));
        s2 = make_float2(sc * s2.x, sc * s2.y);
      }
      m = gm;
    }
    if (m != -INFINITY) group_accumulate<T, kLoads>(r, m, s2, u2);
  }
  float s = s2.x + s2.y, u = u2.x + u2.y;
  // the warp maximum, every lane's sums relative to it, then plain sums
  float bm = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
  if (m == -INFINITY || bm == -INFINITY) {
    s = 0.f;
    u = 0.f;
  } else if (m != bm) {
    const float d = m - bm;
    const float sc = fast_exp2(d * kLog2e);
    u = sc * (u + d * s);
    s *= sc;
  }
  int ga = (m == bm && bm != -INFINITY) ? gidx : 0x7fffffff;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    u += __shfl_xor_sync(0xffffffffu, u, o);
    ga = min(ga, __shfl_xor_sync(0xffffffffu, ga, o));
  }
  return StatPartial{bm, s, u, ga};
}

// Columns per row segment of the streaming sampler: 8 vectors per lane (2048 bf16, 1024 fp32).
constexpr int kStreamLoads = 8;
template <typename T>
constexpr int stream_span() {
  return kStreamLoads * 32 * (16 / static_cast<int>(sizeof(T)));
}

// The run of units [floor(w T / W), floor((w + 1) T / W)) belongs to worker w; unit u is worked
// by the largest w whose run starts at or before u, w(u) = floor(((u + 1) W - 1) / T).  Both
// floors are taken of an fp64 quotient, exact while the numerator is below 2^53: for a / b with
// a mod b <= b - 1 the quotient's rounding error (a / b) 2^-53 stays below the gap 1 / b to the
// next integer.
DG_DEV long long stream_run_start(long long w, long long workers, long long total) {
  return static_cast<long long>(floor(static_cast<double>(w * total) / static_cast<double>(workers)));
}
DG_DEV long long stream_worker(long long u, long long workers, long long total) {
  return static_cast<long long>(
      floor(static_cast<double>((u + 1) * workers - 1) / static_cast<double>(total)));
}

// Statistics of every row piece in one launch on a persistent grid of warps.  The rows x segs
// units (one group each) are cut into one contiguous run per warp; a warp streams its run and
// writes one partial per row piece (a run covers a few rows at most) at the piece's first
// segment.  No warp waits on another; sampler_stream_rows_kernel merges the rows.
template <typename T>
__global__ void __launch_bounds__(256, sizeof(T) == 2 ? 4 : 3)
    sampler_stream_kernel(const T* __restrict__ logits, int32_t segs, SamplerArgs p) {
  pdl_enter();
  if (block_done(p.state + kStDone)) return;
  constexpr int kSpan = stream_span<T>();
  const long long workers = static_cast<long long>(gridDim.x) * 8;
  const long long w = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const long long total = static_cast<long long>(p.rows) * segs;
  long long u = w * total / workers;
  const long long u_end = (w + 1) * total / workers;
  while (u < u_end) {
    const int row = static_cast<int>(u / segs);
    const int seg0 = static_cast<int>(u % segs);
    const int len = static_cast<int>(min(u_end, static_cast<long long>(row + 1) * segs) - u);
    const int c0 = seg0 * kSpan;
    const int c1 = min(p.vocab, (seg0 + len) * kSpan);
    const StatPartial r = warp_slice_stats<T, kStreamLoads>(
        logits + static_cast<size_t>(row) * p.vocab, c0, c1);
    if (lane_id() == 0)
      const_cast<StatPartial*>(p.partials)[static_cast<size_t>(row) * segs + seg0] = r;
    u += len;
  }
}

// One warp per row (8 rows per CTA), after sampler_stream_kernel ran with `workers` warps: merge
// the row's pieces (piece k is the part of worker w_lo + k's run inside the row, k = 0 starting at
// the row's first segment; an empty run has none), find the first column holding the row maximum
// in the lowest group reported for it, decide lock / re-noise; the last row to finish runs the
// stop test.  The loads that do not depend on one another are issued together: the stopped flag,
// the pieces and the re-noise draw first, the group holding the maximum before the fp64 sums.
template <typename T>
__global__ void __launch_bounds__(256) sampler_stream_rows_kernel(const T* __restrict__ logits,
                                                                  int32_t segs, SamplerArgs p,
                                                                  long long workers) {
  const int row = static_cast<int>(blockIdx.x) * 8 + static_cast<int>(threadIdx.x >> 5);
  if (row >= p.rows) {
    pdl_enter();
    return;
  }
  constexpr int kC = 4;
  constexpr int kVec = 16 / static_cast<int>(sizeof(T));
  const int lane = static_cast<int>(lane_id());
  // what depends on the arguments alone (the pieces' slots from the static split, the re-noise
  // draw) is worked out while the streaming kernel finishes
  const long long total = static_cast<long long>(p.rows) * segs;
  const long long r0 = static_cast<long long>(row) * segs;
  const long long w_lo = stream_worker(r0, workers, total);
  const long long w_hi = stream_worker(r0 + segs - 1, workers, total);
  const int n = static_cast<int>(w_hi - w_lo + 1);
  const float4* part = reinterpret_cast<const float4*>(p.partials) + r0;
  auto slot_of = [&](int k) -> long long {
    if (k == 0) return 0;
    const long long a = stream_run_start(w_lo + k, workers, total);
    if (w_lo + k < w_hi && a == stream_run_start(w_lo + k + 1, workers, total)) return -1;
    return a - r0;
  };
  long long slot0[kC];  // the slots of the first pass
#pragma unroll
  for (int k = 0; k < kC; ++k) {
    const int i = lane + 32 * k;
    slot0[k] = i < n ? slot_of(i) : -1;
  }
  const int32_t noise = lane == 0 ? renoise_id(p, row) : 0;
  pdl_enter();
  const int stopped = *reinterpret_cast<const volatile int*>(p.state + kStDone);
  float4 q[kC];
  auto load = [&](int base) {
#pragma unroll
    for (int k = 0; k < kC; ++k) {
      const int i = base + lane + 32 * k;
      const long long sl = base == 0 ? slot0[k] : (i < n ? slot_of(i) : -1);
      q[k] = sl >= 0 ? __ldcg(part + sl) : make_float4(-INFINITY, 0.f, 0.f, 0.f);
    }
  };
  // the row maximum and the lowest group holding it
  float m = -INFINITY;
  for (int base = 0; base < n; base += 32 * kC) {
    load(base);
#pragma unroll
    for (int k = 0; k < kC; ++k)
      if (q[k].y > 0.f) m = fmaxf(m, q[k].x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  int g = 0x7fffffff;
  for (int base = 0; base < n; base += 32 * kC) {
    if (n > 32 * kC) load(base);
#pragma unroll
    for (int k = 0; k < kC; ++k)
      if (q[k].y > 0.f && q[k].x == m) g = min(g, __float_as_int(q[k].w));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) g = min(g, __shfl_xor_sync(0xffffffffu, g, o));
  if (stopped) return;  // uniform over the grid
  uint4 v[kStreamLoads];
  if (g != 0x7fffffff)
    warp_load_group<T, kStreamLoads>(logits + static_cast<size_t>(row) * p.vocab, g, p.vocab, v);
  // S and U relative to the row maximum while the group is on its way
  double sum = 0.0, usum = 0.0;
  if (m != -INFINITY) {
    for (int base = 0; base < n; base += 32 * kC) {
      if (n > 32 * kC) load(base);
#pragma unroll
      for (int k = 0; k < kC; ++k)
        if (q[k].y > 0.f) {
          const double d = static_cast<double>(q[k].x) - static_cast<double>(m);
          const double e = exp(d);
          sum += e * q[k].y;
          usum += e * (static_cast<double>(q[k].z) + d * q[k].y);
        }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    usum += __shfl_xor_sync(0xffffffffu, usum, o);
  }
  int a = 0x7fffffff;
  if (g != 0x7fffffff) {
#pragma unroll
    for (int l = kStreamLoads - 1; l >= 0; --l)
#pragma unroll
      for (int j = kVec - 1; j >= 0; --j)
        if (vec_value<T>(v[l], j) == m) a = g + (l * 32 + lane) * kVec + j;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (sampler_row_finish(p, row, StatD{static_cast<double>(m), sum, usum, a}, noise))
    sampler_stop_test(p);
}

}  // namespace dg
