// gemm_cluster.cuh -- the canvas's dense projections (QKV, O, router) as split-K GEMMs whose K
// splits of one weight tile form a thread-block cluster.
//
// Tile: 128 weight rows (the UMMA "A", M = 128) x up to 256 tokens (N) over K / S slabs, where S is
// the cluster size.  Each CTA accumulates its K range in TMEM (warp 0 feeds a TMA ring, warp 1
// issues the UMMAs, as in gemm.cuh); the eight epilogue warps drain the fp32 accumulator into
// shared memory as [token][row]; after a cluster barrier, CTA s of the cluster sums the S partial
// tiles over its own token range in rank order 0..S-1 (distributed shared memory loads, so the
// sum never depends on timing) and applies the consumer's epilogue:
//   kCluQkv:      q and k heads get rotate-half RoPE at absolute positions and go to Q
//                 [Hq, tq, hd] or the K cache; v heads go transposed into V^T of the cache (one
//                 M tile is one head: hd = 128);
//   kCluResidual: x[token][row] += sum (the O projection onto the residual stream);
//   kCluRouter:   router logits, top-k per token (one warp per token), and the CTA of the grid
//                 that finishes last (ticket) builds the expert permutation and chunk list.
// A second cluster barrier keeps each CTA's shared memory alive until its peers have read it.
// Every thread reaches both cluster barriers whatever happened before (a failed bounded wait only
// turns the remaining work off), so the barriers cannot wait for an absent thread.
#pragma once
#include "dg_common.cuh"
#include "layer.cuh"

namespace dg {

enum CluEpi : int { kCluQkv = 0, kCluResidual = 1, kCluRouter = 2 };

constexpr int kCluStages = 4;
constexpr int kCluABytes = 128 * 128;           // 128 rows x 64 bf16
constexpr int kCluBBytes = 256 * 128;           // 256 tokens x 64 bf16
constexpr int kCluStageBytes = kCluABytes + kCluBBytes;
constexpr int kCluRingBytes = kCluStages * kCluStageBytes;  // 192 KB, reused by the epilogue
constexpr int kCluDrainBytes = 256 * 128 * 4;   // fp32 [token][row] partial tile
// ring, 1 KB that lets the V^T scratch overhang the ring, alignment slack, barriers
constexpr int kCluSmemBytes = kCluRingBytes + 1024 + 1024 + 256;
constexpr int kCluThreads = 64 + 32 * 8;
constexpr int kCluMaxSplits = 8;
// epilogue scratch after the drained tile: a V^T tile [128][<= 256 tokens] bf16, or the router
// logits of <= 128 tokens [token][128] fp32
static_assert(kCluDrainBytes + 128 * 257 * 2 <= kCluRingBytes + 1024, "V^T scratch");
static_assert(kCluDrainBytes + 128 * 128 * 4 <= kCluRingBytes, "router scratch");

struct CluParams {
  int n_tokens;   // tokens of this call
  int chunk_n;    // tokens per token chunk (<= 256, a multiple of 32)
  int n_chunks;   // token chunks
  int m_tiles;    // weight tiles of 128 rows
  int m_rows;     // weight rows in use
  int kb_total;   // K / 64
  int splits;     // cluster size S (<= kb_total)
  int b_row_base; // tm_b row of token 0
  // kCluQkv
  int n_heads, n_kv_heads, tq, pos0, ldk;
  const float2* rope_tab;  // [position][hd / 2] (cos, sin)
  __nv_bfloat16* q;
  __nv_bfloat16* k_cache;   // [Hkv, ldk, hd] of this layer
  __nv_bfloat16* vt_cache;  // [Hkv, hd, ldk] of this layer
  // batched canvases: token t belongs to sequence t / seq_len at position pos0 + t % seq_len,
  // whose cache lies seq_kv_stride elements after sequence 0's (seq_len 0: one sequence)
  int seq_len;
  long long seq_kv_stride;
  // kCluResidual
  float* x;                 // [tokens, m_rows] fp32
  // kCluRouter
  float* router_logits;     // [tokens, E]
  int32_t* ids;             // [tokens, k]
  float* wts;               // [tokens, k]
  int top_k;
  RouteArgs route;
  int32_t* ticket;          // starts and ends at zero
  const void* pf_first;     // hinted into L2 by the CTAs that do not route (null: none)
  long long pf_first_bytes;
  int* err;
  const int* done;
};

// Sums over the S cluster ranks of G row groups (token t[g0 + g], rows 4 r4[g0 + g] ..) of the
// drained partial tiles, in rank order, with every load issued before the first add.
template <int G, int SMAX>
DG_DEV void reduce_groups(uint32_t drain_u32, int S, const int (&t)[4], const int (&r4)[4], int g0,
                          float4 (&out)[4]) {
  float4 v[G][SMAX];
#pragma unroll
  for (int src = 0; src < SMAX; ++src)
    if (src < S) {
#pragma unroll
      for (int g = 0; g < G; ++g)
        v[g][src] = dsmem_ld4(dsmem_addr(
            drain_u32 + static_cast<uint32_t>((t[g0 + g] * 128 + 4 * r4[g0 + g]) * 4),
            static_cast<uint32_t>(src)));
    }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int src = 0; src < SMAX; ++src)
      if (src < S) {
        acc.x += v[g][src].x;
        acc.y += v[g][src].y;
        acc.z += v[g][src].z;
        acc.w += v[g][src].w;
      }
    out[g0 + g] = acc;
  }
}

template <int EPI>
__global__ void __launch_bounds__(kCluThreads, 1)
    gemm_cluster_kernel(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b, const CluParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kCluRingBytes + 1024);
  uint64_t* empty = full + kCluStages;
  uint64_t* acc_full = empty + kCluStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  const int warp = threadIdx.x >> 5;
  const int S = p.splits;
  const int s = static_cast<int>(blockIdx.x) % S;  // == cluster rank (cluster dims (S, 1, 1))
  const int tile = static_cast<int>(blockIdx.x) / S;
  const int mt = tile / p.n_chunks, nc = tile % p.n_chunks;
  const int t0 = nc * p.chunk_n;                    // first token of the chunk
  const int n = min(p.chunk_n, p.n_tokens - t0);    // tokens of the chunk
  const int kb0 = s * p.kb_total / S, kb1 = (s + 1) * p.kb_total / S;

  if (warp == 0 && lane_id() == 0) {
    for (int i = 0; i < kCluStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // the setup above overlaps the previous kernel; from here on its results are needed
  pdl_enter();
  if (block_done(p.done)) {  // uniform over the grid: release TMEM and leave
    if (warp == 1) tmem_dealloc(tmem_base, 256);
    return;
  }
  bool ok = true;  // this thread's waits all succeeded

  if (warp == 0) {
    if (elect_one()) {
      const uint64_t pol_a = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();
      const int nbox = (n + 31) >> 5;
      const uint32_t bytes = kCluABytes + nbox * 32 * 128;
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, p.err)) break;
        uint8_t* sa = smem + stage * kCluStageBytes;
        uint8_t* sb = sa + kCluABytes;
        mbar_arrive_expect_tx(&full[stage], bytes);
        tma_load_2d(&tm_a, &full[stage], sa, kb * 64, mt * 128, pol_a);
        for (int bx = 0; bx < nbox; ++bx)
          tma_load_2d(&tm_b, &full[stage], sb + bx * 4096, kb * 64, p.b_row_base + t0 + bx * 32,
                      pol_b);
        if (++stage == kCluStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = idesc_bf16_f32(128, (n + 15) & ~15);
      int stage = 0;
      uint32_t phase = 0;
      bool mok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[stage], phase, p.err)) {
          mok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + stage * kCluStageBytes);
        const uint64_t da = sdesc_sw128(sa);
        const uint64_t db = sdesc_sw128(sa + kCluABytes);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem_base, da + 2 * k, db + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
        umma_commit(&empty[stage]);
        if (++stage == kCluStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (mok) umma_commit(acc_full);  // every UMMA above (and its shared-memory reads) done
    }
  } else {
    // drain: warp quarter q owns TMEM lanes (rows) 32q..32q+31, half h the tokens 128h..128h+127
    const int q = warp & 3, h = (warp - 2) >> 2;
    const int r = q * 32 + lane_id();
    ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, p.err));
    if (ok) {
      tc_fence_after();
      float* drain = reinterpret_cast<float*>(smem);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const int tok = h * 128 + c * 32;
        if (tok >= n) break;
        float v[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + tok, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) drain[(tok + i) * 128 + r] = v[i];
      }
    }
  }
  ok = __syncthreads_and(ok);  // the drain of every warp, and whether all of it happened
  cluster_sync_all();          // #1: every partial tile of the cluster is in shared memory

  // ---- reduction over the cluster and the epilogue (all 320 threads) ----
  const int tid = threadIdx.x;
  const int t_lo = n * s / S, t_hi = n * (s + 1) / S, nt = t_hi - t_lo;
  const uint32_t drain_u32 = smem_u32(smem);
  // sum of the S partials of (token t, rows 4 r4 .. 4 r4 + 3), ranks in order; every peer's load
  // is issued before the first add so the distributed shared memory latencies overlap
  auto reduce4 = [&](int t, int r4) -> float4 {
    const uint32_t off = drain_u32 + static_cast<uint32_t>((t * 128 + 4 * r4) * 4);
    float4 v[kCluMaxSplits];
#pragma unroll
    for (int src = 0; src < kCluMaxSplits; ++src)
      if (src < S) v[src] = dsmem_ld4(dsmem_addr(off, static_cast<uint32_t>(src)));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int src = 0; src < kCluMaxSplits; ++src)
      if (src < S) {
        acc.x += v[src].x;
        acc.y += v[src].y;
        acc.z += v[src].z;
        acc.w += v[src].w;
      }
    return acc;
  };
  // four row groups at once (token, row group) -> sums with all their loads in flight; the
  // groups go two by two when the cluster is larger than four (register budget)
  auto reduce4x4 = [&](const int (&t)[4], const int (&r4)[4], float4 (&out)[4]) {
    if (S <= 4) {
      reduce_groups<4, 4>(drain_u32, S, t, r4, 0, out);
    } else {
      reduce_groups<2, kCluMaxSplits>(drain_u32, S, t, r4, 0, out);
      reduce_groups<2, kCluMaxSplits>(drain_u32, S, t, r4, 2, out);
    }
  };
  const int rows4 = min(32, (p.m_rows - mt * 128 + 3) >> 2);  // valid float4 row groups
  if constexpr (EPI == kCluResidual) {
    if (ok) {
      // two units per pass: the residual rows and every partial in flight together
      const int total = nt * rows4;
      for (int u0 = tid; u0 < total; u0 += 2 * kCluThreads) {
        int tt[4] = {0, 0, 0, 0}, rr[4] = {0, 0, 0, 0};
        float4 xv[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int u = min(u0 + k * kCluThreads, total - 1);
          tt[k] = t_lo + u / rows4;
          rr[k] = u % rows4;
          xv[k] = *reinterpret_cast<const float4*>(
              p.x + static_cast<long long>(t0 + tt[k]) * p.m_rows + mt * 128 + 4 * rr[k]);
        }
        float4 sum[4];
        reduce_groups<2, kCluMaxSplits>(drain_u32, S, tt, rr, 0, sum);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          if (u0 + k * kCluThreads >= total) break;
          float4 a = xv[k];
          a.x += sum[k].x;
          a.y += sum[k].y;
          a.z += sum[k].z;
          a.w += sum[k].w;
          *reinterpret_cast<float4*>(p.x + static_cast<long long>(t0 + tt[k]) * p.m_rows +
                                     mt * 128 + 4 * rr[k]) = a;
        }
      }
    }
  } else if constexpr (EPI == kCluQkv) {
    const int head = mt;  // 128 rows = one head
    // [hd][nt + 1]: the odd row pitch spreads a warp's stores (consecutive row groups) over banks
    __nv_bfloat16* vt_s = reinterpret_cast<__nv_bfloat16*>(smem + kCluDrainBytes);
    const int vp = nt + 1;
    if (head < p.n_heads + p.n_kv_heads) {
      if (ok) {
        // rotate-half pairs (i, i + 64): float4 groups r4 and r4 + 16; two units per pass so
        // that their table and partial loads are all in flight together
        for (int u0 = tid; u0 < nt * 16; u0 += 2 * kCluThreads) {
          int tt[4], rr[4];
          float2 cs[2][4];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int u = min(u0 + k * kCluThreads, nt * 16 - 1);
            const int t = t_lo + u / 16, r4 = u % 16;
            tt[2 * k] = tt[2 * k + 1] = t;
            rr[2 * k] = r4;
            rr[2 * k + 1] = r4 + 16;
            const int tg = t0 + t;
            const int rel = p.seq_len > 0 ? tg % p.seq_len : tg;
            const float2* tab = p.rope_tab + static_cast<long long>(p.pos0 + rel) * 64 + 4 * r4;
#pragma unroll
            for (int i = 0; i < 4; ++i) cs[k][i] = tab[i];
          }
          float4 sum[4];
          reduce4x4(tt, rr, sum);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            if (u0 + k * kCluThreads >= nt * 16) break;
            const int tg = t0 + tt[2 * k], r4 = rr[2 * k];
            const int sq = p.seq_len > 0 ? tg / p.seq_len : 0;
            const int rel = tg - sq * p.seq_len;
            const float4 a = sum[2 * k], b = sum[2 * k + 1];
            __nv_bfloat16* dst =
                head < p.n_heads
                    ? p.q + (static_cast<long long>(head) * p.tq + tg) * 128
                    : p.k_cache + sq * p.seq_kv_stride +
                          (static_cast<long long>(head - p.n_heads) * p.ldk + p.pos0 + rel) * 128;
            const float2 c0 = cs[k][0], c1 = cs[k][1], c2 = cs[k][2], c3 = cs[k][3];
            const float lo[4] = {a.x * c0.x - b.x * c0.y, a.y * c1.x - b.y * c1.y,
                                 a.z * c2.x - b.z * c2.y, a.w * c3.x - b.w * c3.y};
            const float hi[4] = {b.x * c0.x + a.x * c0.y, b.y * c1.x + a.y * c1.y,
                                 b.z * c2.x + a.z * c2.y, b.w * c3.x + a.w * c3.y};
            store4<__nv_bfloat16>(dst + 4 * r4, make_float4(lo[0], lo[1], lo[2], lo[3]));
            store4<__nv_bfloat16>(dst + 64 + 4 * r4, make_float4(hi[0], hi[1], hi[2], hi[3]));
          }
        }
      }
    } else {
      // v head: sums into a [dim][token] bf16 tile, then rows of V^T (contiguous positions)
      if (ok) {
        for (int u = tid; u < nt * 32; u += kCluThreads) {
          const int tl = u / 32, r4 = u % 32;
          const float4 a = reduce4(t_lo + tl, r4);
          vt_s[(4 * r4 + 0) * vp + tl] = __float2bfloat16_rn(a.x);
          vt_s[(4 * r4 + 1) * vp + tl] = __float2bfloat16_rn(a.y);
          vt_s[(4 * r4 + 2) * vp + tl] = __float2bfloat16_rn(a.z);
          vt_s[(4 * r4 + 3) * vp + tl] = __float2bfloat16_rn(a.w);
        }
      }
      __syncthreads();
      if (ok) {
        const int g = head - p.n_heads - p.n_kv_heads;
        for (int u = tid; u < 128 * nt; u += kCluThreads) {
          const int dd = u / nt, tl = u % nt;
          const int tg = t0 + t_lo + tl;
          const int sq = p.seq_len > 0 ? tg / p.seq_len : 0;
          p.vt_cache[sq * p.seq_kv_stride + (static_cast<long long>(g) * 128 + dd) * p.ldk +
                     p.pos0 + tg - sq * p.seq_len] = vt_s[dd * vp + tl];
        }
      }
    }
  } else {  // kCluRouter: E = m_rows <= 128 (one tile), top-k of this CTA's tokens (nt <= 128)
    float* lg = reinterpret_cast<float*>(smem + kCluDrainBytes);  // [nt][128]
    const int E = p.m_rows;
    if (ok) {
      for (int u = tid; u < nt * 32; u += kCluThreads) {
        const int tl = u / 32, r4 = u % 32;
        float4 v = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (r4 < rows4) {
          v = reduce4(t_lo + tl, r4);
          *reinterpret_cast<float4*>(p.router_logits +
                                     static_cast<long long>(t0 + t_lo + tl) * E + 4 * r4) = v;
        }
        *reinterpret_cast<float4*>(lg + tl * 128 + 4 * r4) = v;
      }
    }
    __syncthreads();
    if (ok) {
      for (int tl = warp; tl < nt; tl += kCluThreads / 32) {
        const float4 v0 = *reinterpret_cast<const float4*>(lg + tl * 128 + 4 * lane_id());
        float v[8] = {v0.x, v0.y, v0.z, v0.w, -INFINITY, -INFINITY, -INFINITY, -INFINITY};
        const long long tg = t0 + t_lo + tl;
        router_topk_select(v, E, p.top_k, p.ids + tg * p.top_k, p.wts + tg * p.top_k);
      }
    }
  }
  cluster_sync_all();  // #2: the peers are done with this CTA's shared memory

  if constexpr (EPI == kCluRouter) {
    // the last CTA of the grid routes the whole call (its shared memory is free now)
    __shared__ int is_last;
    if (tid == 0) {
      __threadfence();
      is_last = (atomicAdd(p.ticket, 1) == static_cast<int>(gridDim.x) - 1);
    }
    __syncthreads();
    if (is_last) {
      __threadfence();
      if (tid == 0) *p.ticket = 0;
      route_canvas(p.route, reinterpret_cast<int*>(smem));
    } else if (tid == 0) {
      // the others hint the weights the grouped GEMM streams first into L2 (its items go in
      // expert order, and a canvas' 2,048 slots leave hardly any expert empty)
      prefetch_l2_slice(p.pf_first, p.pf_first_bytes, blockIdx.x, gridDim.x);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

}  // namespace dg
