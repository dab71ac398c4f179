// gemm.cuh -- tcgen05 GEMMs of the denoise step.
//
// gemm_swapab_kernel: D[r, j] = sum_k W[a_row + r, k] * X[b_row + j, k] with the weight tile
// as the UMMA "A" operand (M = 128 rows) and the token tile as "B" (N = n tokens, 16..MAXN).
// Weights stream through shared memory exactly once per tile; the few tokens (256 on a
// canvas, ~16 per expert) ride along as the narrow N side.  One CTA per SM, three roles:
//   warp 0  : TMA producer (one elected thread) filling a STAGES-deep ring of 64-wide K slabs
//   warp 1  : UMMA issuer (one elected thread), fp32 accumulators double-buffered in TMEM
//   warps 2-5: epilogue, TMEM lane quarter (warp % 4), one accumulator row per thread.
// Work items are either arithmetic (dense layers, optional split-K) or a device-built list
// (grouped experts, one item per (expert, 128-row tile, token chunk)).
// Operand formats (FMT): 0 bf16; 1 e4m3 codes (kind::f8f6f4: a 128-byte K slab holds 128
// elements); 2 NVFP4 (kind::mxf4nvf4.block_scale.block16: a slab holds 256 e2m1 codes, and each
// stage also brings the slab's 512-byte scale atoms for A and B, which the MMA thread moves into
// TMEM with tcgen05.cp before the four MMAs that read them).  The ring and the operand
// descriptors are the same for all three; with FMT != 0 the epilogue first scales each
// accumulator by its weight row's scale and its token row's scale.
//
// lmhead_kernel: logits tile = X[256 tokens] * E[256 vocab rows]^T (two M=128 token tiles,
// N = 256 vocab) with the epilogue reducing every row of the tile straight from TMEM to the
// softmax statistics (max, argmax, sum e^(x-m), sum e^(x-m)(x-m)); logits never reach HBM.
#pragma once
#include "dg_common.cuh"
#include "sampler.cuh"

namespace dg {

enum EpiMode : int { kEpiPartialF32 = 0, kEpiGluBf16 = 1, kEpiScatterF32 = 2 };

struct GemmParams {
  // dense items: it -> (m tile, k split, n chunk)
  int m_tiles, k_splits, n_chunks, n_total, n_chunk, a_row_base, b_row_base;
  // grouped items (chunks != nullptr): the shared expert's (m tile, token chunk) pairs first,
  // tile-major, then every routed chunk with each of the m_tiles weight tiles, chunk-major.
  // chunks[c] = (expert, first permuted row, tokens, -), *chunk_count of them (device-built).
  const int4* chunks;
  const int* chunk_count;
  int a_rows_per_group;
  int kb_total;  // K / 64
  int m_valid;   // rows of A per group that are real (epilogue guard)
  // epilogue
  float* out_f32;
  __nv_bfloat16* out_bf16;
  long long ld_out;
  long long split_stride;
  const int* perm;     // scatter: destination (token * k + slot) of each permuted row
  const float* scale;  // scatter: route weight of each permuted row (indexed like B's rows)
  // the shared expert folded into a grouped launch (alt_group >= 0): its items read tm_a2 /
  // tm_b2 (rows of the unpermuted tokens), run alt_kb_total K slabs, write alt_out_* with no
  // permutation and weight 1
  int alt_group;
  int alt_m_tiles;   // weight tiles of the shared expert
  int alt_chunks;    // token chunks of the shared expert (n_chunk tokens each)
  int alt_tokens;
  int alt_kb_total;
  int alt_m_valid;
  float* alt_out_f32;
  __nv_bfloat16* alt_out_bf16;
  long long alt_ld_out;
  // weights of the kernels that follow, hinted into L2 by each CTA's producer once its items are
  // all issued (the last wave leaves HBM idle); null for none
  const void* pf0;
  long long pf0_bytes;
  const void* pf1;
  long long pf1_bytes;
  // e4m3 operands: one fp32 scale per weight row (indexed by global weight row) and per token
  // row of B (indexed by B row); alt_* for the alternate group
  const float* a_scale;
  const float* b_scale;
  const float* alt_a_scale;
  const float* alt_b_scale;
  // NVFP4 block-scale atoms (512 B each, 4 * kb_total per 128-row tile of A, per routed chunk
  // of B, per token chunk of the alternate group's B)
  const uint8_t* a_sf;
  const uint8_t* b_sf;
  const uint8_t* alt_a_sf;
  const uint8_t* alt_b_sf;
  // routed items that read their token rows straight from the unpermuted tokens (gather_src
  // non-null): B row j of a routed chunk is token gather_perm[b_row + j] / gather_k, its K slab
  // kb the 128 bytes at gather_src + token * gather_ld + 128 kb; the producer warp copies them
  // with cp.async (the alternate group keeps its TMA loads)
  const uint8_t* gather_src;
  const int* gather_perm;
  int gather_k;
  int gather_ld;
  int* err;
  const int* done;
};

struct GemmItem {
  int a_row, b_row, n, kb0, kb1, r_base, aux;
  int chunk;  // routed chunk, or token chunk of the alternate group (NVFP4 scale atoms of B)
  bool alt;
};

DG_DEV GemmItem gemm_item(const GemmParams& p, int it) {
  GemmItem w;
  w.alt = false;
  w.kb0 = 0;
  w.chunk = 0;
  if (p.chunks == nullptr) {
    const int mt = it % p.m_tiles;
    const int rest = it / p.m_tiles;
    const int split = rest % p.k_splits;
    const int nc = rest / p.k_splits;
    w.r_base = mt * 128;
    w.a_row = p.a_row_base + w.r_base;
    w.b_row = p.b_row_base + nc * p.n_chunk;
    w.n = min(p.n_chunk, p.n_total - nc * p.n_chunk);
    w.kb0 = split * p.kb_total / p.k_splits;
    w.kb1 = (split + 1) * p.kb_total / p.k_splits;
    w.aux = split;
  } else {
    const int sh_items = p.alt_group >= 0 ? p.alt_chunks * p.alt_m_tiles : 0;
    if (it < sh_items) {  // consecutive items share a weight tile, which L2 then serves
      const int m = it / p.alt_chunks, ch = it % p.alt_chunks;
      w.alt = true;
      w.r_base = m * 128;
      w.a_row = w.r_base;
      w.b_row = ch * p.n_chunk;
      w.n = min(p.n_chunk, p.alt_tokens - ch * p.n_chunk);
      w.kb1 = p.alt_kb_total;
      w.aux = p.alt_group;
      w.chunk = ch;
    } else {
      const int r = it - sh_items;
      const int ch = r / p.m_tiles, m = r % p.m_tiles;
      const int4 c = p.chunks[ch];
      w.r_base = m * 128;
      w.a_row = c.x * p.a_rows_per_group + w.r_base;
      w.b_row = c.y;
      w.n = c.z;
      w.kb1 = p.kb_total;
      w.aux = c.x;
      w.chunk = ch;
    }
  }
  return w;
}

DG_DEV int gemm_item_count(const GemmParams& p) {
  if (p.chunks == nullptr) return p.m_tiles * p.k_splits * p.n_chunks;
  const int sh_items = p.alt_group >= 0 ? p.alt_chunks * p.alt_m_tiles : 0;
  return sh_items + *reinterpret_cast<const volatile int*>(p.chunk_count) * p.m_tiles;
}

template <int MAXN, int STAGES, int FMT = 0>
struct GemmCfg {
  static constexpr int kABytes = 128 * 128;   // 128 rows x 128 B (64 bf16 / 128 e4m3 / 256 e2m1)
  static constexpr int kBBytes = MAXN * 128;  // MAXN rows x 128 B
  // NVFP4: the slab's four scale atoms for A, then for B (one per 128 rows of B)
  static constexpr int kSfaBytes = FMT == 2 ? 4 * 512 : 0;
  static constexpr int kSfbBytes = FMT == 2 ? 4 * 512 * ((MAXN + 127) / 128) : 0;
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  static constexpr int kAccBufs = MAXN <= 128 ? 4 : 2;  // TMEM accumulators in flight
  static constexpr int kAccCols = kAccBufs * MAXN;
  // NVFP4: per stage 16 TMEM columns of A scales and 16 per 128 rows of B after the accumulators
  static constexpr int kSfCols = FMT == 2 ? 16 + 16 * ((MAXN + 127) / 128) : 0;
  static constexpr int kTmemUsed = kAccCols + STAGES * kSfCols;
  static constexpr int kTmemCols = kTmemUsed <= 256 ? 256 : 512;
  static_assert(kTmemUsed <= 512, "TMEM");
  // epilogue warps: two per TMEM lane quarter for wide token tiles (they split the columns)
  static constexpr int kEpiWarps = MAXN >= 128 ? 8 : 4;
  // + the gather warps after the epilogue warps (idle unless the launch gathers token rows):
  // 16-byte units per gather thread and stage, at most MAXN rows x 8 units over their threads
  static constexpr int kGatherWarps = 4;
  static constexpr int kGatherPer = MAXN * 8 / (32 * kGatherWarps);
  static constexpr int kThreads = 64 + 32 * kEpiWarps + 32 * kGatherWarps;
  static constexpr int kSmemBytes = STAGES * kStageBytes + 1024 + 256;
  static_assert(MAXN % 32 == 0 && MAXN >= 32 && MAXN <= 256, "MAXN");
};

template <int EPI>
DG_DEV void gemm_epilogue_chunk(const GemmParams& p, const GemmItem& w, const float (&v)[32],
                                int c, int r, int dst_lane = 0, float scale_lane = 1.0f) {
  const int row = w.r_base + r;  // row inside the group (output feature / gate-up row)
  const int m_valid = w.alt ? p.alt_m_valid : p.m_valid;
  if constexpr (EPI == kEpiPartialF32) {
    if (row < m_valid) {
      float* o = p.out_f32 + static_cast<long long>(w.aux) * p.split_stride +
                 static_cast<long long>(w.b_row + c) * p.ld_out + row;
      const long long ld = p.ld_out;
      if (c + 32 <= w.n) {
#pragma unroll
        for (int i = 0; i < 32; ++i, o += ld) *o = v[i];
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i, o += ld)
          if (c + i < w.n) *o = v[i];
      }
    }
  } else if constexpr (EPI == kEpiGluBf16) {
    // rows come in (gate, up) pairs on adjacent lanes: lane 2u has gate unit u, 2u+1 up unit u
    const bool gate_lane = (lane_id() & 1) == 0;
    const int unit = row >> 1;
    const long long ld = w.alt ? p.alt_ld_out : p.ld_out;
    // gate lanes store tokens c..c+15, up lanes tokens c+16..c+31
    __nv_bfloat16* out = (w.alt ? p.alt_out_bf16 : p.out_bf16) +
                         static_cast<long long>(w.b_row + c + (gate_lane ? 0 : 16)) * ld + unit;
    const bool ok_row = row < m_valid;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, v[i], 1);
      if (((i >> 4) & 1) == (gate_lane ? 0 : 1)) {
        if (ok_row && c + i < w.n) {
          const float g = gate_lane ? v[i] : other;
          const float u = gate_lane ? other : v[i];
          *out = __float2bfloat16_rn(g / (1.0f + __expf(-g)) * u);
        }
        out += ld;
      }
    }
  } else {  // kEpiScatterF32
    if (row < m_valid) {
      if (w.alt) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c + i < w.n) p.alt_out_f32[static_cast<long long>(w.b_row + c + i) * p.alt_ld_out + row] = v[i];
      } else {
        // lane i of the warp holds the destination row and weight of token c + i
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int dst = __shfl_sync(0xffffffffu, dst_lane, i);
          const float s = __shfl_sync(0xffffffffu, scale_lane, i);
          if (c + i < w.n) p.out_f32[static_cast<long long>(dst) * p.ld_out + row] = v[i] * s;
        }
      }
    }
  }
}

template <int MAXN, int STAGES, int EPI, int FMT = 0>
__global__ void __launch_bounds__(GemmCfg<MAXN, STAGES, FMT>::kThreads, 1)
    gemm_swapab_kernel(const __grid_constant__ CUtensorMap tm_a,
                       const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_a2,
                       const __grid_constant__ CUtensorMap tm_b2, const GemmParams p) {
  using C = GemmCfg<MAXN, STAGES, FMT>;
  constexpr bool kScaled = FMT != 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + C::kAccBufs;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + C::kAccBufs);
  const int warp = threadIdx.x >> 5;
  // gathered token rows: every producer lane signals its copies on the stage's full barrier
  const bool gather = FMT != 2 && p.gather_src != nullptr;

  if (warp == 0 && lane_id() == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], gather ? 1 + 32 * C::kGatherWarps : 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 32 * C::kEpiWarps);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (p.alt_group >= 0) {
      tma_prefetch_desc(&tm_a2);
      tma_prefetch_desc(&tm_b2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // the setup above overlaps the previous kernel; from here on its results are needed
  pdl_enter();
  if (block_done(p.done)) {  // uniform over the grid: release TMEM and leave
    if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
    return;
  }
  const int n_items = gemm_item_count(p);

  if (warp == 0) {
    if (elect_one()) {
      const uint64_t pol_a = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // each item's descriptor is read one item ahead, so its load latency overlaps the copies
      GemmItem wn{};
      if (static_cast<int>(blockIdx.x) < n_items) wn = gemm_item(p, blockIdx.x);
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const GemmItem w = wn;
        if (it + static_cast<int>(gridDim.x) < n_items) wn = gemm_item(p, it + gridDim.x);
        const bool gat = gather && !w.alt;  // B rows come from the gather warp
        const int nbox = (w.n + 31) >> 5;
        const uint32_t bytes =
            C::kABytes + (gat ? 0 : nbox * 32 * 128) + C::kSfaBytes + C::kSfbBytes;
        const CUtensorMap* ta = w.alt ? &tm_a2 : &tm_a;
        const CUtensorMap* tb = w.alt ? &tm_b2 : &tm_b;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.err)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::kStageBytes;
          uint8_t* sb = sa + C::kABytes;
          mbar_arrive_expect_tx(&full[stage], bytes);
          const int kx = kb * (FMT != 0 ? 128 : 64);  // map columns per 128-byte slab
          tma_load_2d(ta, &full[stage], sa, kx, w.a_row, pol_a);
          if (!gat)
            for (int bx = 0; bx < nbox; ++bx)
              tma_load_2d(tb, &full[stage], sb + bx * 4096, kx, w.b_row + bx * 32, pol_b);
          if constexpr (FMT == 2) {
            // the slab's scale atoms: A by 128-row tile, B by chunk (4 per slab, padded)
            const int kt = w.alt ? p.alt_kb_total : p.kb_total;
            const uint8_t* fa = (w.alt ? p.alt_a_sf : p.a_sf) +
                                (static_cast<long long>(w.a_row >> 7) * 4 * kt + 4 * kb) * 512;
            const uint8_t* fb = (w.alt ? p.alt_b_sf : p.b_sf) +
                                (static_cast<long long>(w.chunk) * 4 * kt + 4 * kb) * 512 *
                                    ((MAXN + 127) / 128);
            bulk_load(sb + C::kBBytes, fa, C::kSfaBytes, &full[stage]);
            bulk_load(sb + C::kBBytes + C::kSfaBytes, fb, C::kSfbBytes, &full[stage]);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      prefetch_l2_slice(p.pf0, p.pf0_bytes, blockIdx.x, gridDim.x);
      prefetch_l2_slice(p.pf1, p.pf1_bytes, blockIdx.x, gridDim.x);
    }
  } else if (warp == 1) {
    if (elect_one()) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      GemmItem wn{};
      if (static_cast<int>(blockIdx.x) < n_items) wn = gemm_item(p, blockIdx.x);
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const GemmItem w = wn;
        if (it + static_cast<int>(gridDim.x) < n_items) wn = gemm_item(p, it + gridDim.x);
        const uint32_t idesc = FMT == 2   ? idesc_fp4_f32(128, (w.n + 15) & ~15)
                               : FMT == 1 ? idesc_e4m3_f32(128, (w.n + 15) & ~15)
                                          : idesc_bf16_f32(128, (w.n + 15) & ~15);
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * MAXN;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.err)) {
            ok = false;
            break;
          }
          // token rows written by the producer lanes' cp.async (generic proxy) before the UMMA
          // reads them through the async proxy
          if (gather) fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
          const uint64_t da = sdesc_sw128(sa);
          const uint64_t db = sdesc_sw128(sa + C::kABytes);
          if constexpr (FMT == 2) {
            // scale atoms into this stage's TMEM columns (in issue order before their MMAs)
            const uint32_t sfa = sa + C::kABytes + C::kBBytes;
            const uint32_t t_sf = tmem_base + C::kAccCols + stage * C::kSfCols;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              tmem_cp_32x128b_x4(t_sf + 4 * k, sdesc_rows16(sfa + 512 * k));
              tmem_cp_32x128b_x4(t_sf + 16 + 4 * k, sdesc_rows16(sfa + C::kSfaBytes + 512 * k));
            }
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_fp4(d_tmem, da + 2 * k, db + 2 * k, idesc, t_sf + 4 * k, t_sf + 16 + 4 * k,
                       (kb > w.kb0 || k > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if constexpr (FMT == 1)
                umma_e4m3(d_tmem, da + 2 * k, db + 2 * k, idesc, (kb > w.kb0 || k > 0) ? 1u : 0u);
              else
                umma_bf16(d_tmem, da + 2 * k, db + 2 * k, idesc, (kb > w.kb0 || k > 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        umma_commit(&acc_full[acc]);
        if (++acc == C::kAccBufs) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else if (warp >= 2 + C::kEpiWarps) {
    // the gather warps: with gathered token rows they fill B of every routed item's stages.
    // Gather thread g copies 16-byte units g, g + 128, ...: row j = unit / 8 of the item, its
    // piece u = unit % 8 landing at the swizzled 128-byte line of row j (destinations fixed for
    // the kernel, sources per item: token perm[b_row + j] / k, zero fill past the item's rows).
    // Every thread signals its copies on the stage's full barrier, for the alternate group's
    // stages too (none pending); like the TMA producer each warp first waits for the stage to
    // be free, which keeps the arrivals in step with the stage's uses.
    if (gather) {
      constexpr int kPer = C::kGatherPer;
      constexpr uint32_t kSkip = 0xffffffffu, kZero = 0xfffffffeu;
      const int lane = static_cast<int>(lane_id());
      const int gt = (warp - 2 - C::kEpiWarps) * 32 + lane;
      uint32_t dst_off[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int c = gt + 32 * C::kGatherWarps * i, row = c >> 3, u = c & 7;
        dst_off[i] = (row >> 3) * 1024 + (row & 7) * 128 + ((u ^ (row & 7)) << 4);
      }
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const GemmItem w = gemm_item(p, it);
        const bool gat = !w.alt;
        const int npad = (w.n + 15) & ~15;  // B rows the UMMA reads
        uint32_t src_off[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
          const int c = gt + 32 * C::kGatherWarps * i, row = c >> 3, u = c & 7;
          src_off[i] = !gat || row >= npad ? kSkip
                       : row >= w.n        ? kZero
                                           : static_cast<uint32_t>(__ldg(p.gather_perm + w.b_row + row) /
                                                                   p.gather_k) *
                                                     static_cast<uint32_t>(p.gather_ld) +
                                                 u * 16;
        }
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          int ready = 1;
          if (lane == 0) ready = mbar_wait(&empty[stage], phase ^ 1u, p.err) ? 1 : 0;
          if (!__shfl_sync(0xffffffffu, ready, 0)) {
            ok = false;
            break;
          }
          const uint32_t sbase = smem_u32(smem + stage * C::kStageBytes + C::kABytes);
          const uint8_t* src = p.gather_src + kb * 128;
#pragma unroll
          for (int i = 0; i < kPer; ++i)
            if (src_off[i] != kSkip) {
              const bool real = src_off[i] != kZero;
              cp_async_16(sbase + dst_off[i], real ? src + src_off[i] : p.gather_src, real ? 16u : 0u);
            }
          cp_async_mbar_arrive(&full[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane_id();
    constexpr int kGroups = C::kEpiWarps / 4;  // warps sharing a lane quarter split the chunks
    const int grp = (warp - 2) >> 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    // descriptor one item ahead; the item's row data below are independent loads indexed by its
    // B rows, issued before the accumulator wait
    GemmItem wn{};
    if (static_cast<int>(blockIdx.x) < n_items) wn = gemm_item(p, blockIdx.x);
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
      const GemmItem w = wn;
      if (it + static_cast<int>(gridDim.x) < n_items) wn = gemm_item(p, it + gridDim.x);
      // scatter: this lane's token of each 32-wide chunk, loaded before the accumulator is ready
      int dst_lane[MAXN / 32];
      float scale_lane[MAXN / 32];
      if constexpr (EPI == kEpiScatterF32) {
#pragma unroll
        for (int cc = 0; cc < MAXN / 32; ++cc) {
          const int j = cc * 32 + lane_id();
          dst_lane[cc] = 0;
          scale_lane[cc] = 1.0f;
          if (!w.alt && j < w.n) {
            dst_lane[cc] = p.perm ? p.perm[w.b_row + j] : w.b_row + j;
            scale_lane[cc] = p.scale ? p.scale[w.b_row + j] : 1.0f;
          }
        }
      }
      // e4m3 / NVFP4: this lane's weight-row scale and token scales, loaded before the
      // accumulator is ready
      float row_scale = 1.0f;
      float tok_scale[MAXN / 32];
      if constexpr (kScaled) {
        const float* as = w.alt ? p.alt_a_scale : p.a_scale;
        const float* bs = w.alt ? p.alt_b_scale : p.b_scale;
        const int m_valid = w.alt ? p.alt_m_valid : p.m_valid;
        row_scale = (w.r_base + r < m_valid) ? as[w.a_row + r] : 0.0f;
#pragma unroll
        for (int cc = 0; cc < MAXN / 32; ++cc) {
          const int j = cc * 32 + lane_id();
          tok_scale[cc] = j < w.n ? bs[gather && !w.alt ? __ldcg(p.gather_perm + w.b_row + j) / p.gather_k
                                                      : w.b_row + j]
                                  : 0.0f;
        }
      }
      if (!mbar_wait(&acc_full[acc], acc_phase, p.err)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + acc * MAXN + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int cc = 0; cc < MAXN / 32; ++cc) {
        const int c = cc * 32;
        if (cc % kGroups == grp && c < w.n) {
          float v[32];
          tmem_ld32(t_row + c, v);
          if constexpr (kScaled) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              v[i] *= row_scale * __shfl_sync(0xffffffffu, tok_scale[cc], i);
          }
          if constexpr (EPI == kEpiScatterF32)
            gemm_epilogue_chunk<EPI>(p, w, v, c, r, dst_lane[cc], scale_lane[cc]);
          else
            gemm_epilogue_chunk<EPI>(p, w, v, c, r);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if (++acc == C::kAccBufs) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
struct LmHeadParams {
  int n_tokens;   // valid token rows of this launch (<= 256), starting at token row tok_base
  int tok_base;   // first token row (tm_x row, partial / logits row) of this launch
  int n_vtiles;   // vocab / 256
  int kb_total;   // d / 64
  StatPartial* partials;  // [n_tokens, n_vtiles]
  float* logits;          // debug: [n_tokens, vocab] when not null (statistics skipped)
  int vocab;
  float inv_t;            // 1 / sampling temperature: statistics of logits / T
  // e4m3 head (kF8): per-row scales of the token codes [n_tokens] and of the vocabulary rows [V]
  const float* x_scale;
  const float* e_scale;
  int* err;
  const int* done;
};

constexpr int kLmStages = 3;
constexpr int kLmStageBytes = 2 * 16384 + 32768;  // two token tiles + one 256-row vocab tile
constexpr int kLmSmemBytes = kLmStages * kLmStageBytes + 1024 + 256;

constexpr int kLmThreads = 64 + 32 * 8;  // TMA, MMA, two epilogue warpgroups (one per token tile)

// kF8: tokens and vocabulary rows are e4m3 codes (kind::f8f6f4; a 128-byte K slab holds 128
// codes, so the ring and descriptors are unchanged) and every accumulator is scaled by its
// token's and its vocabulary row's scale before the statistics (or the debug logits).
template <bool kStats, bool kF8 = false>
__global__ void __launch_bounds__(kLmThreads, 1)
    lmhead_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_e,
                  const LmHeadParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kLmStages * kLmStageBytes);
  uint64_t* empty = full + kLmStages;
  uint64_t* acc_full = empty + kLmStages;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 1);
  const int warp = threadIdx.x >> 5;
  const int n_ttiles = (p.n_tokens + 127) >> 7;

  if (warp == 0 && lane_id() == 0) {
    for (int s = 0; s < kLmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 256);
    fence_barrier_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_e);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // the setup above overlaps the previous kernel; from here on its results are needed
  pdl_enter();
  if (block_done(p.done)) {  // uniform over the grid: release TMEM and leave
    if (warp == 1) tmem_dealloc(tmem_base, 512);
    return;
  }

  if (warp == 0) {
    if (elect_one()) {
      const uint64_t pol_x = policy_evict_last();
      const uint64_t pol_e = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int vt = blockIdx.x; vt < p.n_vtiles && ok; vt += gridDim.x) {
        for (int kb = 0; kb < p.kb_total; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.err)) {
            ok = false;
            break;
          }
          uint8_t* s0 = smem + stage * kLmStageBytes;
          mbar_arrive_expect_tx(&full[stage], n_ttiles * 16384 + 32768);
          const int kx = kb * (kF8 ? 128 : 64);  // elements per 128-byte K slab
          for (int tt = 0; tt < n_ttiles; ++tt)
            tma_load_2d(&tm_x, &full[stage], s0 + tt * 16384, kx, p.tok_base + tt * 128, pol_x);
          tma_load_2d(&tm_e, &full[stage], s0 + 32768, kx, vt * 256, pol_e);
          if (++stage == kLmStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      const uint32_t idesc = kF8 ? idesc_e4m3_f32(128, 256) : idesc_bf16_f32(128, 256);
      bool ok = true;
      for (int vt = blockIdx.x; vt < p.n_vtiles && ok; vt += gridDim.x) {
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, p.err)) break;
        tc_fence_after();
        for (int kb = 0; kb < p.kb_total; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t s0 = smem_u32(smem + stage * kLmStageBytes);
          const uint64_t de = sdesc_sw128(s0 + 32768);
          for (int tt = 0; tt < n_ttiles; ++tt) {
            const uint64_t dx = sdesc_sw128(s0 + tt * 16384);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if constexpr (kF8)
                umma_e4m3(tmem_base + tt * 256, dx + 2 * k, de + 2 * k, idesc,
                          (kb > 0 || k > 0) ? 1u : 0u);
              else
                umma_bf16(tmem_base + tt * 256, dx + 2 * k, de + 2 * k, idesc,
                          (kb > 0 || k > 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == kLmStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        umma_commit(acc_full);
        acc_phase ^= 1u;
      }
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane_id();
    const int tt = (warp - 2) >> 2;  // token tile of this epilogue warpgroup
    uint32_t acc_phase = 0;
    for (int vt = blockIdx.x; vt < p.n_vtiles; vt += gridDim.x) {
      if (!mbar_wait(acc_full, acc_phase, p.err)) break;
      tc_fence_after();
      if (tt < n_ttiles) {
        const int tok = tt * 128 + r;
        const uint32_t t_row = tmem_base + tt * 256 + (static_cast<uint32_t>(q * 32) << 16);
        // e4m3: accumulator (tok, column c) x x_scale[tok] x e_scale[vocab row of c]
        const float xs = kF8 ? (tok < p.n_tokens ? p.x_scale[p.tok_base + tok] : 0.f) : 1.f;
        const float* es = kF8 ? p.e_scale + vt * 256 : nullptr;
        auto scale32 = [&](float (&v)[32], int c) {
          if constexpr (kF8) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 e4 = __ldg(reinterpret_cast<const float4*>(es + c + i));
              v[i] *= xs * e4.x;
              v[i + 1] *= xs * e4.y;
              v[i + 2] *= xs * e4.z;
              v[i + 3] *= xs * e4.w;
            }
          }
        };
        if constexpr (kStats) {
          float m = -INFINITY;
          int a = 0;
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            float v[32];
            tmem_ld32(t_row + c, v);
            scale32(v, c);
            // tree argmax of the chunk, lowest index on equal values
            int idx[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) idx[i] = i;
#pragma unroll
            for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
              for (int i = 0; i < w; ++i) {
                const bool take = v[i + w] > v[i] || (v[i + w] == v[i] && idx[i + w] < idx[i]);
                v[i] = take ? v[i + w] : v[i];
                idx[i] = take ? idx[i + w] : idx[i];
              }
            if (v[0] > m) {  // strict: an earlier chunk keeps equal maxima
              m = v[0];
              a = c + idx[0];
            }
          }
          float s4[4] = {0.f, 0.f, 0.f, 0.f}, u4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            float v[32];
            tmem_ld32(t_row + c, v);
            scale32(v, c);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float d = (v[i] - m) * p.inv_t;
              const float e = __expf(d);
              s4[i & 3] += e;
              u4[i & 3] = fmaf(e, d, u4[i & 3]);
            }
          }
          const float s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
          const float u = (u4[0] + u4[1]) + (u4[2] + u4[3]);
          if (tok < p.n_tokens)
            p.partials[static_cast<long long>(p.tok_base + tok) * p.n_vtiles + vt] =
                StatPartial{m * p.inv_t, s, u, vt * 256 + a};
        } else {
          for (int c = 0; c < 256; c += 32) {
            float v[32];
            tmem_ld32(t_row + c, v);
            scale32(v, c);
            if (tok < p.n_tokens) {
              float4* dst = reinterpret_cast<float4*>(
                  p.logits + static_cast<long long>(p.tok_base + tok) * p.vocab + vt * 256 + c);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
      acc_phase ^= 1u;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace dg
