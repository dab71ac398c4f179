// fp8.cuh -- e4m3 quantisation for the FP8 expert format.
//
// The model ships as BF16, FP8 or NVFP4 weights (jakiprompt.pl, "Diffusion Gemma – nowy model
// językowy Google", section "Wymagania sprzętowe"); the pages give no scheme, so the plainest symmetric
// one is used.  A row v (an output row of an expert weight matrix, or one token's activation row
// where it enters an expert GEMM) gets one fp32 scale s = max|v| / 448 and e4m3 codes
// rn_satfinite(v / s) (IEEE division, round to nearest even, clamp to +-448); an all-zero row
// has s = 0 and zero codes.  The expert GEMMs multiply codes (tcgen05 kind::f8f6f4, fp32
// accumulation) and scale the sums by (weight row scale) x (token scale) in their epilogues.
//
// quant_rows_kernel quantises up to two segments of bf16 rows, one warp per row.  Segment rows
// may be gathered (row p reads source row perm[p] / top_k), which turns the routed-token gather
// of the grouped GEMMs into a gather + quantise with the same launch; the second segment then
// quantises the unpermuted tokens for the shared expert.
#pragma once
#include <cuda_fp8.h>

#include "dg_common.cuh"
#include "layer.cuh"

namespace dg {

struct QuantSeg {
  const __nv_bfloat16* src;
  long long ld_src;     // elements between source rows
  const int32_t* perm;  // null: row p reads source row p; else source row perm[p] / top_k
  int top_k;
  const float* wsrc;    // with perm: wdst[p] = wsrc[perm[p]] (route weights in permuted order)
  float* wdst;
  int rows, cols;       // cols % 16 == 0
  uint8_t* dst;
  long long ld_dst;     // bytes between destination rows (multiple of 16); [cols, ld_dst) = 0
  float* scale;         // one per destination row
};

struct QuantJob {
  QuantSeg seg[2];
  int n_seg;
  ExpertPrefetch pf;  // expert weights of the first routed chunks, hinted into L2 (optional)
};

DG_DEV float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
DG_DEV float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// One warp quantises one row of `cols` bf16 values (16-byte vectors, cols % 8 == 0) into a
// destination row of `pitch` bytes (pitch % 8 == 0), zero past the codes.
DG_DEV void quant_row_warp(const __nv_bfloat16* __restrict__ src, int cols, int pitch,
                           uint8_t* __restrict__ dst, float* __restrict__ scale) {
  const int lane = lane_id();
  const int nv = cols >> 3;
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  float amax = 0.f;
  for (int i = lane; i < nv; i += 32) {
    const uint4 u = s4[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, kE4m3Max);
  if (lane == 0) *scale = s;
  uint2* d2 = reinterpret_cast<uint2*>(dst);
  for (int i = lane; i < nv; i += 32) {
    const uint4 u = s4[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t p[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      p[j] = s > 0.f ? e4m3x2(__fdiv_rn(bf16_lo(w[j]), s), __fdiv_rn(bf16_hi(w[j]), s)) : 0u;
    d2[i] = make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
  }
  for (int i = nv + lane; i < (pitch >> 3); i += 32) d2[i] = make_uint2(0u, 0u);
}

__global__ void __launch_bounds__(256) quant_rows_kernel(const QuantJob job, const int* done) {
  pdl_enter();
  if (block_done(done)) return;
  const ExpertPrefetch& pf = job.pf;
  if (threadIdx.x == 0 && pf.w != nullptr && pf.n_first > 0) {
    const int nf = min(pf.n_first, *pf.n_chunks);
    if (nf > 0 && static_cast<int>(gridDim.x) >= nf) {
      const int c = blockIdx.x % nf, parts = gridDim.x / nf, part = blockIdx.x / nf;
      if (part < parts)
        prefetch_l2_slice(static_cast<const uint8_t*>(pf.w) + pf.chunks[c].x * pf.expert_bytes,
                          pf.expert_bytes, part, parts);
    }
  }
  int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  for (int sg = 0; sg < job.n_seg; ++sg) {
    const QuantSeg& q = job.seg[sg];
    if (row < q.rows) {
      int sr = row;
      if (q.perm) {
        const int slot = q.perm[row];
        if (lane_id() == 0 && q.wdst) q.wdst[row] = q.wsrc[slot];
        sr = slot / q.top_k;
      }
      quant_row_warp(q.src + static_cast<long long>(sr) * q.ld_src, q.cols,
                     static_cast<int>(q.ld_dst), q.dst + static_cast<long long>(row) * q.ld_dst,
                     q.scale + row);
      return;
    }
    row -= q.rows;
  }
}

}  // namespace dg
