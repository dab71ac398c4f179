// fp4.cuh -- NVFP4 quantisation for the 4-bit expert format.
//
// The model ships as BF16, FP8 or NVFP4 weights (jakiprompt.pl, "Diffusion Gemma – nowy model
// językowy Google", section "Wymagania sprzętowe") and runs NVFP4 kernels on Blackwell
// (aitoday.skyai.vn, "Bắt đầu ngay hôm nay"); the pages give no arithmetic, so the plainest
// reading is used.  A row v (an expert weight row, or one token's activation row where it enters
// an expert GEMM) of K values gets:
//   g    = max|v| / (6 * 448)                          fp32 row scale (IEEE division)
//   s_b  = e4m3_rn_satfinite((max|block| / 6) / g)     one per 16 consecutive values along K
//   code = e2m1_rn_satfinite(v / (s_b * g))            4-bit codes, two per byte (low nibble first)
// so that v ~= code * s_b * g; a zero row has g = 0, a block whose scale rounds to 0 has zero codes.
//
// Storage, chosen for tcgen05.mma kind::mxf4nvf4.block_scale.block16:
//   codes   rows of K / 2 bytes at a pitch of round_up(K / 2, 128) bytes (128-byte K slabs);
//   scales  512-byte atoms, one per (128-row tile, 64-wide K group): 128 rows x 4 blocks, byte
//           (r mod 32) * 16 + (r div 32) * 4 + block -- the order tcgen05.cp.32x128b.warpx4
//           moves into the four TMEM columns one MMA reads.  Atoms of a tile are consecutive
//           along K, so one 128-byte code slab (K = 256) has its four scale atoms in 2 KB; a
//           tile holds 4 * ceil(K / 256) atoms (the ones past K / 64 are zero), so the last
//           slab's 2 KB never reaches into the next tile.
//   Weight rows tile by 128 from row 0; token rows tile by routed chunk (a chunk's rows are
//   rows 0.. of its own atoms), see QuantFp4Seg.
#pragma once
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "dg_common.cuh"
#include "fp8.cuh"
#include "layer.cuh"

namespace dg {

constexpr float kE2m1Max = 6.0f;
constexpr int kFp4Block = 16;
constexpr int kSfAtomBytes = 512;

// Byte of the scale of (row r of a 128-row tile, 16-wide block b of a 64-wide K group) in its atom.
DG_DEV int sf_atom_byte(int r, int b) { return (r & 31) * 16 + (r >> 5) * 4 + b; }

// Two e2m1 codes in one byte, `a` in the low nibble.
DG_DEV uint32_t e2m1x2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp4x2(make_float2(a, b), __NV_E2M1,
                                                       cudaRoundNearest));
}

// e4m3 code of a non-negative value (round to nearest even, saturating) and its value.
DG_DEV float e4m3_round(float t, uint8_t* code) {
  const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3);
  *code = static_cast<uint8_t>(c);
  const __half_raw h = __nv_cvt_fp8_to_halfraw(c, __NV_E4M3);
  return __half2float(__half(h));
}

// Where the scale atoms of one row go: atom (tile, K group) at sf + (tile * n_groups + group) * 512.
struct Fp4RowDst {
  uint8_t* codes;  // this row's codes
  uint8_t* sf;     // the row's tile's first atom
  int r;           // row inside the tile (0..127)
};

// One warp quantises one row of `cols` bf16 values (cols % 64 == 0) to NVFP4.
DG_DEV void nvfp4_row_warp(const __nv_bfloat16* __restrict__ src, int cols, const Fp4RowDst& d,
                           float* __restrict__ row_scale) {
  const int lane = lane_id();
  const int nb = cols / kFp4Block;
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  float amax = 0.f;
  for (int i = lane; i < cols / 8; i += 32) {
    const uint4 u = s4[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[j] << 16)),
                               fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float g = __fdiv_rn(amax, kE2m1Max * kE4m3Max);
  if (lane == 0) *row_scale = g;
  for (int b = lane; b < nb; b += 32) {
    float v[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 u = s4[2 * b + h];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * h + 2 * j] = __uint_as_float(w[j] << 16);
        v[8 * h + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    }
    float bmax = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(v[j]));
    uint8_t sc = 0;
    float step = 0.f;
    if (g > 0.f) {
      const float t = __fdiv_rn(__fdiv_rn(bmax, kE2m1Max), g);
      step = __fmul_rn(e4m3_round(t, &sc), g);
    }
    uint32_t p[2] = {0u, 0u};
    if (step > 0.f) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t byte = e2m1x2(__fdiv_rn(v[2 * j], step), __fdiv_rn(v[2 * j + 1], step));
        p[j >> 2] |= byte << (8 * (j & 3));
      }
    }
    *reinterpret_cast<uint2*>(d.codes + 8 * b) = make_uint2(p[0], p[1]);
    d.sf[(b >> 2) * kSfAtomBytes + sf_atom_byte(d.r, b & 3)] = sc;
  }
}

// One segment of rows to quantise.  Weight-like rows (chunks == nullptr) tile by tile_rows
// (<= 128) from row 0; routed rows (chunks != nullptr, row p = permuted slot p reading token
// perm[p] / top_k) tile by routed chunk: row p of chunk c (chunks[c].y <= p < chunks[c].y +
// chunks[c].z, at most 128 rows) is row p - chunks[c].y of chunk c's atoms.  Atom rows that no
// row fills are never initialised: they scale B rows beyond an item's tokens, whose products
// land in accumulator columns the epilogue does not read.
struct QuantFp4Seg {
  const __nv_bfloat16* src;
  long long ld_src;       // elements between source rows
  const int32_t* perm;    // optional gather: row p reads source row perm[p] / top_k
  int top_k;
  const float* wsrc;      // with perm: wdst[p] = wsrc[perm[p]]
  float* wdst;
  int rows, cols;         // cols % 64 == 0
  uint8_t* codes;
  long long pitch;        // bytes between code rows (multiple of 16)
  uint8_t* sf;            // scale atoms
  float* row_scale;       // one per row
  const int4* chunks;     // routed chunk list (device-built) or null
  const int* n_chunks;
  int tile_rows;          // rows per atom tile when chunks == null: 128 for weights, the token
                          // chunk width (<= 128) for the shared expert's tokens
};

struct QuantFp4Job {
  QuantFp4Seg seg[2];
  int n_seg;
  ExpertPrefetch pf;
};

// The routed chunk holding permuted row p: the last chunk whose first row is <= p.
DG_DEV int chunk_of_row(const int4* chunks, int n, int p) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (chunks[mid].y <= p) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(256) quant_fp4_rows_kernel(const QuantFp4Job job,
                                                             const int* done) {
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
    const QuantFp4Seg& q = job.seg[sg];
    if (row < q.rows) {
      int sr = row;
      if (q.perm) {
        const int slot = q.perm[row];
        if (lane_id() == 0 && q.wdst) q.wdst[row] = q.wsrc[slot];
        sr = slot / q.top_k;
      }
      const int groups = 4 * ((q.cols + 255) / 256);  // atoms per tile, padded to whole slabs
      int tile, r;
      if (q.chunks) {
        const int c = chunk_of_row(q.chunks, *q.n_chunks, row);
        tile = c;
        r = row - q.chunks[c].y;
      } else {
        tile = row / q.tile_rows;
        r = row % q.tile_rows;
      }
      Fp4RowDst d;
      d.codes = q.codes + static_cast<long long>(row) * q.pitch;
      d.sf = q.sf + static_cast<long long>(tile) * groups * kSfAtomBytes;
      d.r = r;
      nvfp4_row_warp(q.src + static_cast<long long>(sr) * q.ld_src, q.cols, d,
                     q.row_scale + row);
      if (lane_id() == 0) {
        // zero the code pad past K / 2 bytes (never read by the kernels; kept deterministic)
        for (long long b = q.cols / 2; b < q.pitch; b += 16)
          *reinterpret_cast<uint4*>(d.codes + b) = make_uint4(0u, 0u, 0u, 0u);
      }
      return;
    }
    row -= q.rows;
  }
}

}  // namespace dg
