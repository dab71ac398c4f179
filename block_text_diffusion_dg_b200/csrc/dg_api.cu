// dg_api.cu -- the C ABI of libdg: argument checks, workspace planning, TMA descriptors and
// the launch sequences of the denoise step, the sampler, prefill/commit and the standalone
// operators.  Kernels live in the *.cuh files included below; nothing here computes.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/dg.h"
#include "attention.cuh"
#include "dg_common.cuh"
#include "fp32_path.cuh"
#include "fp4.cuh"
#include "fp8.cuh"
#include "gemm.cuh"
#include "gemm_cluster.cuh"
#include "layer.cuh"
#include "sampler.cuh"

using namespace dg;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

#define DG_CUDA(call)                                                                        \
  do {                                                                                       \
    cudaError_t e_ = (call);                                                                 \
    if (e_ != cudaSuccess)                                                                   \
      return fail(DG_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_),       \
                  __FILE__, __LINE__);                                                       \
  } while (0)

std::atomic<uint64_t> g_launches{0};

// Optional per-kernel event hook (dg_profile_kernel).
struct ProfileHook {
  int kind = -1;
  std::vector<cudaEvent_t> events;
  int n_pairs = 0;
  int recorded = 0;
} g_prof;

inline void prof_before(int kind, cudaStream_t st) {
  if (g_prof.kind == kind && g_prof.recorded < g_prof.n_pairs)
    cudaEventRecord(g_prof.events[2 * g_prof.recorded], st);
}
inline void prof_after(int kind, cudaStream_t st) {
  if (g_prof.kind == kind && g_prof.recorded < g_prof.n_pairs) {
    cudaEventRecord(g_prof.events[2 * g_prof.recorded + 1], st);
    ++g_prof.recorded;
  }
}

#define DG_LAUNCHED()                                                                        \
  do {                                                                                       \
    cudaError_t e_ = cudaGetLastError();                                                     \
    if (e_ != cudaSuccess)                                                                   \
      return fail(DG_ERR_CUDA, "launch failed: %s (%s:%d)", cudaGetErrorString(e_), __FILE__, \
                  __LINE__);                                                                 \
    g_launches.fetch_add(1, std::memory_order_relaxed);                                      \
  } while (0)

#define DG_TRY(expr)        \
  do {                      \
    int rc_ = (expr);       \
    if (rc_ != DG_OK) return rc_; \
  } while (0)

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline int cdiv(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }
// Row pitch (bytes) of an e4m3 matrix with `cols` codes per row (DG_E4M3_PITCH).
inline int e4m3_pitch(int cols) { return (cols + 127) / 128 * 128; }
constexpr int kMaxBatch = 16;  // sequences of a batched context

// ---- TMA descriptor encoding through the driver entry point ---------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Matrix [rows, cols] of bf16 (elem 2) or e4m3 codes (elem 1) with row pitch `pitch` elements;
// box = one 128-byte row segment (64 bf16 or 128 codes) x box_rows, 128-byte swizzle (the
// layout the UMMA descriptors expect).  Columns past `cols` read as zero.
int make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch,
              uint32_t box_rows, int elem = 2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0 || (pitch * elem) % 16 != 0)
    return fail(DG_ERR_INVALID_ARG, "TMA operand not 16-byte aligned (base %p, pitch %llu)", base,
                (unsigned long long)pitch);
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch * elem};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, elem == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) rows=%llu cols=%llu box=%u",
                static_cast<int>(r), (unsigned long long)rows, (unsigned long long)cols, box_rows);
  return DG_OK;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// Resident 256-thread CTAs of a kernel on the whole GPU (its persistent grid size).
template <typename K>
int resident_ctas(K kernel) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  return per_sm * num_sms();
}

template <typename K>
int set_smem(K kernel, int bytes) {
  DG_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  return DG_OK;
}

// Every kernel goes through cudaLaunchKernelEx with programmatic stream serialisation: the next
// kernel in the stream may begin launching while this one drains; each kernel's first act is
// griddepcontrol.wait, so it still sees all of its predecessor's writes.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
               Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return fail(DG_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
  return DG_OK;
}

// launch_pdl with thread-block clusters of the given dimensions.
template <typename... KArgs, typename... Args>
int launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, dim3 cluster, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster.x;
  attr[1].val.clusterDim.y = cluster.y;
  attr[1].val.clusterDim.z = cluster.z;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return fail(DG_ERR_CUDA, "cluster launch failed: %s", cudaGetErrorString(e));
  return DG_OK;
}

// ---- GEMM launch helpers -----------------------------------------------------------------
constexpr int kGroupN = 64, kGroupStages = 8;
// Passes that give each expert many tokens (a batch of canvases, a prompt encoded at once) take
// wider token chunks, so each expert weight tile streams once per 128 or 256 tokens instead of
// once per 64: from 48 slots per expert on average a good part of the experts would otherwise
// need a second 64-token chunk (a second pass over their weights).  The 128-token instance keeps
// six stages in flight; the 256-token one, for prompt passes, four.
constexpr int kGroupMidN = 128, kGroupMidStages = 6;
constexpr int kGroupWideN = 256, kGroupWideStages = 4;
int group_chunk(long long n_slots, int n_experts) {
  if (n_slots < 48ll * n_experts) return kGroupN;
  return n_slots < 160ll * n_experts ? kGroupMidN : kGroupWideN;
}
constexpr int kRouterChunk = 64;  // tokens per router cluster
constexpr int kPrefetchExperts = 4;  // routed chunks whose expert weights the gather prefetches
// Decode layers: routed experts whose gate/up weights the router's CTAs that do not route hint into
// L2 (about 48 MB in bf16) while HBM is idle; 8 or 10 slowed the router more than they saved.
constexpr int kRouterPrefetchExperts = 6;

// ta2/tb2 are read only by items of the alternate group (p.alt_group >= 0).
template <int MAXN, int STAGES, int EPI, int FMT = 0>
int launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, int grid,
                cudaStream_t st, int kind = -1, const CUtensorMap* ta2 = nullptr,
                const CUtensorMap* tb2 = nullptr) {
  auto k = gemm_swapab_kernel<MAXN, STAGES, EPI, FMT>;
  constexpr int smem = GemmCfg<MAXN, STAGES, FMT>::kSmemBytes;
  if (p.alt_group >= 0 && (!ta2 || !tb2))
    return fail(DG_ERR_INVALID_ARG, "alternate group without its tensor maps");
  DG_TRY(set_smem(k, smem));
  prof_before(kind, st);
  DG_TRY(launch_pdl(k, dim3(grid), dim3(GemmCfg<MAXN, STAGES, FMT>::kThreads), smem, st, ta, tb,
                    ta2 ? *ta2 : ta, tb2 ? *tb2 : tb, p));
  DG_LAUNCHED();
  prof_after(kind, st);
  return DG_OK;
}

// Split-K projection with the K splits of each tile in one cluster: grid m_tiles x n_chunks x S.
template <int EPI>
int launch_cluster(const CUtensorMap& ta, const CUtensorMap& tb, const CluParams& p,
                   cudaStream_t st, int kind) {
  auto k = gemm_cluster_kernel<EPI>;
  DG_TRY(set_smem(k, kCluSmemBytes));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(p.m_tiles * p.n_chunks * p.splits);
  cfg.blockDim = dim3(kCluThreads);
  cfg.dynamicSmemBytes = kCluSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = p.splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  prof_before(kind, st);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, ta, tb, p);
  if (e != cudaSuccess) return fail(DG_ERR_CUDA, "cluster launch failed: %s", cudaGetErrorString(e));
  DG_LAUNCHED();
  prof_after(kind, st);
  return DG_OK;
}

// Shape part of the cluster projection parameters: `m_rows` weight rows, `n` tokens, K = 64 kb.
CluParams clu_params(int m_rows, int n, int kb, int splits, int* err, const int* done,
                     int chunk_n = 256) {
  CluParams p{};
  p.n_tokens = n;
  p.chunk_n = chunk_n;
  p.n_chunks = cdiv(n, chunk_n);
  p.m_tiles = cdiv(m_rows, 128);
  p.m_rows = m_rows;
  p.kb_total = kb;
  p.splits = std::max(1, std::min(splits, kb));
  p.err = err;
  p.done = done;
  return p;
}

// Cluster size (K splits) of a split-K projection with `tiles` weight x token tiles: enough CTAs
// to cover the SMs, at most kCluMaxSplits and at most one 64-wide K slab per split.
int clu_splits(int tiles, int kb_total, int sms) {
  return std::max(1, std::min({kCluMaxSplits, kb_total, sms / std::max(1, tiles)}));
}

// Grouped expert GEMM with the token-chunk width the pass needs (see group_chunk).  NVFP4 runs
// the 64-token instance only (its scale atoms are laid out per chunk of at most 128 rows).
constexpr int kGroupFp4Stages = 7;
template <int EPI, int FMT>
int launch_grouped(int nch, const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                   int sms, cudaStream_t st, int kind, const CUtensorMap* ta2,
                   const CUtensorMap* tb2) {
  if constexpr (FMT == 2) {
    return launch_gemm<kGroupN, kGroupFp4Stages, EPI, FMT>(ta, tb, p, sms, st, kind, ta2, tb2);
  } else {
    if (nch == kGroupWideN)
      return launch_gemm<kGroupWideN, kGroupWideStages, EPI, FMT>(ta, tb, p, sms, st, kind, ta2,
                                                                 tb2);
    if (nch == kGroupMidN)
      return launch_gemm<kGroupMidN, kGroupMidStages, EPI, FMT>(ta, tb, p, sms, st, kind, ta2,
                                                               tb2);
    return launch_gemm<kGroupN, kGroupStages, EPI, FMT>(ta, tb, p, sms, st, kind, ta2, tb2);
  }
}

// The expert half of an MoE pass once the routing exists: gather the routed token rows (bf16),
// or gather and quantise them (e4m3, together with the unpermuted tokens for the shared
// expert); grouped gate/up GEMM with the SiLU-GLU epilogue; e4m3: quantise h per slot and the
// shared h per token; grouped down GEMM with the weighted scatter.  The shared expert rides
// along in both GEMMs as the alternate group.
struct ExpertPass {
  int n, d, k, E, hid, hs;
  int fmt;                  // expert operands: 0 bf16, 1 e4m3, 2 NVFP4
  const int32_t* perm;
  const float* topk_w;
  float* w_perm;            // [n k]: topk_w in permuted order (written by the gather)
  const int4* chunks;
  const int* n_chunks;
  const __nv_bfloat16* xn;  // normed tokens [n, d]
  void* x_perm;             // routed rows [n k, d]: bf16, or e4m3 / e2m1 codes
  float* x_perm_scale;      // e4m3 / NVFP4: row scales [n k]
  void* x_sh;               // e4m3 / NVFP4: quantised tokens [n, d] for the shared expert
  float* x_sh_scale;
  __nv_bfloat16* h;         // SiLU-GLU output per slot [n k, hid]
  __nv_bfloat16* h_sh;      // shared expert's [n, hs]
  void* hq;                 // e4m3 / NVFP4: codes of h, h_sh and their row scales
  float* hq_scale;
  void* hsq;
  float* hsq_scale;
  uint8_t *x_sf, *x_sh_sf, *h_sf, *hs_sf;  // NVFP4: block-scale atoms of the token operands
  float* y_slot;
  float* y_shared;
  const void* w_gu;  // routed gate/up weights: the first chunks' experts are hinted into L2
  const void* ws_d;  // shared down weights: hinted into L2 by the gate/up GEMM's tail
  const float *w_gu_scale, *w_d_scale, *ws_gu_scale, *ws_d_scale;
  const uint8_t *w_gu_sf, *w_d_sf, *ws_gu_sf, *ws_d_sf;  // NVFP4: weight block-scale atoms
  const CUtensorMap *tm_wgu, *tm_xperm, *tm_wsgu, *tm_xsh, *tm_wd, *tm_h, *tm_wsd, *tm_hs;
  const void* pf0;  // hinted into L2 by the down GEMM's tail
  long long pf0_bytes;
  const void* pf1;
  long long pf1_bytes;
  int* err;
  const int* done;
  bool profile;  // record under the per-kernel profiling kinds
  bool x_sh_ready;  // e4m3: x_sh already holds the codes of xn (written by the ffn norm)
};

// Bytes of one operand row of `cols` values in expert format fmt: bf16 rows are packed, e4m3 and
// NVFP4 code rows are padded to 128-byte multiples.
long long operand_row_bytes(int fmt, int cols) {
  return fmt == 2 ? e4m3_pitch(cols / 2) : fmt == 1 ? e4m3_pitch(cols) : 2ll * cols;
}

// The routed chunk width of a pass: 256-token chunks for long passes, except NVFP4 (64 always).
int route_chunk(int fmt, long long n_slots, int n_experts) {
  return fmt != 2 ? group_chunk(n_slots, n_experts) : kGroupN;
}

template <int EPI>
int launch_grouped_fmt(int fmt, int nch, const CUtensorMap& ta, const CUtensorMap& tb,
                       const GemmParams& p, int sms, cudaStream_t st, int kind,
                       const CUtensorMap* ta2, const CUtensorMap* tb2) {
  if (fmt == 2) return launch_grouped<EPI, 2>(nch, ta, tb, p, sms, st, kind, ta2, tb2);
  if (fmt == 1) return launch_grouped<EPI, 1>(nch, ta, tb, p, sms, st, kind, ta2, tb2);
  return launch_grouped<EPI, 0>(nch, ta, tb, p, sms, st, kind, ta2, tb2);
}

// Quantise (e4m3 or NVFP4) up to two row segments: routed rows (optionally gathered by perm,
// NVFP4 scale atoms per routed chunk) and the shared expert's token rows (atoms per token chunk).
int launch_quant(const ExpertPass& e, const __nv_bfloat16* src0, long long ld0, const int32_t* perm,
                 int rows0, void* dst0, float* scale0, uint8_t* sf0, const __nv_bfloat16* src1,
                 long long ld1, int rows1, void* dst1, float* scale1, uint8_t* sf1, int cols0,
                 int cols1, int tok_chunk, const ExpertPrefetch& pf, cudaStream_t st) {
  const int rows = rows0 + rows1;
  if (e.fmt == 2) {
    QuantFp4Job j{};
    j.seg[0] = QuantFp4Seg{src0, ld0, perm, e.k, perm ? e.topk_w : nullptr, perm ? e.w_perm : nullptr,
                           rows0, cols0, static_cast<uint8_t*>(dst0), operand_row_bytes(2, cols0),
                           sf0, scale0, e.chunks, e.n_chunks, 0};
    j.seg[1] = QuantFp4Seg{src1, ld1, nullptr, 1, nullptr, nullptr, rows1, cols1,
                           static_cast<uint8_t*>(dst1), operand_row_bytes(2, cols1), sf1, scale1,
                           nullptr, nullptr, tok_chunk};
    j.n_seg = rows1 > 0 ? 2 : 1;
    j.pf = pf;
    DG_TRY(launch_pdl(quant_fp4_rows_kernel, dim3(cdiv(rows, 8)), dim3(256), 0, st, j, e.done));
  } else {
    QuantJob j{};
    j.seg[0] = QuantSeg{src0, ld0, perm, e.k, perm ? e.topk_w : nullptr, perm ? e.w_perm : nullptr,
                        rows0, cols0, static_cast<uint8_t*>(dst0), operand_row_bytes(1, cols0),
                        scale0};
    j.seg[1] = QuantSeg{src1, ld1, nullptr, 1, nullptr, nullptr, rows1, cols1,
                        static_cast<uint8_t*>(dst1), operand_row_bytes(1, cols1), scale1};
    j.n_seg = rows1 > 0 ? 2 : 1;
    j.pf = pf;
    DG_TRY(launch_pdl(quant_rows_kernel, dim3(cdiv(rows, 8)), dim3(256), 0, st, j, e.done));
  }
  DG_LAUNCHED();
  return DG_OK;
}

int launch_experts(const ExpertPass& e, int sms, cudaStream_t st) {
  const int n_slots = e.n * e.k;
  const bool shared = e.hs > 0;
  const int nch = route_chunk(e.fmt, n_slots, e.E);
  const int slab = 64 << e.fmt;  // K elements per 128-byte slab: 64 bf16, 128 e4m3, 256 e2m1
  const long long row_d = operand_row_bytes(e.fmt, e.d);
  const long long row_hs = operand_row_bytes(e.fmt, e.hs);
  // bf16 and e4m3 with 64-token chunks (decode): the gate/up GEMM copies each routed row's token
  // (normed bf16, or its e4m3 codes quantised once per token) straight into its operand tiles.
  // Wider chunks (prefill, batched canvases) read a permuted copy by TMA boxes instead: there a
  // gather thread would issue 8-16 copies per stage.  NVFP4 quantises the routed rows in
  // permuted order with their per-chunk scale atoms (and hints the first experts' weights into
  // L2, which the router does for the others).
  const bool gemm_gather = e.fmt != 2 && nch == kGroupN;
  const int sh_rows = shared && !e.x_sh_ready ? e.n : 0;  // e4m3 tokens for the shared expert
  const bool launch_g = e.fmt == 2 || !gemm_gather || (e.fmt == 1 && !e.x_sh_ready);
  const int kind_g = e.profile && launch_g ? DG_KERNEL_GATHER : -1;
  prof_before(kind_g, st);
  if (e.fmt == 2) {
    const ExpertPrefetch epf{e.chunks, e.n_chunks, kPrefetchExperts, e.w_gu, 2ll * e.hid * row_d};
    DG_TRY(launch_quant(e, e.xn, e.d, e.perm, n_slots, e.x_perm, e.x_perm_scale, e.x_sf, e.xn, e.d,
                        shared ? e.n : 0, e.x_sh, e.x_sh_scale, e.x_sh_sf, e.d, e.d, nch, epf, st));
  } else if (e.fmt == 1 && gemm_gather) {
    if (!e.x_sh_ready)
      DG_TRY(launch_quant(e, e.xn, e.d, nullptr, e.n, e.x_sh, e.x_sh_scale, nullptr, nullptr, 0, 0,
                          nullptr, nullptr, nullptr, e.d, e.d, nch, ExpertPrefetch{}, st));
  } else if (e.fmt == 1) {
    DG_TRY(launch_quant(e, e.xn, e.d, e.perm, n_slots, e.x_perm, e.x_perm_scale, nullptr, e.xn, e.d,
                        sh_rows, e.x_sh, e.x_sh_scale, nullptr, e.d, e.d, nch, ExpertPrefetch{}, st));
  } else if (!gemm_gather) {
    DG_TRY(launch_pdl(gather_rows_kernel, dim3(cdiv(n_slots, 4)), dim3(256), 0, st, e.xn, e.perm,
                      e.k, e.d, n_slots, static_cast<__nv_bfloat16*>(e.x_perm), e.done));
    DG_LAUNCHED();
  }
  prof_after(kind_g, st);

  GemmParams p{};
  p.chunks = e.chunks;
  p.chunk_count = e.n_chunks;
  p.m_tiles = cdiv(2 * e.hid, 128);
  p.n_chunk = nch;
  p.alt_m_tiles = cdiv(2 * e.hs, 128);
  p.alt_chunks = cdiv(e.n, nch);
  p.alt_tokens = e.n;
  p.a_rows_per_group = 2 * e.hid;
  p.kb_total = cdiv(e.d, slab);
  p.m_valid = 2 * e.hid;
  p.out_bf16 = e.h;
  p.ld_out = e.hid;
  p.alt_group = shared ? e.E : -1;
  p.alt_kb_total = cdiv(e.d, slab);
  p.alt_m_valid = 2 * e.hs;
  p.alt_out_bf16 = e.h_sh;
  p.alt_ld_out = e.hs;
  p.a_scale = e.w_gu_scale;
  p.b_scale = e.fmt == 1 && gemm_gather ? e.x_sh_scale : e.x_perm_scale;
  if (gemm_gather) {
    p.gather_src = static_cast<const uint8_t*>(e.fmt == 1 ? e.x_sh : static_cast<const void*>(e.xn));
    p.gather_perm = e.perm;
    p.gather_k = e.k;
    p.gather_ld = static_cast<int>(row_d);
  }
  p.alt_a_scale = e.ws_gu_scale;
  p.alt_b_scale = e.x_sh_scale;
  p.a_sf = e.w_gu_sf;
  p.b_sf = e.x_sf;
  p.alt_a_sf = e.ws_gu_sf;
  p.alt_b_sf = e.x_sh_sf;
  if (shared) {  // the down GEMM starts with the shared expert's items
    p.pf0 = e.ws_d;
    p.pf0_bytes = static_cast<long long>(e.d) * row_hs;
  }
  p.err = e.err;
  p.done = e.done;
  const int kind_gu = e.profile ? DG_KERNEL_EXPERT_GATE_UP : -1;
  DG_TRY(launch_grouped_fmt<kEpiGluBf16>(e.fmt, nch, *e.tm_wgu, *e.tm_xperm, p, sms, st, kind_gu,
                                         shared ? e.tm_wsgu : nullptr,
                                         shared ? e.tm_xsh : nullptr));

  if (e.fmt != 0) {
    const int kind_q = e.profile ? DG_KERNEL_QUANT_H : -1;
    prof_before(kind_q, st);
    DG_TRY(launch_quant(e, e.h, e.hid, nullptr, n_slots, e.hq, e.hq_scale, e.h_sf, e.h_sh, e.hs,
                        shared ? e.n : 0, e.hsq, e.hsq_scale, e.hs_sf, e.hid, e.hs, nch,
                        ExpertPrefetch{}, st));
    prof_after(kind_q, st);
  }

  GemmParams q{};
  q.chunks = e.chunks;
  q.chunk_count = e.n_chunks;
  q.m_tiles = cdiv(e.d, 128);
  q.n_chunk = nch;
  q.alt_m_tiles = cdiv(e.d, 128);
  q.alt_chunks = cdiv(e.n, nch);
  q.alt_tokens = e.n;
  q.a_rows_per_group = e.d;
  q.kb_total = cdiv(e.hid, slab);
  q.m_valid = e.d;
  q.out_f32 = e.y_slot;
  q.ld_out = e.d;
  q.perm = e.perm;
  q.scale = e.w_perm;
  q.alt_group = shared ? e.E : -1;
  q.alt_kb_total = cdiv(e.hs, slab);
  q.alt_m_valid = e.d;
  q.alt_out_f32 = e.y_shared;
  q.alt_ld_out = e.d;
  q.a_scale = e.w_d_scale;
  q.b_scale = e.hq_scale;
  q.alt_a_scale = e.ws_d_scale;
  q.alt_b_scale = e.hsq_scale;
  q.a_sf = e.w_d_sf;
  q.b_sf = e.h_sf;
  q.alt_a_sf = e.ws_d_sf;
  q.alt_b_sf = e.hs_sf;
  q.pf0 = e.pf0;
  q.pf0_bytes = e.pf0_bytes;
  q.pf1 = e.pf1;
  q.pf1_bytes = e.pf1_bytes;
  q.err = e.err;
  q.done = e.done;
  const int kind_d = e.profile ? DG_KERNEL_EXPERT_DOWN : -1;
  DG_TRY(launch_grouped_fmt<kEpiScatterF32>(e.fmt, nch, *e.tm_wd, *e.tm_h, q, sms, st, kind_d,
                                            shared ? e.tm_wsd : nullptr,
                                            shared ? e.tm_hs : nullptr));
  return DG_OK;
}

}  // namespace

// ---------------------------------------------------------------------------------------
struct dg_ctx {
  dg_config cfg;
  std::vector<dg_layer_weights> layers;
  const void* embed;
  const float* final_norm;
  const void* head_codes;   // e4m3 head: embedding codes [V, pitch] and row scales [V]
  const float* head_scale;
  uint8_t* xhq;             // e4m3 head: codes [batch * T, pitch] and scales of the normed tokens
  float* xhs;
  uint8_t* kv;
  uint8_t* scratch;
  int32_t kv_len;
  int sms;
  int batch;        // sequences decoded together (>= 1)
  bool bf16;
  int esz;          // bytes per stored element (2 or 4)
  int tq;           // query rows per head in the Q buffer
  int qkv_rows;
  int split_r;  // cluster size of the router projection
  int att_splits_max;
  size_t part_elems;
  // scratch views
  int32_t *canvas, *argmax, *prev_argmax, *locked, *state, *ticket, *err;
  int32_t* all_done;  // [0] every canvas stopped, [1] stopped canvases (after the state words)
  float *entropy, *conf;
  double* row_h;
  float* x;
  void* xn;
  float* part;
  void* q;
  float* o_part;
  float2* ml_part;
  void* o;
  float* router_logits;
  int32_t *topk_ids, *offsets, *perm, *n_chunks, *route_ticket;
  float* topk_w;
  int4* chunks;  // routed token chunks of the grouped GEMMs
  void *x_perm, *h, *hs;
  int fmt;  // expert operands: 0 bf16, 1 e4m3, 2 NVFP4
  uint8_t *x_sf, *x_sh_sf, *h_sf, *hs_sf;  // NVFP4 token-side scale atoms
  void *x_sh, *hq, *hsq;  // e4m3 codes: shared-expert tokens, h per slot, shared h per token
  float *x_perm_scale, *x_sh_scale, *hq_scale, *hsq_scale;
  float* w_perm;  // route weights in permuted order
  int32_t* commit_ids;  // sticky locks: the ids a block commits
  float *y_slot, *y_shared;
  StatPartial* lm_part;
  float* logits;  // fp32 path
  float2* rope_tab;
  void *kc, *vtc;
  // tensor maps (bf16)
  CUtensorMap tm_xn32, tm_xn128, tm_o32, tm_xperm, tm_h, tm_hs, tm_q, tm_k, tm_vt, tm_embed;
  CUtensorMap tm_xsh;  // e4m3: B operand of the shared expert's gate/up
  CUtensorMap tm_xhq, tm_ehq;  // e4m3 head: token codes (128-row boxes), vocabulary codes (256)
  std::vector<CUtensorMap> tm_wqkv, tm_wo, tm_wr, tm_wgu, tm_wd, tm_wsgu, tm_wsd;
  uint64_t seed;
  uint32_t block;
};

namespace {

int check_config(const dg_config* c) {
  if (!c) return fail(DG_ERR_INVALID_ARG, "null config");
  if (c->n_layers < 1 || c->d_model < 1 || c->n_heads < 1 || c->n_kv_heads < 1 ||
      c->head_dim < 2 || c->n_experts < 1 || c->top_k < 1 || c->expert_hidden < 1 ||
      c->shared_hidden < 0 || c->vocab < 2 || c->canvas < 1 || c->kv_capacity < 1)
    return fail(DG_ERR_INVALID_ARG, "config has a non-positive size");
  if (c->n_heads % c->n_kv_heads != 0)
    return fail(DG_ERR_INVALID_ARG, "n_heads must be a multiple of n_kv_heads");
  if (c->top_k > 8 || c->top_k > c->n_experts || c->n_experts > 256)
    return fail(DG_ERR_UNSUPPORTED, "need top_k <= min(8, E) and E <= 256");
  if (c->canvas > 256) return fail(DG_ERR_UNSUPPORTED, "canvas must be <= 256");
  if (c->kv_capacity % 8 != 0 || c->kv_capacity < c->canvas)
    return fail(DG_ERR_INVALID_ARG, "kv_capacity must be a multiple of 8 and >= canvas");
  // TMA row coordinates of the K cache ([L * Hkv * cap] rows) and the per-layer V^T offsets are
  // 32-bit
  if (static_cast<long long>(std::max(1, c->batch)) * c->n_layers * c->n_kv_heads *
              c->kv_capacity >= (1ll << 31) ||
      static_cast<long long>(c->n_kv_heads) * c->head_dim * c->kv_capacity >= (1ll << 31))
    return fail(DG_ERR_UNSUPPORTED, "kv_capacity too large for 32-bit cache coordinates");
  if (c->head_dim % 4 != 0) return fail(DG_ERR_INVALID_ARG, "head_dim must be a multiple of 4");
  if (c->d_model % 4 != 0 || c->d_model > 4096)
    return fail(DG_ERR_UNSUPPORTED, "d_model must be a multiple of 4 and at most 4096");
  if (c->n_experts % 4 != 0)
    return fail(DG_ERR_UNSUPPORTED, "n_experts must be a multiple of 4");
  if (c->vocab % 8 != 0) return fail(DG_ERR_UNSUPPORTED, "vocab must be a multiple of 8");
  if (c->max_steps < 1 || c->fixed_steps < 0)
    return fail(DG_ERR_INVALID_ARG, "max_steps must be >= 1 and fixed_steps >= 0");
  if (c->prefill_chunk < 0 || c->prefill_chunk % 128 != 0 || c->prefill_chunk > 4096)
    return fail(DG_ERR_INVALID_ARG, "prefill_chunk must be 0 or a multiple of 128, <= 4096");
  if (c->batch < 0 || c->batch > kMaxBatch)
    return fail(DG_ERR_INVALID_ARG, "batch must be in [0, %d]", kMaxBatch);
  if (c->batch > 1 && (c->dtype == DG_DTYPE_FP32 || c->canvas % 128 != 0 ||
                       c->batch * c->canvas > 4096))
    return fail(DG_ERR_UNSUPPORTED,
                "batch > 1 needs a bf16 dtype, canvas %% 128 == 0 and batch * canvas <= 4096");
  if (c->lm_head_e4m3 < 0 || c->lm_head_e4m3 > 1 ||
      (c->lm_head_e4m3 && c->dtype == DG_DTYPE_FP32))
    return fail(DG_ERR_INVALID_ARG, "lm_head_e4m3 must be 0 or 1 (1 needs a bf16 dtype)");
  if (c->commit_reuse_kv < 0 || c->commit_reuse_kv > 1)
    return fail(DG_ERR_INVALID_ARG, "commit_reuse_kv must be 0 or 1");
  if (!(c->temperature >= 0.0f) || c->temperature > 1e4f)
    return fail(DG_ERR_INVALID_ARG, "temperature must be in (0, 1e4] (0 means 1)");
  if (c->lock_rule < 0 || c->lock_rule > 1 || !(c->entropy_lock >= 0.0) || c->sticky_locks < 0 ||
      c->sticky_locks > 1)
    return fail(DG_ERR_INVALID_ARG, "lock_rule must be 0 or 1, entropy_lock >= 0, sticky 0 or 1");
  if (c->dtype == DG_DTYPE_BF16_NVFP4 && c->d_model % 128)
    return fail(DG_ERR_UNSUPPORTED, "NVFP4 experts need d a multiple of 128");
  if (c->dtype == DG_DTYPE_BF16 || c->dtype == DG_DTYPE_BF16_E4M3 ||
      c->dtype == DG_DTYPE_BF16_NVFP4) {
    if (c->head_dim != 128) return fail(DG_ERR_UNSUPPORTED, "bf16 path needs head_dim 128");
    if (c->d_model % 64 || c->expert_hidden % 64 || c->shared_hidden % 64)
      return fail(DG_ERR_UNSUPPORTED, "bf16 path needs d, h, hs multiples of 64");
    if (c->n_experts > 128 || c->d_model < 128)
      return fail(DG_ERR_UNSUPPORTED, "bf16 path needs E <= 128 and d >= 128 (one router tile)");
    if (c->vocab % 256) return fail(DG_ERR_UNSUPPORTED, "bf16 path needs vocab % 256 == 0");
  } else if (c->dtype == DG_DTYPE_FP32) {
    if (c->head_dim > 128) return fail(DG_ERR_UNSUPPORTED, "fp32 path needs head_dim <= 128");
    if (c->vocab % 4) return fail(DG_ERR_UNSUPPORTED, "fp32 path needs vocab % 4 == 0");
  } else {
    return fail(DG_ERR_INVALID_ARG, "unknown dtype %d", c->dtype);
  }
  return DG_OK;
}

// Workspace plan: every buffer at a 256-byte boundary, in this order.
struct Plan {
  size_t off[56];
  size_t total;
  size_t kv;
};

enum Buf {
  B_CANVAS, B_ARGMAX, B_PREV, B_LOCKED, B_STATE, B_TICKET, B_ERR, B_ENT, B_CONF, B_ROWH, B_X,
  B_XN, B_PART, B_Q, B_OPART, B_ML, B_O, B_RLOG, B_IDS, B_W, B_OFF, B_PERM, B_CHUNKS,
  B_NCHUNKS, B_RTICKET, B_XPERM, B_H, B_HS, B_YSLOT, B_YSH, B_LMPART, B_LOGITS, B_ROPE,
  B_XPS, B_XSH, B_XSHS, B_HQ, B_HQS, B_HSQ, B_HSQS, B_WPERM, B_COMMIT, B_XSF, B_XSHSF, B_HSF,
  B_HSSF, B_XHQ, B_XHS, B_END
};

struct Derived {
  int tq, qkv_rows, split_r, att_splits, esz;
  size_t part_elems;
  long long max_chunks;
};

// Sequences decoded together (batched canvases).
int n_seq(const dg_config& c) { return std::max(1, c.batch); }
// Most tokens one forward pass carries: the batch's canvases, or a prefill chunk of one prompt.
int tokens_max(const dg_config& c) { return std::max(n_seq(c) * c.canvas, c.prefill_chunk); }

Derived derive(const dg_config& c, int sms) {
  Derived d{};
  const bool bf16 = c.dtype != DG_DTYPE_FP32;
  d.esz = bf16 ? 2 : 4;
  const long long T = tokens_max(c);
  d.tq = bf16 ? std::max(256, cdiv(static_cast<int>(T), 128) * 128) : static_cast<int>(T);
  d.qkv_rows = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim;
  if (bf16) {
    // cluster size of the router projection (QKV and O pick theirs per call)
    d.split_r = std::min(kCluMaxSplits, c.d_model / 64);
    d.part_elems = 1;
  } else {
    d.split_r = 1;
    d.part_elems = std::max({static_cast<size_t>(T) * d.qkv_rows,
                             static_cast<size_t>(T) * c.d_model,
                             static_cast<size_t>(T) * c.n_experts});
  }
  const int group = c.n_heads / c.n_kv_heads;
  const int m_tiles = group * cdiv(c.canvas, 128) * n_seq(c);  // a denoise pass takes the most splits
  d.att_splits = std::max(1, std::min(kMaxAttnSplits, sms / std::max(1, m_tiles * c.n_kv_heads)));
  d.max_chunks = c.n_experts + (T * c.top_k + kGroupN - 1) / kGroupN;
  return d;
}

Plan plan(const dg_config& c, int sms) {
  Plan p{};
  const Derived dv = derive(c, sms);
  const bool bf16 = c.dtype != DG_DTYPE_FP32;
  const int fmt = c.dtype == DG_DTYPE_BF16_E4M3 ? 1 : c.dtype == DG_DTYPE_BF16_NVFP4 ? 2 : 0;
  const bool f8 = fmt != 0;  // quantised expert operands
  // Tc: canvas positions of all sequences; per-canvas arrays are [batch][canvas]
  const size_t Tc = static_cast<size_t>(c.canvas) * n_seq(c), T = tokens_max(c), d = c.d_model,
               E = c.n_experts, k = c.top_k, es = dv.esz;
  const size_t hd = c.head_dim, Hq = c.n_heads;
  const size_t nv = bf16 ? c.vocab / 256 : cdiv(c.vocab, 4096);
  size_t sz[B_END];
  sz[B_CANVAS] = sz[B_ARGMAX] = sz[B_PREV] = sz[B_LOCKED] = Tc * 4;
  // state words per sequence, then the all-done flag and count
  sz[B_STATE] = (static_cast<size_t>(n_seq(c)) * kStWords + 2) * 4;
  sz[B_TICKET] = static_cast<size_t>(n_seq(c)) * 4;
  sz[B_ERR] = 4;
  sz[B_ENT] = sz[B_CONF] = Tc * 4;
  sz[B_ROWH] = Tc * 8;
  sz[B_X] = T * d * 4;
  sz[B_XN] = T * d * es;
  sz[B_PART] = dv.part_elems * 4;
  sz[B_Q] = Hq * dv.tq * hd * es;
  sz[B_OPART] = bf16 ? static_cast<size_t>(dv.att_splits) * Hq * dv.tq * 128 * 4 : 0;
  sz[B_ML] = bf16 ? static_cast<size_t>(dv.att_splits) * Hq * dv.tq * 8 : 0;
  sz[B_O] = T * Hq * hd * es;
  sz[B_RLOG] = T * E * 4;
  sz[B_IDS] = sz[B_W] = T * k * 4;
  sz[B_OFF] = (E + 1) * 4;
  sz[B_PERM] = T * k * 4;
  sz[B_CHUNKS] = bf16 ? dv.max_chunks * 16 : 0;
  sz[B_NCHUNKS] = 4;
  sz[B_RTICKET] = 4;
  const size_t dp = operand_row_bytes(fmt, c.d_model),
               hp = operand_row_bytes(fmt, c.expert_hidden),
               hsp = operand_row_bytes(fmt, std::max(64, c.shared_hidden));
  sz[B_XPERM] = bf16 ? T * k * (f8 ? dp : d * es) : 0;
  sz[B_H] = bf16 ? T * k * c.expert_hidden * es : 0;
  sz[B_HS] = bf16 ? T * std::max<size_t>(1, c.shared_hidden) * es : 0;
  sz[B_YSLOT] = T * k * d * 4;
  sz[B_YSH] = T * d * 4;
  sz[B_LMPART] = Tc * nv * sizeof(StatPartial);
  sz[B_LOGITS] = bf16 ? 0 : Tc * c.vocab * 4;
  sz[B_ROPE] = static_cast<size_t>(c.kv_capacity) * (hd / 2) * 8;
  // e4m3 experts: slot-row scales of x_perm, quantised tokens for the shared expert, quantised h
  sz[B_XPS] = f8 ? T * k * 4 : 0;
  sz[B_XSH] = f8 ? T * dp : 0;
  sz[B_XSHS] = f8 ? T * 4 : 0;
  sz[B_HQ] = f8 ? T * k * hp : 0;
  sz[B_HQS] = f8 ? T * k * 4 : 0;
  sz[B_HSQ] = f8 ? T * hsp : 0;
  sz[B_HSQS] = f8 ? T * 4 : 0;
  sz[B_WPERM] = bf16 ? T * k * 4 : 0;
  sz[B_COMMIT] = Tc * 4;  // committed ids with sticky locks
  // NVFP4: token-side scale atoms, per routed chunk (routed rows) and per 64-token chunk
  // (the shared expert's rows), 4 * ceil(K / 256) atoms of 512 B each
  const size_t tok_chunks = cdiv(static_cast<long long>(T), kGroupN);
  const size_t atoms_d = 4 * cdiv(c.d_model, 256), atoms_h = 4 * cdiv(c.expert_hidden, 256),
               atoms_hs = 4 * cdiv(std::max(64, c.shared_hidden), 256);
  sz[B_XSF] = fmt == 2 ? dv.max_chunks * atoms_d * 512 : 0;
  sz[B_XSHSF] = fmt == 2 ? tok_chunks * atoms_d * 512 : 0;
  sz[B_HSF] = fmt == 2 ? dv.max_chunks * atoms_h * 512 : 0;
  sz[B_HSSF] = fmt == 2 ? tok_chunks * atoms_hs * 512 : 0;
  // e4m3 head: codes and scales of the final normed canvas tokens
  sz[B_XHQ] = c.lm_head_e4m3 ? Tc * e4m3_pitch(c.d_model) : 0;
  sz[B_XHS] = c.lm_head_e4m3 ? Tc * 4 : 0;
  size_t o = 0;
  for (int b = 0; b < B_END; ++b) {
    p.off[b] = o;
    o += align256(std::max<size_t>(sz[b], 1));
  }
  p.total = o;
  // K of every (sequence, layer), then V^T of every (sequence, layer)
  p.kv = 2 * static_cast<size_t>(n_seq(c)) * c.n_layers * c.n_kv_heads * c.kv_capacity * hd * es;
  return p;
}

// ---- the layer pipeline -----------------------------------------------------------------
// Runs every layer over n tokens at positions pos0.. (canvas buffer or caller ids), writes their
// K/V into cache slots pos0..pos0+n-1 and leaves the final-normed hidden state in xn.
// parts: bit 0 = attention sub-block (QKV .. O projection, residual, ffn norm), bit 1 = MoE
// sub-block (router .. weighted combine, residual, next norm).
// seq0: the sequence whose cache the pass uses (a prefill pass of one prompt); seq_len > 0: the n
// tokens are consecutive runs of seq_len tokens of sequences 0, 1, ... (a denoise or commit pass
// over a batch of canvases), each at positions pos0.. of its own cache.
int run_layer(dg_ctx* c, int l, int n, int pos0, int causal, const float* next_norm,
              const int* done, cudaStream_t st, int parts = 3, int seq0 = 0, int seq_len = 0);

int run_forward(dg_ctx* c, const int32_t* ids, int n, int pos0, int causal, const int* done,
                cudaStream_t st, int seq0 = 0, int seq_len = 0) {
  const dg_config& g = c->cfg;
  prof_before(DG_KERNEL_EMBED, st);
  if (c->bf16)
    DG_TRY(launch_pdl(embed_norm_kernel<__nv_bfloat16, __nv_bfloat16>, dim3(n), dim3(256), 0, st,
        ids, static_cast<const __nv_bfloat16*>(c->embed), g.d_model, g.vocab,
        c->layers[0].attn_norm, g.eps, c->x, static_cast<__nv_bfloat16*>(c->xn), done, c->err));
  else
    DG_TRY(launch_pdl(embed_norm_kernel<float, float>, dim3(n), dim3(256), 0, st, ids,
        static_cast<const float*>(c->embed), g.d_model, g.vocab, c->layers[0].attn_norm, g.eps,
        c->x, static_cast<float*>(c->xn), done, c->err));
  DG_LAUNCHED();
  prof_after(DG_KERNEL_EMBED, st);
  for (int l = 0; l < g.n_layers; ++l) {
    const float* nn = (l + 1 < g.n_layers) ? c->layers[l + 1].attn_norm : c->final_norm;
    DG_TRY(run_layer(c, l, n, pos0, causal, nn, done, st, 3, seq0, seq_len));
  }
  return DG_OK;
}

template <typename TA>
int layer_tail_common(dg_ctx* c, int l, int n, int pos0, const int* done, cudaStream_t st,
                      long long qkv_ss, int splits_qkv) {
  const dg_config& g = c->cfg;
  const int hd = g.head_dim;
  const size_t kv_head_elems = static_cast<size_t>(g.kv_capacity) * hd;
  TA* kc = static_cast<TA*>(c->kc) + static_cast<size_t>(l) * g.n_kv_heads * kv_head_elems;
  TA* vtc = static_cast<TA*>(c->vtc) + static_cast<size_t>(l) * g.n_kv_heads * kv_head_elems;
  prof_before(DG_KERNEL_QKV_FINALIZE, st);
  DG_TRY(launch_pdl(qkv_finalize_kernel<TA>, dim3(cdiv(n, kQkvTok), g.n_heads + 2 * g.n_kv_heads), dim3(128), 0, st, 
      c->part, splits_qkv, qkv_ss, c->qkv_rows, hd, g.n_heads, g.n_kv_heads, c->rope_tab, n, pos0,
      static_cast<TA*>(c->q), c->tq, kc, vtc, g.kv_capacity, done));
  DG_LAUNCHED();
  prof_after(DG_KERNEL_QKV_FINALIZE, st);
  return DG_OK;
}

int run_layer(dg_ctx* c, int l, int n, int pos0, int causal, const float* next_norm,
              const int* done, cudaStream_t st, int parts, int seq0, int seq_len) {
  const dg_config& g = c->cfg;
  // cache layer block of (sequence seq0, layer l); sequences are L layer blocks apart
  const long long lb = static_cast<long long>(seq0) * g.n_layers + l;
  const long long seq_blocks = seq_len > 0 ? g.n_layers : 0;
  const dg_layer_weights& w = c->layers[l];
  const int d = g.d_model, hd = g.head_dim, k = g.top_k, E = g.n_experts;
  // keys each query sees: the committed history plus its own sequence's new tokens
  const int n_keys = pos0 + (seq_len > 0 ? seq_len : n);
  const int n_slots = n * k;
  if (!c->bf16) {
    // ---------------- all-fp32 path ----------------
    const float* xn = static_cast<const float*>(c->xn);
    if (parts & 1) {
    DG_TRY(launch_pdl(gemm_f32_nt_kernel, dim3(cdiv(c->qkv_rows, 64), cdiv(n, 64)), dim3(256), 0, st,
        xn, static_cast<const float*>(w.wqkv), n, c->qkv_rows, d, c->part, c->qkv_rows, done));
    DG_LAUNCHED();
    DG_TRY(layer_tail_common<float>(c, l, n, pos0, done, st, 0, 1));
    const size_t kv_head_elems = static_cast<size_t>(g.kv_capacity) * hd;
    const float* kc = static_cast<const float*>(c->kc) + static_cast<size_t>(l) * g.n_kv_heads * kv_head_elems;
    const float* vtc = static_cast<const float*>(c->vtc) + static_cast<size_t>(l) * g.n_kv_heads * kv_head_elems;
    const int smem = (n_keys + hd) * 4;
    if (smem > 200 * 1024) return fail(DG_ERR_UNSUPPORTED, "fp32 attention: too many keys");
    DG_TRY(set_smem(attention_f32_kernel, smem));
    DG_TRY(launch_pdl(attention_f32_kernel, dim3(n, g.n_heads), dim3(128), smem, st, 
        static_cast<const float*>(c->q), kc, vtc, static_cast<float*>(c->o), g.n_heads,
        g.n_heads / g.n_kv_heads, c->tq, hd, g.kv_capacity, n_keys, causal ? pos0 : -1,
        1.0f / sqrtf(static_cast<float>(hd)), done));
    DG_LAUNCHED();
    DG_TRY(launch_pdl(gemm_f32_nt_kernel, dim3(cdiv(d, 64), cdiv(n, 64)), dim3(256), 0, st, 
        static_cast<const float*>(c->o), static_cast<const float*>(w.wo), n, d, g.n_heads * hd,
        c->part, d, done));
    DG_LAUNCHED();
    DG_TRY(launch_pdl(residual_norm_kernel<float>, dim3(n), dim3(256), 0, st, c->x, c->part, 1, 0, d, w.ffn_norm, g.eps,
                                                   static_cast<float*>(c->xn), nullptr, 0, nullptr, done));
    DG_LAUNCHED();
    }
    if (!(parts & 2)) return DG_OK;
    DG_TRY(launch_pdl(gemm_f32_nt_kernel, dim3(cdiv(E, 64), cdiv(n, 64)), dim3(256), 0, st, 
        xn, static_cast<const float*>(w.wr), n, E, d, c->part, E, done));
    DG_LAUNCHED();
    DG_TRY(launch_pdl(router_topk_kernel, dim3(cdiv(n, 4)), dim3(128), 0, st, c->part, 1, 0, n, E, k, c->router_logits,
                                                   c->topk_ids, c->topk_w, done));
    DG_LAUNCHED();
    const int smem_e = (d + g.expert_hidden) * 4;
    DG_TRY(set_smem(moe_expert_f32_kernel, smem_e));
    DG_TRY(launch_pdl(moe_expert_f32_kernel, dim3(n_slots), dim3(256), smem_e, st, 
        xn, c->topk_ids, c->topk_w, k, static_cast<const float*>(w.w_gu),
        static_cast<const float*>(w.w_d), d, g.expert_hidden, c->y_slot, done));
    DG_LAUNCHED();
    const float* ysh = nullptr;
    if (g.shared_hidden > 0) {
      const int smem_s = (d + g.shared_hidden) * 4;
      DG_TRY(set_smem(moe_expert_f32_kernel, std::max(smem_s, smem_e)));
      DG_TRY(launch_pdl(moe_expert_f32_kernel, dim3(n), dim3(256), smem_s, st, 
          xn, nullptr, nullptr, 1, static_cast<const float*>(w.ws_gu),
          static_cast<const float*>(w.ws_d), d, g.shared_hidden, c->y_shared, done));
      DG_LAUNCHED();
      ysh = c->y_shared;
    }
    DG_TRY(launch_pdl(moe_combine_norm_kernel<float>, dim3(n), dim3(256), 0, st, c->x, c->y_slot, k, ysh, d, next_norm,
                                                      g.eps, static_cast<float*>(c->xn), done));
    DG_LAUNCHED();
    return DG_OK;
  }
  // ---------------- bf16 tcgen05 path ----------------
  if (parts & 1) {
  // QKV projection (cluster split-K) with RoPE, Q and the K / V^T cache writes in its epilogue
  {
    const size_t kv_head_elems = static_cast<size_t>(g.kv_capacity) * hd;
    CluParams p = clu_params(c->qkv_rows, n, d / 64,
                             clu_splits(cdiv(c->qkv_rows, 128) * cdiv(n, 256), d / 64, c->sms),
                             c->err, done);
    p.n_heads = g.n_heads;
    p.n_kv_heads = g.n_kv_heads;
    p.tq = c->tq;
    p.pos0 = pos0;
    p.ldk = g.kv_capacity;
    p.rope_tab = c->rope_tab;
    p.q = static_cast<__nv_bfloat16*>(c->q);
    p.k_cache = static_cast<__nv_bfloat16*>(c->kc) + static_cast<size_t>(lb) * g.n_kv_heads * kv_head_elems;
    p.vt_cache = static_cast<__nv_bfloat16*>(c->vtc) + static_cast<size_t>(lb) * g.n_kv_heads * kv_head_elems;
    p.seq_len = seq_len;
    p.seq_kv_stride = seq_blocks * g.n_kv_heads * static_cast<long long>(kv_head_elems);
    DG_TRY(launch_cluster<kCluQkv>(c->tm_wqkv[l], c->tm_xn32, p, st, DG_KERNEL_QKV));
  }
  // attention over [cache 0..pos0 | new tokens], split over keys
  {
    const int group = g.n_heads / g.n_kv_heads;
    const int tph = cdiv(n, 128);  // query tiles per head in use
    const int m_tiles = group * tph;
    const int n_kv_tiles = cdiv(n_keys, 128);
    int splits = std::max(1, std::min(c->att_splits_max, c->sms / (m_tiles * g.n_kv_heads)));
    splits = std::min(splits, n_kv_tiles);
    const int tps = cdiv(n_kv_tiles, splits);
    splits = cdiv(n_kv_tiles, tps);
    AttnParams a{};
    a.group = group;
    a.tq = c->tq;
    a.tiles_per_head = tph;
    a.n_queries = n;
    a.n_keys = n_keys;
    a.causal_prefix = causal ? pos0 : -1;
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(hd)));
    a.tiles_per_split = tps;
    a.q_row_base = 0;
    a.k_row_base = lb * g.n_kv_heads * g.kv_capacity;
    a.ldk = g.kv_capacity;
    a.vt_row_base = static_cast<int>(lb * g.n_kv_heads * hd);
    a.seq_len = seq_len;
    a.k_seq_rows = seq_blocks * g.n_kv_heads * g.kv_capacity;
    a.vt_seq_rows = static_cast<int>(seq_blocks * g.n_kv_heads * hd);
    a.n_heads = g.n_heads;
    a.o_part = c->o_part;
    a.ml_part = c->ml_part;
    a.o = static_cast<__nv_bfloat16*>(c->o);
    if (parts & 2 && g.shared_hidden > 0) {  // the shared expert's weights of this layer
      a.pf0 = w.ws_gu;
      a.pf0_bytes = 2ll * g.shared_hidden * operand_row_bytes(c->fmt, d);
    }
    a.err = c->err;
    a.done = done;
    DG_TRY(set_smem(attention_kernel, kAttnSmemBytes));
    prof_before(DG_KERNEL_ATTENTION, st);
    DG_TRY(launch_pdl_cluster(attention_kernel, dim3(m_tiles, g.n_kv_heads, splits),
                              dim3(kAttnThreads), kAttnSmemBytes, st, dim3(1, 1, splits), c->tm_q,
                              c->tm_k, c->tm_vt, a));
    DG_LAUNCHED();
    prof_after(DG_KERNEL_ATTENTION, st);
  }
  // O projection onto the residual stream (cluster split-K), then the ffn norm
  {
    CluParams p = clu_params(d, n, g.n_heads * hd / 64,
                             clu_splits(cdiv(d, 128) * cdiv(n, 256), g.n_heads * hd / 64, c->sms),
                             c->err, done);
    p.x = c->x;
    DG_TRY(launch_cluster<kCluResidual>(c->tm_wo[l], c->tm_o32, p, st, DG_KERNEL_O_PROJ));
    prof_before(DG_KERNEL_RESIDUAL_NORM, st);
    // with e4m3 experts it also writes the e4m3 codes of its output, the experts' token operand
    const bool q8 = c->fmt == 1;
    DG_TRY(launch_pdl(q8 ? residual_norm_kernel<__nv_bfloat16, true>
                         : residual_norm_kernel<__nv_bfloat16, false>,
                      dim3(n), dim3(256), 0, st, c->x, c->part, 0, 0ll, d, w.ffn_norm, g.eps,
                      static_cast<__nv_bfloat16*>(c->xn),
                      q8 ? static_cast<uint8_t*>(c->x_sh) : nullptr,
                      static_cast<int>(operand_row_bytes(1, d)), q8 ? c->x_sh_scale : nullptr, done));
    DG_LAUNCHED();
    prof_after(DG_KERNEL_RESIDUAL_NORM, st);
  }
  }
  if (!(parts & 2)) return DG_OK;
  // router (cluster split-K) with top-k in its epilogue; the grid's last CTA routes the canvas
  const bool shared = g.shared_hidden > 0;
  {
    // 64-token chunks: the top-k of a chunk is spread over its 8 CTAs
    CluParams p = clu_params(E, n, d / 64, c->split_r, c->err, done, kRouterChunk);
    p.router_logits = c->router_logits;
    p.ids = c->topk_ids;
    p.wts = c->topk_w;
    p.top_k = k;
    p.route = RouteArgs{c->topk_ids, n, k, E, route_chunk(c->fmt, n_slots, E), c->offsets,
                        c->perm, c->chunks, c->n_chunks, nullptr, nullptr};
    if (c->fmt != 2) {  // the gate/up GEMM gathers the rows itself; the routing permutes the weights
      p.route.wts = c->topk_w;
      p.route.w_perm = c->w_perm;
      p.pf_first = w.w_gu;  // the first routed experts' gate/up weights
      p.pf_first_bytes = std::min(kRouterPrefetchExperts, E) * 2ll * g.expert_hidden *
                         operand_row_bytes(c->fmt, d);
    }
    p.ticket = c->route_ticket;
    DG_TRY(launch_cluster<kCluRouter>(c->tm_wr[l], c->tm_xn32, p, st, DG_KERNEL_ROUTER));
  }
  // permutation gather (+ e4m3 quantisation) and grouped expert GEMMs; the shared expert rides
  // along as group E
  {
    ExpertPass e{};
    e.n = n;
    e.d = d;
    e.k = k;
    e.E = E;
    e.hid = g.expert_hidden;
    e.hs = g.shared_hidden;
    e.fmt = c->fmt;
    e.perm = c->perm;
    e.topk_w = c->topk_w;
    e.w_perm = c->w_perm;
    e.chunks = c->chunks;
    e.n_chunks = c->n_chunks;
    e.xn = static_cast<const __nv_bfloat16*>(c->xn);
    e.x_perm = c->x_perm;
    e.x_perm_scale = c->x_perm_scale;
    e.x_sh = c->x_sh;
    e.x_sh_scale = c->x_sh_scale;
    e.x_sh_ready = c->fmt == 1;  // the ffn norm wrote the codes
    e.h = static_cast<__nv_bfloat16*>(c->h);
    e.h_sh = static_cast<__nv_bfloat16*>(c->hs);
    e.hq = c->hq;
    e.hq_scale = c->hq_scale;
    e.hsq = c->hsq;
    e.hsq_scale = c->hsq_scale;
    e.x_sf = c->x_sf;
    e.x_sh_sf = c->x_sh_sf;
    e.h_sf = c->h_sf;
    e.hs_sf = c->hs_sf;
    e.y_slot = c->y_slot;
    e.y_shared = c->y_shared;
    e.w_gu = w.w_gu;
    e.ws_d = w.ws_d;
    e.w_gu_scale = w.w_gu_scale;
    e.w_d_scale = w.w_d_scale;
    e.ws_gu_scale = w.ws_gu_scale;
    e.ws_d_scale = w.ws_d_scale;
    e.w_gu_sf = static_cast<const uint8_t*>(w.w_gu_sf);
    e.w_d_sf = static_cast<const uint8_t*>(w.w_d_sf);
    e.ws_gu_sf = static_cast<const uint8_t*>(w.ws_gu_sf);
    e.ws_d_sf = static_cast<const uint8_t*>(w.ws_d_sf);
    e.tm_wgu = &c->tm_wgu[l];
    e.tm_xperm = &c->tm_xperm;
    e.tm_wsgu = &c->tm_wsgu[l];
    e.tm_xsh = c->fmt != 0 ? &c->tm_xsh : &c->tm_xn32;
    e.tm_wd = &c->tm_wd[l];
    e.tm_h = &c->tm_h;
    e.tm_wsd = &c->tm_wsd[l];
    e.tm_hs = &c->tm_hs;
    if (l + 1 < g.n_layers) {  // the next layer's QKV and O projections
      const dg_layer_weights& wn = c->layers[l + 1];
      e.pf0 = wn.wqkv;
      e.pf0_bytes = static_cast<long long>(c->qkv_rows) * d * 2;
      e.pf1 = wn.wo;
      e.pf1_bytes = static_cast<long long>(d) * g.n_heads * hd * 2;
    } else {  // the first vocabulary tiles of the LM head
      e.pf0 = c->embed;
      e.pf0_bytes = std::min<long long>(64ll << 20, static_cast<long long>(g.vocab) * d * 2);
    }
    e.err = c->err;
    e.done = done;
    e.profile = true;
    DG_TRY(launch_experts(e, c->sms, st));
  }
  const float* ysh = shared ? c->y_shared : nullptr;
  prof_before(DG_KERNEL_COMBINE_NORM, st);
  DG_TRY(launch_pdl(moe_combine_norm_kernel<__nv_bfloat16>, dim3(n), dim3(256), 0, st, 
      c->x, c->y_slot, k, ysh, d, next_norm, g.eps, static_cast<__nv_bfloat16*>(c->xn), done));
  DG_LAUNCHED();
  prof_after(DG_KERNEL_COMBINE_NORM, st);
  return DG_OK;
}

int run_lm_head(dg_ctx* c, float* logits_out, const int* done, cudaStream_t st) {
  const dg_config& g = c->cfg;
  const int T = g.canvas;
  if (c->bf16) {
    // one launch per 256 canvas tokens (each launch holds two 128-token accumulators in TMEM)
    const int n_tok = T * c->batch;
    const bool f8h = g.lm_head_e4m3 != 0;
    if (f8h) {  // e4m3 codes and scales of the final normed tokens
      QuantJob j{};
      j.seg[0] = QuantSeg{static_cast<const __nv_bfloat16*>(c->xn), g.d_model, nullptr, 1, nullptr,
                          nullptr, n_tok, g.d_model, c->xhq, e4m3_pitch(g.d_model), c->xhs};
      j.n_seg = 1;
      DG_TRY(launch_pdl(quant_rows_kernel, dim3(cdiv(n_tok, 8)), dim3(256), 0, st, j, done));
      DG_LAUNCHED();
    }
    for (int t0 = 0; t0 < n_tok; t0 += 256) {
      LmHeadParams p{};
      p.n_tokens = std::min(256, n_tok - t0);
      p.tok_base = t0;
      p.n_vtiles = g.vocab / 256;
      p.kb_total = f8h ? cdiv(g.d_model, 128) : g.d_model / 64;
      p.x_scale = c->xhs;
      p.e_scale = c->head_scale;
      p.partials = c->lm_part;
      p.logits = logits_out;
      p.vocab = g.vocab;
      p.inv_t = g.temperature > 0.0f ? 1.0f / g.temperature : 1.0f;
      p.err = c->err;
      p.done = done;
      const int grid = std::min(p.n_vtiles, c->sms);
      prof_before(DG_KERNEL_LM_HEAD, st);
      const CUtensorMap& tx = f8h ? c->tm_xhq : c->tm_xn128;
      const CUtensorMap& te = f8h ? c->tm_ehq : c->tm_embed;
      if (logits_out) {
        auto k = f8h ? lmhead_kernel<false, true> : lmhead_kernel<false, false>;
        DG_TRY(set_smem(k, kLmSmemBytes));
        DG_TRY(launch_pdl(k, dim3(grid), dim3(kLmThreads), kLmSmemBytes, st, tx, te, p));
      } else {
        auto k = f8h ? lmhead_kernel<true, true> : lmhead_kernel<true, false>;
        DG_TRY(set_smem(k, kLmSmemBytes));
        DG_TRY(launch_pdl(k, dim3(grid), dim3(kLmThreads), kLmSmemBytes, st, tx, te, p));
      }
      DG_LAUNCHED();
      prof_after(DG_KERNEL_LM_HEAD, st);
    }
    return DG_OK;
  }
  float* dst = logits_out ? logits_out : c->logits;
  DG_TRY(launch_pdl(gemm_f32_nt_kernel, dim3(cdiv(g.vocab, 64), cdiv(T, 64)), dim3(256), 0, st, 
      static_cast<const float*>(c->xn), static_cast<const float*>(c->embed), T, g.vocab, g.d_model,
      dst, g.vocab, done));
  DG_LAUNCHED();
  if (!logits_out) {
    DG_TRY(launch_pdl(logits_stats_kernel<float, 16>, dim3(cdiv(g.vocab, 4096), T), dim3(256), 0, st,
        c->logits, g.vocab, 4096, c->lm_part, done,
        g.temperature > 0.0f ? 1.0f / g.temperature : 1.0f));
    DG_LAUNCHED();
  }
  return DG_OK;
}

int bind_tmaps(dg_ctx* c) {
  const dg_config& g = c->cfg;
  const uint64_t T = tokens_max(g), d = g.d_model, hd = g.head_dim, k = g.top_k;
  DG_TRY(make_tmap(&c->tm_xn32, c->xn, T, d, d, 32));
  DG_TRY(make_tmap(&c->tm_xn128, c->xn, T, d, d, 128));
  DG_TRY(make_tmap(&c->tm_o32, c->o, T, g.n_heads * hd, g.n_heads * hd, 32));
  // expert GEMM operands: bf16, or e4m3 / e2m1 codes (maps over bytes: K or K / 2 columns)
  // with rows at the 128-byte pitch
  const bool q8 = c->fmt != 0;
  const int eb = q8 ? 1 : 2;
  auto mcols = [&](int kk) { return static_cast<uint64_t>(c->fmt == 2 ? kk / 2 : kk); };
  auto mpitch = [&](int kk) {
    return static_cast<uint64_t>(q8 ? operand_row_bytes(c->fmt, kk) : kk);
  };
  DG_TRY(make_tmap(&c->tm_xperm, c->x_perm, T * k, mcols(d), mpitch(d), 32, eb));
  DG_TRY(make_tmap(&c->tm_h, q8 ? c->hq : c->h, T * k, mcols(g.expert_hidden),
                   mpitch(g.expert_hidden), 32, eb));
  if (g.shared_hidden > 0)
    DG_TRY(make_tmap(&c->tm_hs, q8 ? c->hsq : c->hs, T, mcols(g.shared_hidden),
                     mpitch(g.shared_hidden), 32, eb));
  if (q8) DG_TRY(make_tmap(&c->tm_xsh, c->x_sh, T, mcols(d), mpitch(d), 32, 1));
  DG_TRY(make_tmap(&c->tm_q, c->q, static_cast<uint64_t>(g.n_heads) * c->tq, hd, hd, 128));
  // every (sequence, layer) pair of a batched context is one more layer block of the cache
  const uint64_t kv_rows =
      static_cast<uint64_t>(c->batch) * g.n_layers * g.n_kv_heads * g.kv_capacity;
  DG_TRY(make_tmap(&c->tm_k, c->kc, kv_rows, hd, hd, 128));
  const uint64_t vt_rows = static_cast<uint64_t>(c->batch) * g.n_layers * g.n_kv_heads * hd;
  DG_TRY(make_tmap(&c->tm_vt, c->vtc, vt_rows, g.kv_capacity, g.kv_capacity, 128));
  DG_TRY(make_tmap(&c->tm_embed, c->embed, g.vocab, d, d, 256));
  if (g.lm_head_e4m3) {
    const uint64_t hp = e4m3_pitch(g.d_model);
    DG_TRY(make_tmap(&c->tm_xhq, c->xhq, static_cast<uint64_t>(g.canvas) * c->batch, d, hp, 128, 1));
    DG_TRY(make_tmap(&c->tm_ehq, c->head_codes, g.vocab, d, hp, 256, 1));
  }
  const int L = g.n_layers;
  c->tm_wqkv.resize(L);
  c->tm_wo.resize(L);
  c->tm_wr.resize(L);
  c->tm_wgu.resize(L);
  c->tm_wd.resize(L);
  c->tm_wsgu.resize(L);
  c->tm_wsd.resize(L);
  for (int l = 0; l < L; ++l) {
    const dg_layer_weights& w = c->layers[l];
    DG_TRY(make_tmap(&c->tm_wqkv[l], w.wqkv, c->qkv_rows, d, d, 128));
    DG_TRY(make_tmap(&c->tm_wo[l], w.wo, d, g.n_heads * hd, g.n_heads * hd, 128));
    DG_TRY(make_tmap(&c->tm_wr[l], w.wr, g.n_experts, d, d, 128));
    DG_TRY(make_tmap(&c->tm_wgu[l], w.w_gu, static_cast<uint64_t>(g.n_experts) * 2 * g.expert_hidden,
                     mcols(d), mpitch(d), 128, eb));
    DG_TRY(make_tmap(&c->tm_wd[l], w.w_d, static_cast<uint64_t>(g.n_experts) * d,
                     mcols(g.expert_hidden), mpitch(g.expert_hidden), 128, eb));
    if (g.shared_hidden > 0) {
      DG_TRY(make_tmap(&c->tm_wsgu[l], w.ws_gu, 2ull * g.shared_hidden, mcols(d), mpitch(d), 128,
                       eb));
      DG_TRY(make_tmap(&c->tm_wsd[l], w.ws_d, d, mcols(g.shared_hidden), mpitch(g.shared_hidden),
                       128, eb));
    }
  }
  return DG_OK;
}

int check_ctx(const dg_ctx* c) {
  if (!c) return fail(DG_ERR_INVALID_ARG, "null context");
  return DG_OK;
}

}  // namespace

// =======================================================================================
extern "C" {

const char* dg_last_error(void) { return g_last_error.c_str(); }
const char* dg_version(void) { return "libdg 0.1 sm_100a"; }

uint64_t dg_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int dg_profile_kernel(int32_t kernel_kind, int32_t n_pairs) {
  if (n_pairs < 0 || n_pairs > (1 << 20) ||
      (n_pairs > 0 && (kernel_kind < 0 || kernel_kind >= DG_KERNEL_KINDS)))
    return fail(DG_ERR_INVALID_ARG, "bad profile request");
  for (cudaEvent_t e : g_prof.events)
    if (e) cudaEventDestroy(e);
  g_prof.events.assign(2 * static_cast<size_t>(n_pairs), nullptr);
  for (auto& e : g_prof.events) DG_CUDA(cudaEventCreate(&e));
  g_prof.kind = n_pairs > 0 ? kernel_kind : -1;
  g_prof.n_pairs = n_pairs;
  g_prof.recorded = 0;
  return DG_OK;
}

int32_t dg_profile_read(float* durations_ms, int32_t max_pairs) {
  if (!durations_ms || max_pairs < 0) return fail(DG_ERR_INVALID_ARG, "bad profile read");
  const int n = std::min(max_pairs, g_prof.recorded);
  for (int i = 0; i < n; ++i) {
    DG_CUDA(cudaEventSynchronize(g_prof.events[2 * i + 1]));
    DG_CUDA(cudaEventElapsedTime(&durations_ms[i], g_prof.events[2 * i], g_prof.events[2 * i + 1]));
  }
  return n;
}

int dg_workspace_bytes(const dg_config* cfg, size_t* kv_bytes, size_t* scratch_bytes) {
  DG_TRY(check_config(cfg));
  if (!kv_bytes || !scratch_bytes) return fail(DG_ERR_INVALID_ARG, "null output pointer");
  const Plan p = plan(*cfg, num_sms());
  *kv_bytes = p.kv;
  *scratch_bytes = p.total;
  return DG_OK;
}

int dg_create(const dg_config* cfg, const dg_weights* w, void* d_kv, void* d_scratch, void* stream,
              dg_ctx** out) {
  DG_TRY(check_config(cfg));
  if (!w || !w->embed || !w->final_norm || !w->layers || !d_kv || !d_scratch || !out)
    return fail(DG_ERR_INVALID_ARG, "null weights or buffers");
  if (cfg->lm_head_e4m3 && (!w->head_codes || !w->head_scale ||
                            reinterpret_cast<uintptr_t>(w->head_codes) % 16))
    return fail(DG_ERR_INVALID_ARG, "lm_head_e4m3 needs 16-byte aligned head codes and scales");
  if (reinterpret_cast<uintptr_t>(d_kv) % 256 || reinterpret_cast<uintptr_t>(d_scratch) % 256)
    return fail(DG_ERR_INVALID_ARG, "kv and scratch must be 256-byte aligned");
  for (int l = 0; l < cfg->n_layers; ++l) {
    const dg_layer_weights& lw = w->layers[l];
    if (!lw.attn_norm || !lw.wqkv || !lw.wo || !lw.ffn_norm || !lw.wr || !lw.w_gu || !lw.w_d)
      return fail(DG_ERR_INVALID_ARG, "layer %d has a null weight", l);
    if (cfg->shared_hidden > 0 && (!lw.ws_gu || !lw.ws_d))
      return fail(DG_ERR_INVALID_ARG, "layer %d lacks shared expert weights", l);
    if ((cfg->dtype == DG_DTYPE_BF16_E4M3 || cfg->dtype == DG_DTYPE_BF16_NVFP4) &&
        (!lw.w_gu_scale || !lw.w_d_scale ||
         (cfg->shared_hidden > 0 && (!lw.ws_gu_scale || !lw.ws_d_scale))))
      return fail(DG_ERR_INVALID_ARG, "layer %d lacks e4m3 expert scales", l);
    if (cfg->dtype == DG_DTYPE_BF16_NVFP4 &&
        (!lw.w_gu_sf || !lw.w_d_sf || (cfg->shared_hidden > 0 && (!lw.ws_gu_sf || !lw.ws_d_sf))))
      return fail(DG_ERR_INVALID_ARG, "layer %d lacks NVFP4 block-scale atoms", l);
  }
  dg_ctx* c = new dg_ctx();
  c->cfg = *cfg;
  c->layers.assign(w->layers, w->layers + cfg->n_layers);
  c->embed = w->embed;
  c->final_norm = w->final_norm;
  c->head_codes = w->head_codes;
  c->head_scale = w->head_scale;
  c->kv = static_cast<uint8_t*>(d_kv);
  c->scratch = static_cast<uint8_t*>(d_scratch);
  c->kv_len = 0;
  c->sms = num_sms();
  c->batch = n_seq(*cfg);
  c->bf16 = cfg->dtype != DG_DTYPE_FP32;
  c->fmt = cfg->dtype == DG_DTYPE_BF16_E4M3 ? 1 : cfg->dtype == DG_DTYPE_BF16_NVFP4 ? 2 : 0;
  const Derived dv = derive(*cfg, c->sms);
  c->esz = dv.esz;
  c->tq = dv.tq;
  c->qkv_rows = dv.qkv_rows;
  c->split_r = dv.split_r;
  c->att_splits_max = dv.att_splits;
  c->part_elems = dv.part_elems;
  const Plan p = plan(*cfg, c->sms);
  uint8_t* s = c->scratch;
  c->canvas = reinterpret_cast<int32_t*>(s + p.off[B_CANVAS]);
  c->argmax = reinterpret_cast<int32_t*>(s + p.off[B_ARGMAX]);
  c->prev_argmax = reinterpret_cast<int32_t*>(s + p.off[B_PREV]);
  c->locked = reinterpret_cast<int32_t*>(s + p.off[B_LOCKED]);
  c->state = reinterpret_cast<int32_t*>(s + p.off[B_STATE]);
  c->all_done = c->state + static_cast<size_t>(c->batch) * kStWords;
  c->ticket = reinterpret_cast<int32_t*>(s + p.off[B_TICKET]);
  c->err = reinterpret_cast<int32_t*>(s + p.off[B_ERR]);
  c->entropy = reinterpret_cast<float*>(s + p.off[B_ENT]);
  c->conf = reinterpret_cast<float*>(s + p.off[B_CONF]);
  c->row_h = reinterpret_cast<double*>(s + p.off[B_ROWH]);
  c->x = reinterpret_cast<float*>(s + p.off[B_X]);
  c->xn = s + p.off[B_XN];
  c->part = reinterpret_cast<float*>(s + p.off[B_PART]);
  c->q = s + p.off[B_Q];
  c->o_part = reinterpret_cast<float*>(s + p.off[B_OPART]);
  c->ml_part = reinterpret_cast<float2*>(s + p.off[B_ML]);
  c->o = s + p.off[B_O];
  c->router_logits = reinterpret_cast<float*>(s + p.off[B_RLOG]);
  c->topk_ids = reinterpret_cast<int32_t*>(s + p.off[B_IDS]);
  c->topk_w = reinterpret_cast<float*>(s + p.off[B_W]);
  c->offsets = reinterpret_cast<int32_t*>(s + p.off[B_OFF]);
  c->perm = reinterpret_cast<int32_t*>(s + p.off[B_PERM]);
  c->chunks = reinterpret_cast<int4*>(s + p.off[B_CHUNKS]);
  c->n_chunks = reinterpret_cast<int32_t*>(s + p.off[B_NCHUNKS]);
  c->route_ticket = reinterpret_cast<int32_t*>(s + p.off[B_RTICKET]);
  c->x_perm = s + p.off[B_XPERM];
  c->h = s + p.off[B_H];
  c->hs = s + p.off[B_HS];
  c->y_slot = reinterpret_cast<float*>(s + p.off[B_YSLOT]);
  c->y_shared = reinterpret_cast<float*>(s + p.off[B_YSH]);
  c->lm_part = reinterpret_cast<StatPartial*>(s + p.off[B_LMPART]);
  c->logits = reinterpret_cast<float*>(s + p.off[B_LOGITS]);
  c->rope_tab = reinterpret_cast<float2*>(s + p.off[B_ROPE]);
  c->x_perm_scale = reinterpret_cast<float*>(s + p.off[B_XPS]);
  c->x_sh = s + p.off[B_XSH];
  c->x_sh_scale = reinterpret_cast<float*>(s + p.off[B_XSHS]);
  c->hq = s + p.off[B_HQ];
  c->hq_scale = reinterpret_cast<float*>(s + p.off[B_HQS]);
  c->hsq = s + p.off[B_HSQ];
  c->hsq_scale = reinterpret_cast<float*>(s + p.off[B_HSQS]);
  c->w_perm = reinterpret_cast<float*>(s + p.off[B_WPERM]);
  c->commit_ids = reinterpret_cast<int32_t*>(s + p.off[B_COMMIT]);
  c->xhq = s + p.off[B_XHQ];
  c->xhs = reinterpret_cast<float*>(s + p.off[B_XHS]);
  c->x_sf = s + p.off[B_XSF];
  c->x_sh_sf = s + p.off[B_XSHSF];
  c->h_sf = s + p.off[B_HSF];
  c->hs_sf = s + p.off[B_HSSF];
  const size_t kv_half = p.kv / 2;
  c->kc = c->kv;
  c->vtc = c->kv + kv_half;
  if (c->bf16) {
    const int rc = bind_tmaps(c);
    if (rc != DG_OK) {
      delete c;
      return rc;
    }
  }
  cudaStream_t st = S(stream);
  cudaError_t e = cudaMemsetAsync(c->kv, 0, p.kv, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->scratch, 0, p.total, st);
  if (e != cudaSuccess) {
    delete c;
    return fail(DG_ERR_CUDA, "memset failed: %s", cudaGetErrorString(e));
  }
  const int half = cfg->head_dim / 2;
  const long long n_tab = static_cast<long long>(cfg->kv_capacity) * half;
  DG_TRY(launch_pdl(rope_table_kernel, dim3(cdiv(n_tab, 256)), dim3(256), 0, st, c->rope_tab, cfg->kv_capacity, half,
                                                       static_cast<double>(cfg->rope_theta)));
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    delete c;
    return fail(DG_ERR_CUDA, "rope table launch failed: %s", cudaGetErrorString(e));
  }
  *out = c;
  return DG_OK;
}

void dg_destroy(dg_ctx* ctx) { delete ctx; }

int32_t dg_kv_length(const dg_ctx* ctx) { return ctx ? ctx->kv_len : -1; }

int dg_kv_truncate(dg_ctx* ctx, int32_t length) {
  DG_TRY(check_ctx(ctx));
  if (length < 0 || length > ctx->kv_len)
    return fail(DG_ERR_INVALID_ARG, "truncate length %d outside [0, %d]", length, ctx->kv_len);
  ctx->kv_len = length;
  return DG_OK;
}

int dg_kv_append(dg_ctx* ctx, const int32_t* d_ids, int32_t n, void* stream) {
  DG_TRY(check_ctx(ctx));
  if (!d_ids || n <= 0) return fail(DG_ERR_INVALID_ARG, "need ids and n > 0");
  if (static_cast<long long>(ctx->kv_len) + n + ctx->cfg.canvas > ctx->cfg.kv_capacity)
    return fail(DG_ERR_CAPACITY, "cache of %d positions cannot take %d more plus a canvas of %d",
                ctx->cfg.kv_capacity, ctx->kv_len + n, ctx->cfg.canvas);
  cudaStream_t st = S(stream);
  const int chunk = ctx->cfg.prefill_chunk > 0 ? ctx->cfg.prefill_chunk : ctx->cfg.canvas;
  // every sequence's prompt (row b of d_ids) into its own cache, in passes of `chunk` tokens
  for (int b = 0; b < ctx->batch; ++b)
    for (int off = 0; off < n; off += chunk) {
      const int m = std::min(chunk, n - off);
      DG_TRY(run_forward(ctx, d_ids + static_cast<size_t>(b) * n + off, m, ctx->kv_len + off, 1,
                         nullptr, st, b, 0));
    }
  ctx->kv_len += n;
  return DG_OK;
}

int dg_canvas_init(dg_ctx* ctx, uint64_t seed, uint32_t block, void* stream) {
  DG_TRY(check_ctx(ctx));
  if (ctx->kv_len + ctx->cfg.canvas > ctx->cfg.kv_capacity)
    return fail(DG_ERR_CAPACITY, "no room for a canvas after %d committed positions", ctx->kv_len);
  ctx->seed = seed;
  ctx->block = block;
  DG_TRY(launch_pdl(canvas_init_kernel, dim3(cdiv(ctx->cfg.canvas * ctx->batch, 256)), dim3(256),
      0, S(stream), ctx->canvas, ctx->cfg.canvas, ctx->batch, ctx->cfg.vocab, seed, block,
      ctx->state, ctx->ticket, ctx->locked, ctx->all_done));
  DG_LAUNCHED();
  return DG_OK;
}

int dg_reset_block(dg_ctx* ctx, void* stream) {
  DG_TRY(check_ctx(ctx));
  DG_TRY(launch_pdl(block_reset_kernel, dim3(cdiv(ctx->cfg.canvas * ctx->batch, 256)), dim3(256),
                    0, S(stream), ctx->state, ctx->ticket, ctx->locked, ctx->cfg.canvas,
                    ctx->batch, ctx->all_done));
  DG_LAUNCHED();
  return DG_OK;
}

int dg_denoise_step(dg_ctx* ctx, uint32_t step, void* stream) {
  DG_TRY(check_ctx(ctx));
  if (step < 1) return fail(DG_ERR_INVALID_ARG, "steps are numbered from 1");
  if (ctx->kv_len + ctx->cfg.canvas > ctx->cfg.kv_capacity)
    return fail(DG_ERR_CAPACITY, "no room for the canvas");
  cudaStream_t st = S(stream);
  // a no-op on the device once every canvas has stopped
  const int* done = ctx->all_done;
  DG_TRY(run_forward(ctx, ctx->canvas, ctx->cfg.canvas * ctx->batch, ctx->kv_len, 0, done, st, 0,
                     ctx->cfg.canvas));
  DG_TRY(run_lm_head(ctx, nullptr, done, st));
  return DG_OK;
}

int dg_sample_update(dg_ctx* ctx, uint32_t step, void* stream) {
  DG_TRY(check_ctx(ctx));
  if (step < 1) return fail(DG_ERR_INVALID_ARG, "steps are numbered from 1");
  const dg_config& g = ctx->cfg;
  SamplerArgs a{};
  a.partials = ctx->lm_part;
  a.nsplit = ctx->bf16 ? g.vocab / 256 : cdiv(g.vocab, 4096);
  a.rows = g.canvas;
  a.vocab = g.vocab;
  a.seed = ctx->seed;
  a.block = ctx->block;
  a.step = step;
  a.tau = g.tau;
  a.h_bound = g.h_bound;
  a.lock_rule = g.lock_rule;
  a.entropy_lock = static_cast<float>(g.entropy_lock);
  a.sticky = g.sticky_locks;
  a.max_steps = g.max_steps;
  a.fixed_steps = g.fixed_steps;
  a.canvas = ctx->canvas;
  a.argmax = ctx->argmax;
  a.prev_argmax = ctx->prev_argmax;
  a.entropy = ctx->entropy;
  a.conf = ctx->conf;
  a.row_h = ctx->row_h;
  a.locked = ctx->locked;
  a.state = ctx->state;
  a.ticket = ctx->ticket;
  a.n_seq = ctx->batch;
  a.all_done = ctx->all_done;
  prof_before(DG_KERNEL_SAMPLER, S(stream));
  DG_TRY(launch_pdl(sampler_merge_kernel, dim3(g.canvas * ctx->batch), dim3(256), 0, S(stream), a));
  DG_LAUNCHED();
  prof_after(DG_KERNEL_SAMPLER, S(stream));
  return DG_OK;
}

int dg_commit_block(dg_ctx* ctx, int32_t* d_out_ids, int32_t* d_state, void* stream) {
  DG_TRY(check_ctx(ctx));
  const dg_config& g = ctx->cfg;
  if (ctx->kv_len + g.canvas > g.kv_capacity) return fail(DG_ERR_CAPACITY, "cache full");
  cudaStream_t st = S(stream);
  // the committed ids: the argmax of the stop step, or with sticky locks the locked tokens
  const int n_tok = g.canvas * ctx->batch;
  const int32_t* ids = ctx->argmax;
  if (g.sticky_locks) {
    DG_TRY(launch_pdl(commit_ids_kernel, dim3(cdiv(n_tok, 256)), dim3(256), 0, st,
                      static_cast<const int32_t*>(ctx->canvas),
                      static_cast<const int32_t*>(ctx->argmax),
                      static_cast<const int32_t*>(ctx->locked), ctx->commit_ids, n_tok));
    DG_LAUNCHED();
    ids = ctx->commit_ids;
  }
  if (d_out_ids)
    DG_CUDA(cudaMemcpyAsync(d_out_ids, ids, static_cast<size_t>(n_tok) * 4,
                            cudaMemcpyDeviceToDevice, st));
  if (d_state)
    DG_CUDA(cudaMemcpyAsync(d_state, ctx->state, static_cast<size_t>(ctx->batch) * kStWords * 4,
                            cudaMemcpyDeviceToDevice, st));
  // re-encode causally (every sequence's block into its own cache), or keep the canvas K/V the
  // last denoise step left in slots P..P+T-1
  if (!g.commit_reuse_kv)
    DG_TRY(run_forward(ctx, ids, n_tok, ctx->kv_len, 1, nullptr, st, 0, g.canvas));
  ctx->kv_len += g.canvas;
  return DG_OK;
}

int dg_get_buffers(const dg_ctx* ctx, int32_t** canvas, int32_t** argmax, float** entropy,
                   float** conf, int32_t** state) {
  DG_TRY(check_ctx(ctx));
  if (canvas) *canvas = ctx->canvas;
  if (argmax) *argmax = ctx->argmax;
  if (entropy) *entropy = ctx->entropy;
  if (conf) *conf = ctx->conf;
  if (state) *state = ctx->state;
  return DG_OK;
}

int dg_check_device_status(dg_ctx* ctx, void* stream) {
  DG_TRY(check_ctx(ctx));
  DG_CUDA(cudaStreamSynchronize(S(stream)));
  int err = 0;
  DG_CUDA(cudaMemcpy(&err, ctx->err, 4, cudaMemcpyDeviceToHost));
  if (err == kDevErrBadId)
    return fail(DG_ERR_INVALID_ARG, "a token id outside [0, %d) reached the embedding",
                ctx->cfg.vocab);
  if (err != 0) return fail(DG_ERR_TIMEOUT, "a device wait gave up (code %d)", err);
  return DG_OK;
}

int dg_debug_logits(dg_ctx* ctx, float* d_logits, void* stream) {
  DG_TRY(check_ctx(ctx));
  if (!d_logits) return fail(DG_ERR_INVALID_ARG, "null logits");
  return run_lm_head(ctx, d_logits, nullptr, S(stream));
}

int dg_debug_routing(const dg_ctx* ctx, int32_t** d_ids, float** d_weights,
                     float** d_router_logits) {
  DG_TRY(check_ctx(ctx));
  if (d_ids) *d_ids = ctx->topk_ids;
  if (d_weights) *d_weights = ctx->topk_w;
  if (d_router_logits) *d_router_logits = ctx->router_logits;
  return DG_OK;
}

int dg_debug_layer_part(dg_ctx* ctx, int32_t layer, int32_t part, const float* d_x_in,
                        float* d_x_out, int32_t n, int32_t causal, void* stream) {
  DG_TRY(check_ctx(ctx));
  const dg_config& g = ctx->cfg;
  if (layer < 0 || layer >= g.n_layers) return fail(DG_ERR_INVALID_ARG, "bad layer %d", layer);
  if (part != 0 && part != 1) return fail(DG_ERR_INVALID_ARG, "part must be 0 or 1");
  // a batched context runs the layer over all its canvases' tokens (n = batch * canvas)
  const int seq_len = ctx->batch > 1 ? g.canvas : 0;
  if (!d_x_in || !d_x_out || n < 1 || (seq_len ? n != g.canvas * ctx->batch : n > g.canvas))
    return fail(DG_ERR_INVALID_ARG, "need x_in, x_out and 1 <= n <= canvas (batch * canvas)");
  // every sequence writes its own tokens' K/V at positions P.. of its own cache
  if (ctx->kv_len + (seq_len ? seq_len : n) > g.kv_capacity)
    return fail(DG_ERR_CAPACITY, "cache full");
  cudaStream_t st = S(stream);
  DG_CUDA(cudaMemcpyAsync(ctx->x, d_x_in, static_cast<size_t>(n) * g.d_model * 4,
                          cudaMemcpyDeviceToDevice, st));
  const float* w = part == 0 ? ctx->layers[layer].attn_norm : ctx->layers[layer].ffn_norm;
  const bool q8 = part == 1 && ctx->fmt == 1;  // the MoE half's token operand, as in run_layer
  if (ctx->bf16)
    DG_TRY(launch_pdl(q8 ? residual_norm_kernel<__nv_bfloat16, true>
                         : residual_norm_kernel<__nv_bfloat16, false>, dim3(n), dim3(256), 0, st,
        ctx->x, ctx->part, 0, 0, g.d_model, w, g.eps, static_cast<__nv_bfloat16*>(ctx->xn),
        q8 ? static_cast<uint8_t*>(ctx->x_sh) : nullptr,
        static_cast<int>(operand_row_bytes(1, g.d_model)), q8 ? ctx->x_sh_scale : nullptr, nullptr));
  else
    DG_TRY(launch_pdl(residual_norm_kernel<float>, dim3(n), dim3(256), 0, st, ctx->x, ctx->part, 0, 0, g.d_model, w, g.eps,
                                                   static_cast<float*>(ctx->xn), nullptr, 0, nullptr, nullptr));
  DG_LAUNCHED();
  const float* nn = (layer + 1 < g.n_layers) ? ctx->layers[layer + 1].attn_norm : ctx->final_norm;
  DG_TRY(run_layer(ctx, layer, n, ctx->kv_len, causal, nn, nullptr, st, part == 0 ? 1 : 2, 0,
                   seq_len));
  DG_CUDA(cudaMemcpyAsync(d_x_out, ctx->x, static_cast<size_t>(n) * g.d_model * 4,
                          cudaMemcpyDeviceToDevice, st));
  return DG_OK;
}

int dg_debug_tensors(const dg_ctx* ctx, void** d_q, void** d_o, void** d_xn) {
  DG_TRY(check_ctx(ctx));
  if (d_q) *d_q = ctx->q;
  if (d_o) *d_o = ctx->o;
  if (d_xn) *d_xn = ctx->xn;
  return DG_OK;
}

int dg_debug_hidden(const dg_ctx* ctx, float** d_x) {
  DG_TRY(check_ctx(ctx));
  if (!d_x) return fail(DG_ERR_INVALID_ARG, "null output");
  *d_x = ctx->x;
  return DG_OK;
}

int dg_debug_layer(dg_ctx* ctx, int32_t layer, const float* d_x_in, float* d_x_out, int32_t n,
                   int32_t causal, void* stream) {
  DG_TRY(check_ctx(ctx));
  const dg_config& g = ctx->cfg;
  if (layer < 0 || layer >= g.n_layers) return fail(DG_ERR_INVALID_ARG, "bad layer %d", layer);
  // a batched context runs the layer over all its canvases' tokens (n = batch * canvas)
  const int seq_len = ctx->batch > 1 ? g.canvas : 0;
  if (!d_x_in || !d_x_out || n < 1 || (seq_len ? n != g.canvas * ctx->batch : n > g.canvas))
    return fail(DG_ERR_INVALID_ARG, "need x_in, x_out and 1 <= n <= canvas (batch * canvas)");
  // every sequence writes its own tokens' K/V at positions P.. of its own cache
  if (ctx->kv_len + (seq_len ? seq_len : n) > g.kv_capacity)
    return fail(DG_ERR_CAPACITY, "cache full");
  cudaStream_t st = S(stream);
  DG_CUDA(cudaMemcpyAsync(ctx->x, d_x_in, static_cast<size_t>(n) * g.d_model * 4,
                          cudaMemcpyDeviceToDevice, st));
  const float* w = ctx->layers[layer].attn_norm;
  if (ctx->bf16)
    DG_TRY(launch_pdl(residual_norm_kernel<__nv_bfloat16>, dim3(n), dim3(256), 0, st,
        ctx->x, ctx->part, 0, 0, g.d_model, w, g.eps, static_cast<__nv_bfloat16*>(ctx->xn),
        nullptr, 0, nullptr, nullptr));
  else
    DG_TRY(launch_pdl(residual_norm_kernel<float>, dim3(n), dim3(256), 0, st, ctx->x, ctx->part, 0, 0, g.d_model, w, g.eps,
                                                   static_cast<float*>(ctx->xn), nullptr, 0, nullptr, nullptr));
  DG_LAUNCHED();
  const float* nn = (layer + 1 < g.n_layers) ? ctx->layers[layer + 1].attn_norm : ctx->final_norm;
  DG_TRY(run_layer(ctx, layer, n, ctx->kv_len, causal, nn, nullptr, st, 3, 0, seq_len));
  DG_CUDA(cudaMemcpyAsync(d_x_out, ctx->x, static_cast<size_t>(n) * g.d_model * 4,
                          cudaMemcpyDeviceToDevice, st));
  return DG_OK;
}

// ---- standalone sampler ----------------------------------------------------------------

// The streaming sampler cuts rows into segments of stream_span<T>() columns (2048 for bf16, 1024
// for fp32); the workspace holds one partial per segment at the finer of the two.
static size_t sampler_segs_max(int vocab) { return cdiv(vocab, stream_span<float>()); }

int dg_sampler_workspace_bytes(int32_t rows, int32_t vocab, size_t* bytes) {
  if (rows < 1 || rows > 1024 || vocab < 2 || vocab % 8 || !bytes)
    return fail(DG_ERR_INVALID_ARG, "need 1 <= rows <= 1024, vocab % 8 == 0");
  *bytes = align256(rows * sampler_segs_max(vocab) * sizeof(StatPartial)) + 3 * align256(rows * 8) +
           256;
  return DG_OK;
}

static void sampler_views(void* ws, int rows, int vocab, StatPartial** part, int32_t** prev,
                          double** row_h, int32_t** locked, int32_t** ticket) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  *part = reinterpret_cast<StatPartial*>(b);
  b += align256(rows * sampler_segs_max(vocab) * sizeof(StatPartial));
  *prev = reinterpret_cast<int32_t*>(b);
  b += align256(rows * 8);
  *row_h = reinterpret_cast<double*>(b);
  b += align256(rows * 8);
  *locked = reinterpret_cast<int32_t*>(b);
  b += align256(rows * 8);
  *ticket = reinterpret_cast<int32_t*>(b);
}

int dg_sampler_reset(int32_t rows, int32_t vocab, void* d_workspace, int32_t* d_state,
                     void* stream) {
  size_t bytes = 0;
  DG_TRY(dg_sampler_workspace_bytes(rows, vocab, &bytes));
  if (!d_workspace || !d_state) return fail(DG_ERR_INVALID_ARG, "null workspace or state");
  DG_CUDA(cudaMemsetAsync(d_workspace, 0, bytes, S(stream)));
  DG_CUDA(cudaMemsetAsync(d_state, 0, kStWords * 4, S(stream)));
  return DG_OK;
}

int dg_sampler_step(const void* d_logits, int32_t dtype, int32_t rows, int32_t vocab, uint64_t seed,
                    uint32_t block, uint32_t step, double tau, double h_bound, int32_t max_steps,
                    int32_t fixed_steps, void* d_workspace, int32_t* d_canvas, int32_t* d_argmax,
                    float* d_entropy, float* d_conf, int32_t* d_state, void* stream) {
  size_t bytes = 0;
  DG_TRY(dg_sampler_workspace_bytes(rows, vocab, &bytes));
  if (!d_logits || !d_workspace || !d_canvas || !d_argmax || !d_entropy || !d_conf || !d_state)
    return fail(DG_ERR_INVALID_ARG, "null pointer argument");
  if (reinterpret_cast<uintptr_t>(d_logits) % 16)
    return fail(DG_ERR_INVALID_ARG, "logits must be 16-byte aligned");
  if (step < 1 || max_steps < 1 || fixed_steps < 0)
    return fail(DG_ERR_INVALID_ARG, "bad step / max_steps / fixed_steps");
  if (dtype != DG_DTYPE_BF16 && dtype != DG_DTYPE_FP32)
    return fail(DG_ERR_INVALID_ARG, "dtype must be bf16 or fp32");
  StatPartial* part;
  int32_t *prev, *locked, *ticket;
  double* row_h;
  sampler_views(d_workspace, rows, vocab, &part, &prev, &row_h, &locked, &ticket);
  cudaStream_t st = S(stream);
  const bool bf16 = dtype == DG_DTYPE_BF16;
  const int segs = cdiv(vocab, bf16 ? stream_span<__nv_bfloat16>() : stream_span<float>());
  SamplerArgs a{};
  a.partials = part;
  a.nsplit = segs;
  a.rows = rows;
  a.vocab = vocab;
  a.seed = seed;
  a.block = block;
  a.step = step;
  a.tau = tau;
  a.h_bound = h_bound;
  a.max_steps = max_steps;
  a.fixed_steps = fixed_steps;
  a.canvas = d_canvas;
  a.argmax = d_argmax;
  a.prev_argmax = prev;
  a.entropy = d_entropy;
  a.conf = d_conf;
  a.row_h = row_h;
  a.locked = locked;
  a.state = d_state;
  a.ticket = ticket;
  a.n_seq = 1;
  // one wave of resident CTAs; each of their warps streams an equal run of segments, then one
  // warp per row merges the row
  static const int grid_bf16 = resident_ctas(sampler_stream_kernel<__nv_bfloat16>);
  static const int grid_f32 = resident_ctas(sampler_stream_kernel<float>);
  const long long units = static_cast<long long>(rows) * segs;
  const int grid = static_cast<int>(std::min<long long>(cdiv(units, 8), bf16 ? grid_bf16 : grid_f32));
  const long long workers = static_cast<long long>(grid) * 8;
  prof_before(DG_KERNEL_SAMPLER, st);
  if (bf16) {
    const auto* x = static_cast<const __nv_bfloat16*>(d_logits);
    DG_TRY(launch_pdl(sampler_stream_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, x, segs, a));
    DG_LAUNCHED();
    DG_TRY(launch_pdl(sampler_stream_rows_kernel<__nv_bfloat16>, dim3(cdiv(rows, 8)), dim3(256), 0,
                      st, x, segs, a, workers));
  } else {
    const auto* x = static_cast<const float*>(d_logits);
    DG_TRY(launch_pdl(sampler_stream_kernel<float>, dim3(grid), dim3(256), 0, st, x, segs, a));
    DG_LAUNCHED();
    DG_TRY(launch_pdl(sampler_stream_rows_kernel<float>, dim3(cdiv(rows, 8)), dim3(256), 0, st, x,
                      segs, a, workers));
  }
  DG_LAUNCHED();
  prof_after(DG_KERNEL_SAMPLER, st);
  return DG_OK;
}

// ---- standalone attention --------------------------------------------------------------
int dg_attention_workspace_bytes(int32_t n_heads, int32_t n_kv_heads, int32_t tq, int32_t n_keys,
                                 size_t* bytes) {
  if (n_heads < 1 || n_kv_heads < 1 || tq < 128 || tq % 128 || n_keys < 1 || !bytes)
    return fail(DG_ERR_INVALID_ARG, "bad attention shape");
  const int splits = std::max(1, cdiv(n_keys, 128));
  *bytes = align256(static_cast<size_t>(splits) * n_heads * tq * 128 * 4) +
           align256(static_cast<size_t>(splits) * n_heads * tq * 8) +
           align256(static_cast<size_t>(n_heads) * tq / 128 * 4) + 4 * 256;
  return DG_OK;
}

int dg_canvas_attention(const void* d_q, const void* d_k, const void* d_vt, void* d_o,
                        int32_t n_heads, int32_t n_kv_heads, int32_t t, int32_t tq, int32_t n_keys,
                        int32_t ldk, int32_t causal_prefix, float scale, void* d_workspace,
                        size_t workspace_bytes, void* stream) {
  if (!d_q || !d_k || !d_vt || !d_o || !d_workspace) return fail(DG_ERR_INVALID_ARG, "null pointer");
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads || t < 1 || tq < t || tq % 128 ||
      n_keys < 1 || ldk < n_keys || ldk % 8)
    return fail(DG_ERR_INVALID_ARG, "bad attention shape");
  if (causal_prefix >= 0 && causal_prefix + t > n_keys)
    return fail(DG_ERR_INVALID_ARG, "causal prefix + queries exceeds keys");
  const int sms = num_sms();
  const int group = n_heads / n_kv_heads;
  const int tph = cdiv(t, 128);  // query tiles per head in use
  const int m_tiles = group * tph;
  const int n_kv_tiles = cdiv(n_keys, 128);
  int splits = std::max(1, std::min(kMaxAttnSplits, sms / (m_tiles * n_kv_heads)));
  splits = std::min(splits, n_kv_tiles);
  const int tps = cdiv(n_kv_tiles, splits);
  splits = cdiv(n_kv_tiles, tps);
  const size_t o_bytes = align256(static_cast<size_t>(splits) * n_heads * tq * 128 * 4);
  const size_t ml_bytes = align256(static_cast<size_t>(splits) * n_heads * tq * 8);
  const size_t tk_bytes = align256(static_cast<size_t>(n_kv_heads) * m_tiles * 4);
  const size_t need = o_bytes + ml_bytes + tk_bytes + 256;
  if (workspace_bytes < need) return fail(DG_ERR_CAPACITY, "attention workspace too small");
  uint8_t* ws = static_cast<uint8_t*>(d_workspace);
  CUtensorMap tq_m, tk_m, tv_m;
  DG_TRY(make_tmap(&tq_m, d_q, static_cast<uint64_t>(n_heads) * tq, 128, 128, 128));
  DG_TRY(make_tmap(&tk_m, d_k, static_cast<uint64_t>(n_kv_heads) * ldk, 128, 128, 128));
  DG_TRY(make_tmap(&tv_m, d_vt, static_cast<uint64_t>(n_kv_heads) * 128, ldk, ldk, 128));
  AttnParams a{};
  a.group = group;
  a.tq = tq;
  a.tiles_per_head = tph;
  a.n_queries = t;
  a.n_keys = n_keys;
  a.causal_prefix = causal_prefix;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.tiles_per_split = tps;
  a.q_row_base = 0;
  a.k_row_base = 0;
  a.ldk = ldk;
  a.vt_row_base = 0;
  a.n_heads = n_heads;
  a.o_part = reinterpret_cast<float*>(ws);
  a.ml_part = reinterpret_cast<float2*>(ws + o_bytes);
  a.err = reinterpret_cast<int*>(ws + need - 256);
  a.done = nullptr;
  cudaStream_t st = S(stream);
  DG_CUDA(cudaMemsetAsync(a.err, 0, 4, st));
  a.o = static_cast<__nv_bfloat16*>(d_o);
  DG_TRY(set_smem(attention_kernel, kAttnSmemBytes));
  DG_TRY(launch_pdl_cluster(attention_kernel, dim3(m_tiles, n_kv_heads, splits), dim3(kAttnThreads),
                            kAttnSmemBytes, st, dim3(1, 1, splits), tq_m, tk_m, tv_m, a));
  DG_LAUNCHED();
  return DG_OK;
}

// ---- standalone MoE --------------------------------------------------------------------
namespace {
enum MoeBuf {
  M_RLOG, M_IDS, M_W, M_OFF, M_PERM, M_CHUNKS, M_WORDS, M_XPERM, M_H, M_HS, M_YSH, M_YSLOT,
  M_XPS, M_XSH, M_XSHS, M_HQ, M_HQS, M_HSQ, M_HSQS, M_WPERM, M_XSF, M_XSHSF, M_HSF, M_HSSF,
  M_END
};
struct MoePlan {
  size_t off[M_END];
  size_t total;
  int split_r;
  long long chunks;
};
// Buffers of both expert formats (the e4m3 ones are small next to the bf16 x_perm).
MoePlan moe_plan(int t, int d, int E, int k, int hid, int hs) {
  MoePlan m{};
  m.split_r = std::min(kCluMaxSplits, d / 64);
  m.chunks = E + (static_cast<long long>(t) * k + kGroupN - 1) / kGroupN;
  const size_t T = t, tk = static_cast<size_t>(t) * k, hs1 = std::max(hs, 1);
  size_t sz[M_END];
  sz[M_RLOG] = T * E * 4;     // router logits (internal)
  sz[M_IDS] = tk * 4;         // ids (internal)
  sz[M_W] = tk * 4;           // weights (internal)
  sz[M_OFF] = (E + 1) * 4;    // offsets
  sz[M_PERM] = tk * 4;        // perm
  sz[M_CHUNKS] = m.chunks * 16;  // routed token chunks
  sz[M_WORDS] = 16;           // chunk count, -, error word, route ticket
  sz[M_XPERM] = tk * d * 2;   // x_perm (bf16; e4m3 rows at the 128-byte pitch fit: d >= 128)
  sz[M_H] = tk * hid * 2;     // h
  sz[M_HS] = T * hs1 * 2;     // shared h
  sz[M_YSH] = T * d * 4;      // y_shared
  sz[M_YSLOT] = tk * d * 4;   // y_slot
  sz[M_XPS] = tk * 4;         // e4m3: x_perm row scales
  sz[M_XSH] = T * e4m3_pitch(d);    // e4m3: quantised tokens for the shared expert
  sz[M_XSHS] = T * 4;
  sz[M_HQ] = tk * e4m3_pitch(hid);  // e4m3: quantised h and its scales
  sz[M_HQS] = tk * 4;
  sz[M_HSQ] = T * e4m3_pitch(static_cast<int>(hs1));  // e4m3: quantised shared h, scales
  sz[M_HSQS] = T * 4;
  sz[M_WPERM] = tk * 4;       // route weights in permuted order
  // NVFP4 token-side scale atoms (per routed chunk, per 64-token chunk of the shared expert)
  const size_t tok_chunks = (T + kGroupN - 1) / kGroupN;
  sz[M_XSF] = m.chunks * 4 * cdiv(d, 256) * 512;
  sz[M_XSHSF] = tok_chunks * 4 * cdiv(d, 256) * 512;
  sz[M_HSF] = m.chunks * 4 * cdiv(hid, 256) * 512;
  sz[M_HSSF] = tok_chunks * 4 * cdiv(static_cast<int>(hs1), 256) * 512;
  size_t o = 0;
  for (int i = 0; i < M_END; ++i) {
    m.off[i] = o;
    o += align256(std::max<size_t>(sz[i], 1));
  }
  m.total = o;
  return m;
}

struct MoeScales {
  const float *w_gu, *w_d, *ws_gu, *ws_d;
  const void *w_gu_sf, *w_d_sf, *ws_gu_sf, *ws_d_sf;  // NVFP4 block-scale atoms
};

int moe_ffn_impl(int fmt, const MoeScales& sc, const void* d_x, const float* d_residual,
                 const void* d_wr, const void* d_w_gu, const void* d_w_d, const void* d_ws_gu,
                 const void* d_ws_d, float* d_y, int32_t* d_ids, float* d_weights,
                 float* d_router_logits, int32_t t, int32_t d, int32_t n_experts, int32_t top_k,
                 int32_t hidden, int32_t shared_hidden, void* d_workspace, size_t workspace_bytes,
                 void* stream) {
  size_t need = 0;
  DG_TRY(dg_moe_workspace_bytes(t, d, n_experts, top_k, hidden, shared_hidden, &need));
  if (!d_x || !d_wr || !d_w_gu || !d_w_d || !d_y || !d_workspace)
    return fail(DG_ERR_INVALID_ARG, "null pointer argument");
  if (shared_hidden > 0 && (!d_ws_gu || !d_ws_d))
    return fail(DG_ERR_INVALID_ARG, "shared expert weights missing");
  const bool f8 = fmt != 0;  // quantised expert operands
  if (f8 && (!sc.w_gu || !sc.w_d || (shared_hidden > 0 && (!sc.ws_gu || !sc.ws_d))))
    return fail(DG_ERR_INVALID_ARG, "e4m3 expert scales missing");
  if (fmt == 2 && (!sc.w_gu_sf || !sc.w_d_sf ||
                   (shared_hidden > 0 && (!sc.ws_gu_sf || !sc.ws_d_sf))))
    return fail(DG_ERR_INVALID_ARG, "NVFP4 block-scale atoms missing");
  if (fmt == 2 && d % 128) return fail(DG_ERR_UNSUPPORTED, "NVFP4 experts need d % 128 == 0");
  if (workspace_bytes < need) return fail(DG_ERR_CAPACITY, "MoE workspace too small");
  if (t > 4096) return fail(DG_ERR_UNSUPPORTED, "at most 4096 tokens per call");
  const MoePlan m = moe_plan(t, d, n_experts, top_k, hidden, shared_hidden);
  uint8_t* ws = static_cast<uint8_t*>(d_workspace);
  auto at = [&](int b) { return static_cast<void*>(ws + m.off[b]); };
  float* rlog = static_cast<float*>(at(M_RLOG));
  int32_t* ids = static_cast<int32_t*>(at(M_IDS));
  float* wts = static_cast<float*>(at(M_W));
  int32_t* offs = static_cast<int32_t*>(at(M_OFF));
  int32_t* perm = static_cast<int32_t*>(at(M_PERM));
  int4* chunks = static_cast<int4*>(at(M_CHUNKS));
  int32_t* icnt = static_cast<int32_t*>(at(M_WORDS));
  int* err = icnt + 2;
  int32_t* route_ticket = icnt + 3;
  const int sms = num_sms();
  cudaStream_t st = S(stream);
  DG_CUDA(cudaMemsetAsync(err, 0, 8, st));  // error word and route ticket
  const int eb = f8 ? 1 : 2;
  // operand maps: bf16, or e4m3 / e2m1 codes over bytes (K or K / 2 columns) at 128-byte pitches
  auto mc = [&](int kk) { return static_cast<uint64_t>(fmt == 2 ? kk / 2 : kk); };
  auto mp = [&](int kk) { return static_cast<uint64_t>(f8 ? operand_row_bytes(fmt, kk) : kk); };
  const uint64_t tk = static_cast<uint64_t>(t) * top_k;
  CUtensorMap t_x32, t_wr, t_xp, t_wgu, t_h, t_wd, t_wsgu, t_hs, t_wsd, t_xsh;
  DG_TRY(make_tmap(&t_x32, d_x, t, d, d, 32));
  DG_TRY(make_tmap(&t_wr, d_wr, n_experts, d, d, 128));
  DG_TRY(make_tmap(&t_xp, at(M_XPERM), tk, mc(d), mp(d), 32, eb));
  DG_TRY(make_tmap(&t_wgu, d_w_gu, static_cast<uint64_t>(n_experts) * 2 * hidden, mc(d), mp(d),
                   128, eb));
  DG_TRY(make_tmap(&t_h, at(f8 ? M_HQ : M_H), tk, mc(hidden), mp(hidden), 32, eb));
  DG_TRY(make_tmap(&t_wd, d_w_d, static_cast<uint64_t>(n_experts) * d, mc(hidden), mp(hidden),
                   128, eb));
  if (f8) DG_TRY(make_tmap(&t_xsh, at(M_XSH), t, mc(d), mp(d), 32, 1));
  if (shared_hidden > 0) {
    DG_TRY(make_tmap(&t_wsgu, d_ws_gu, 2ull * shared_hidden, mc(d), mp(d), 128, eb));
    DG_TRY(make_tmap(&t_hs, at(f8 ? M_HSQ : M_HS), t, mc(shared_hidden), mp(shared_hidden), 32,
                     eb));
    DG_TRY(make_tmap(&t_wsd, d_ws_d, d, mc(shared_hidden), mp(shared_hidden), 128, eb));
  }
  if (fmt == 2)  // pad atoms must read as zero scales
    DG_CUDA(cudaMemsetAsync(at(M_XSF), 0, m.total - m.off[M_XSF], st));  // the last 4 buffers
  // router
  CluParams pr = clu_params(n_experts, t, d / 64, m.split_r, err, nullptr, kRouterChunk);
  pr.router_logits = d_router_logits ? d_router_logits : rlog;
  pr.ids = ids;
  pr.wts = wts;
  pr.top_k = top_k;
  pr.route = RouteArgs{ids, t, top_k, n_experts,
                       route_chunk(fmt, static_cast<long long>(t) * top_k, n_experts), offs,
                       perm, chunks, icnt, nullptr, nullptr};
  if (fmt != 2) {  // the gate/up GEMM gathers the rows itself; the routing permutes the weights
    pr.route.wts = wts;
    pr.route.w_perm = static_cast<float*>(at(M_WPERM));
    pr.pf_first = d_w_gu;
    pr.pf_first_bytes = std::min(kPrefetchExperts, n_experts) * 2ll * hidden * operand_row_bytes(fmt, d);
  }
  pr.ticket = route_ticket;
  DG_TRY(launch_cluster<kCluRouter>(t_wr, t_x32, pr, st, -1));
  ExpertPass e{};
  e.n = t;
  e.d = d;
  e.k = top_k;
  e.E = n_experts;
  e.hid = hidden;
  e.hs = shared_hidden;
  e.fmt = fmt;
  e.perm = perm;
  e.topk_w = wts;
  e.w_perm = static_cast<float*>(at(M_WPERM));
  e.chunks = chunks;
  e.n_chunks = icnt;
  e.xn = static_cast<const __nv_bfloat16*>(d_x);
  e.x_perm = at(M_XPERM);
  e.x_perm_scale = static_cast<float*>(at(M_XPS));
  e.x_sh = at(M_XSH);
  e.x_sh_scale = static_cast<float*>(at(M_XSHS));
  e.h = static_cast<__nv_bfloat16*>(at(M_H));
  e.h_sh = static_cast<__nv_bfloat16*>(at(M_HS));
  e.hq = at(M_HQ);
  e.hq_scale = static_cast<float*>(at(M_HQS));
  e.hsq = at(M_HSQ);
  e.hsq_scale = static_cast<float*>(at(M_HSQS));
  e.x_sf = static_cast<uint8_t*>(at(M_XSF));
  e.x_sh_sf = static_cast<uint8_t*>(at(M_XSHSF));
  e.h_sf = static_cast<uint8_t*>(at(M_HSF));
  e.hs_sf = static_cast<uint8_t*>(at(M_HSSF));
  e.y_slot = static_cast<float*>(at(M_YSLOT));
  e.y_shared = static_cast<float*>(at(M_YSH));
  e.w_gu = d_w_gu;
  e.ws_d = d_ws_d;
  e.w_gu_scale = sc.w_gu;
  e.w_d_scale = sc.w_d;
  e.ws_gu_scale = sc.ws_gu;
  e.ws_d_scale = sc.ws_d;
  e.w_gu_sf = static_cast<const uint8_t*>(sc.w_gu_sf);
  e.w_d_sf = static_cast<const uint8_t*>(sc.w_d_sf);
  e.ws_gu_sf = static_cast<const uint8_t*>(sc.ws_gu_sf);
  e.ws_d_sf = static_cast<const uint8_t*>(sc.ws_d_sf);
  e.tm_wgu = &t_wgu;
  e.tm_xperm = &t_xp;
  e.tm_wsgu = &t_wsgu;
  e.tm_xsh = f8 ? &t_xsh : &t_x32;
  e.tm_wd = &t_wd;
  e.tm_h = &t_h;
  e.tm_wsd = &t_wsd;
  e.tm_hs = &t_hs;
  e.err = err;
  e.done = nullptr;
  e.profile = false;
  DG_TRY(launch_experts(e, sms, st));
  const float* ysh_ptr = shared_hidden > 0 ? e.y_shared : nullptr;
  if (d_residual)
    DG_CUDA(cudaMemcpyAsync(d_y, d_residual, static_cast<size_t>(t) * d * 4,
                            cudaMemcpyDeviceToDevice, st));
  else
    DG_CUDA(cudaMemsetAsync(d_y, 0, static_cast<size_t>(t) * d * 4, st));
  DG_TRY(launch_pdl(moe_combine_norm_kernel<__nv_bfloat16>, dim3(t), dim3(256), 0, st, d_y,
                    e.y_slot, top_k, ysh_ptr, d, nullptr, 0.f, nullptr, nullptr));
  DG_LAUNCHED();
  if (d_ids)
    DG_CUDA(cudaMemcpyAsync(d_ids, ids, static_cast<size_t>(t) * top_k * 4,
                            cudaMemcpyDeviceToDevice, st));
  if (d_weights)
    DG_CUDA(cudaMemcpyAsync(d_weights, wts, static_cast<size_t>(t) * top_k * 4,
                            cudaMemcpyDeviceToDevice, st));
  return DG_OK;
}
}  // namespace

int dg_moe_workspace_bytes(int32_t t, int32_t d, int32_t n_experts, int32_t top_k, int32_t hidden,
                           int32_t shared_hidden, size_t* bytes) {
  if (t < 1 || d < 128 || d % 64 || d > 4096 || n_experts < 4 || n_experts % 4 || n_experts > 128 ||
      top_k < 1 || top_k > 8 ||
      top_k > n_experts || hidden < 64 || hidden % 64 || shared_hidden < 0 || shared_hidden % 64 ||
      !bytes)
    return fail(DG_ERR_INVALID_ARG, "bad MoE shape");
  *bytes = moe_plan(t, d, n_experts, top_k, hidden, shared_hidden).total;
  return DG_OK;
}

int dg_moe_ffn(const void* d_x, const float* d_residual, const void* d_wr, const void* d_w_gu,
               const void* d_w_d, const void* d_ws_gu, const void* d_ws_d, float* d_y,
               int32_t* d_ids, float* d_weights, float* d_router_logits, int32_t t, int32_t d,
               int32_t n_experts, int32_t top_k, int32_t hidden, int32_t shared_hidden,
               void* d_workspace, size_t workspace_bytes, void* stream) {
  return moe_ffn_impl(0, MoeScales{}, d_x, d_residual, d_wr, d_w_gu, d_w_d, d_ws_gu, d_ws_d,
                      d_y, d_ids, d_weights, d_router_logits, t, d, n_experts, top_k, hidden,
                      shared_hidden, d_workspace, workspace_bytes, stream);
}

int dg_moe_ffn_e4m3(const void* d_x, const float* d_residual, const void* d_wr,
                    const void* d_w_gu, const float* d_w_gu_scale, const void* d_w_d,
                    const float* d_w_d_scale, const void* d_ws_gu, const float* d_ws_gu_scale,
                    const void* d_ws_d, const float* d_ws_d_scale, float* d_y, int32_t* d_ids,
                    float* d_weights, float* d_router_logits, int32_t t, int32_t d,
                    int32_t n_experts, int32_t top_k, int32_t hidden, int32_t shared_hidden,
                    void* d_workspace, size_t workspace_bytes, void* stream) {
  return moe_ffn_impl(1, MoeScales{d_w_gu_scale, d_w_d_scale, d_ws_gu_scale, d_ws_d_scale,
                                   nullptr, nullptr, nullptr, nullptr},
                      d_x, d_residual, d_wr, d_w_gu, d_w_d, d_ws_gu, d_ws_d, d_y, d_ids,
                      d_weights, d_router_logits, t, d, n_experts, top_k, hidden, shared_hidden,
                      d_workspace, workspace_bytes, stream);
}

int dg_moe_ffn_nvfp4(const void* d_x, const float* d_residual, const void* d_wr,
                     const void* d_w_gu, const float* d_w_gu_scale, const void* d_w_gu_sf,
                     const void* d_w_d, const float* d_w_d_scale, const void* d_w_d_sf,
                     const void* d_ws_gu, const float* d_ws_gu_scale, const void* d_ws_gu_sf,
                     const void* d_ws_d, const float* d_ws_d_scale, const void* d_ws_d_sf,
                     float* d_y, int32_t* d_ids, float* d_weights, float* d_router_logits,
                     int32_t t, int32_t d, int32_t n_experts, int32_t top_k, int32_t hidden,
                     int32_t shared_hidden, void* d_workspace, size_t workspace_bytes,
                     void* stream) {
  return moe_ffn_impl(2, MoeScales{d_w_gu_scale, d_w_d_scale, d_ws_gu_scale, d_ws_d_scale,
                                   d_w_gu_sf, d_w_d_sf, d_ws_gu_sf, d_ws_d_sf},
                      d_x, d_residual, d_wr, d_w_gu, d_w_d, d_ws_gu, d_ws_d, d_y, d_ids,
                      d_weights, d_router_logits, t, d, n_experts, top_k, hidden, shared_hidden,
                      d_workspace, workspace_bytes, stream);
}

int dg_quantize_nvfp4(const void* d_in, int32_t rows, int32_t cols, int64_t ld_in,
                      uint8_t* d_codes, int64_t ld_codes, uint8_t* d_sf, float* d_row_scales,
                      void* stream) {
  if (!d_in || !d_codes || !d_sf || !d_row_scales)
    return fail(DG_ERR_INVALID_ARG, "null pointer argument");
  if (rows < 0 || cols < 64 || cols % 64 || ld_in < cols || ld_in % 8 || ld_codes < cols / 2 ||
      ld_codes % 16 || ld_codes > (1 << 30))
    return fail(DG_ERR_INVALID_ARG,
                "need cols %% 64 == 0, ld_in >= cols, ld_in %% 8 == 0, ld_codes >= cols / 2, "
                "ld_codes %% 16 == 0");
  if (reinterpret_cast<uintptr_t>(d_in) % 16 || reinterpret_cast<uintptr_t>(d_codes) % 16 ||
      reinterpret_cast<uintptr_t>(d_sf) % 16 || reinterpret_cast<uintptr_t>(d_row_scales) % 4)
    return fail(DG_ERR_INVALID_ARG, "misaligned pointer");
  if (rows == 0) return DG_OK;
  cudaStream_t st = S(stream);
  const size_t sf_bytes = static_cast<size_t>(cdiv(rows, 128)) * 4 * cdiv(cols, 256) * 512;
  DG_CUDA(cudaMemsetAsync(d_sf, 0, sf_bytes, st));  // pad atoms and rows past `rows` read as 0
  QuantFp4Job j{};
  j.seg[0] = QuantFp4Seg{static_cast<const __nv_bfloat16*>(d_in), ld_in, nullptr, 1, nullptr,
                         nullptr, rows, cols, d_codes, ld_codes, d_sf, d_row_scales, nullptr,
                         nullptr, 128};
  j.n_seg = 1;
  DG_TRY(launch_pdl(quant_fp4_rows_kernel, dim3(cdiv(rows, 8)), dim3(256), 0, st, j,
                    static_cast<const int*>(nullptr)));
  DG_LAUNCHED();
  return DG_OK;
}

int dg_quantize_e4m3(const void* d_in, int32_t rows, int32_t cols, int64_t ld_in,
                     uint8_t* d_codes, int64_t ld_codes, float* d_scales, void* stream) {
  if (!d_in || !d_codes || !d_scales) return fail(DG_ERR_INVALID_ARG, "null pointer argument");
  if (rows < 0 || cols < 16 || cols % 16 || ld_in < cols || ld_in % 8 || ld_codes < cols ||
      ld_codes % 16 || ld_codes > (1 << 30))
    return fail(DG_ERR_INVALID_ARG,
                "need cols %% 16 == 0, ld_in >= cols, ld_in %% 8 == 0, ld_codes >= cols, "
                "ld_codes %% 16 == 0");
  if (reinterpret_cast<uintptr_t>(d_in) % 16 || reinterpret_cast<uintptr_t>(d_codes) % 16 ||
      reinterpret_cast<uintptr_t>(d_scales) % 4)
    return fail(DG_ERR_INVALID_ARG, "misaligned pointer");
  if (rows == 0) return DG_OK;
  QuantJob j{};
  j.seg[0] = QuantSeg{static_cast<const __nv_bfloat16*>(d_in), ld_in, nullptr, 1, nullptr,
                      nullptr, rows, cols, d_codes, ld_codes, d_scales};
  j.n_seg = 1;
  DG_TRY(launch_pdl(quant_rows_kernel, dim3(cdiv(rows, 8)), dim3(256), 0, S(stream), j,
                    static_cast<const int*>(nullptr)));
  DG_LAUNCHED();
  return DG_OK;
}

}  // extern "C"

// ---- sampler without caller-provided workspace -------------------------------------------
// Some callers cannot allocate device memory: for example a host framework whose own pool owns
// the whole device budget, or a latency-critical path that may not risk cudaMalloc's implicit
// device synchronisation.  dg_sampler_step_static keeps the sampler's temporaries and its
// step-to-step stop-test state in one fixed file-scope device array instead of a workspace.
namespace {
constexpr int kStaticRows = 256;
constexpr int kStaticVocab = 262144;
constexpr int kStaticChunks = kStaticVocab / 4096;  // fp32 slices are the finer ones
constexpr size_t kStaticPartBytes = static_cast<size_t>(kStaticRows) * kStaticChunks * sizeof(StatPartial);
constexpr size_t kStaticPrevOff = kStaticPartBytes;
constexpr size_t kStaticRowHOff = kStaticPrevOff + 256 * 4;
constexpr size_t kStaticLockedOff = kStaticRowHOff + 256 * 8;
constexpr size_t kStaticTicketOff = kStaticLockedOff + 256 * 4;
constexpr size_t kStaticBytes = kStaticTicketOff + 256;
}  // namespace

// Held by every GPU that loads this library until the process exits (about 266 KB).
static __device__ __align__(256) uint8_t g_sampler_scratch[kStaticBytes];

namespace {
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

std::mutex g_static_mu;
struct StaticAddr {
  CUcontext ctx;  // the context the address belongs to
  void* ptr;      // device address of g_sampler_scratch in that context
};
StaticAddr g_static_addr[256] = {};  // per device ordinal

// The first call on a device (and the first after that device's context was replaced, e.g. by
// cudaDeviceReset, which reloads this module at a new address) looks up the array's device
// address with that device current; later calls reuse it.
int static_scratch(void** out) {
  int dev = 0;
  DG_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 256) return fail(DG_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  CtxGetCurrentFn cur = ctx_current_fn();
  CUcontext ctx = nullptr;
  if (!cur || cur(&ctx) != CUDA_SUCCESS)
    return fail(DG_ERR_CUDA, "cannot query the current CUDA context");
  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticAddr& a = g_static_addr[dev];
  if (!ctx || !a.ptr || a.ctx != ctx) {
    void* p = nullptr;
    // also makes the device's primary context current when no context was yet
    const cudaError_t e = cudaGetSymbolAddress(&p, g_sampler_scratch);
    if (e != cudaSuccess || !p)
      return fail(DG_ERR_CUDA, "cudaGetSymbolAddress(sampler scratch) failed: %s",
                  cudaGetErrorString(e));
    if (!ctx && (cur(&ctx) != CUDA_SUCCESS || !ctx))
      return fail(DG_ERR_CUDA, "no current CUDA context after the symbol lookup");
    a.ctx = ctx;
    a.ptr = p;
  }
  *out = a.ptr;
  return DG_OK;
}
}  // namespace

extern "C" int dg_sampler_step_static(const void* d_logits, int32_t dtype, int32_t rows,
                                      int32_t vocab, uint64_t seed, uint32_t block, uint32_t step,
                                      double tau, double h_bound, int32_t max_steps,
                                      int32_t fixed_steps, int32_t* d_canvas, int32_t* d_argmax,
                                      float* d_entropy, float* d_conf, int32_t* d_state,
                                      void* stream) {
  if (rows < 1 || rows > kStaticRows || vocab < 2 || vocab > kStaticVocab || vocab % 8)
    return fail(DG_ERR_CAPACITY,
                "dg_sampler_step_static handles at most %d rows and %d vocabulary entries "
                "(vocab a multiple of 8); got rows %d, vocab %d",
                kStaticRows, kStaticVocab, rows, vocab);
  if (!d_logits || !d_canvas || !d_argmax || !d_entropy || !d_conf || !d_state)
    return fail(DG_ERR_INVALID_ARG, "null pointer argument");
  if (reinterpret_cast<uintptr_t>(d_logits) % 16)
    return fail(DG_ERR_INVALID_ARG, "logits must be 16-byte aligned");
  if (step < 1 || max_steps < 1 || fixed_steps < 0)
    return fail(DG_ERR_INVALID_ARG, "bad step / max_steps / fixed_steps");
  if (dtype != DG_DTYPE_BF16 && dtype != DG_DTYPE_FP32)
    return fail(DG_ERR_INVALID_ARG, "dtype must be bf16 or fp32");
  void* base = nullptr;
  DG_TRY(static_scratch(&base));
  uint8_t* b = static_cast<uint8_t*>(base);
  StatPartial* part = reinterpret_cast<StatPartial*>(b);
  int32_t* prev = reinterpret_cast<int32_t*>(b + kStaticPrevOff);
  double* row_h = reinterpret_cast<double*>(b + kStaticRowHOff);
  int32_t* locked = reinterpret_cast<int32_t*>(b + kStaticLockedOff);
  int32_t* ticket = reinterpret_cast<int32_t*>(b + kStaticTicketOff);
  cudaStream_t st = S(stream);
  // the completion ticket must start at zero; the previous argmax is only read from step 2 on
  DG_CUDA(cudaMemsetAsync(ticket, 0, sizeof(int32_t), st));
  const int chunk = dtype == DG_DTYPE_BF16 ? 8192 : 4096;
  const int nchunk = cdiv(vocab, chunk);
  const int* done = d_state + kStDone;
  if (dtype == DG_DTYPE_BF16)
    DG_TRY(launch_pdl(logits_stats_kernel<__nv_bfloat16, 32>, dim3(nchunk, rows), dim3(256), 0, st, 
        static_cast<const __nv_bfloat16*>(d_logits), vocab, chunk, part, done, 1.0f));
  else
    DG_TRY(launch_pdl(logits_stats_kernel<float, 16>, dim3(nchunk, rows), dim3(256), 0, st,
        static_cast<const float*>(d_logits), vocab, chunk, part, done, 1.0f));
  DG_LAUNCHED();
  SamplerArgs a{};
  a.partials = part;
  a.nsplit = nchunk;
  a.rows = rows;
  a.vocab = vocab;
  a.seed = seed;
  a.block = block;
  a.step = step;
  a.tau = tau;
  a.h_bound = h_bound;
  a.max_steps = max_steps;
  a.fixed_steps = fixed_steps;
  a.canvas = d_canvas;
  a.argmax = d_argmax;
  a.prev_argmax = prev;
  a.entropy = d_entropy;
  a.conf = d_conf;
  a.row_h = row_h;
  a.locked = locked;
  a.state = d_state;
  a.ticket = ticket;
  a.n_seq = 1;
  DG_TRY(launch_pdl(sampler_merge_kernel, dim3(rows), dim3(256), 0, st, a));
  DG_LAUNCHED();
  return DG_OK;
}
