// api.cu - the C ABI of libdg.so: argument checks, TMA descriptor set-up,
// launch planning (split-K, split-KV), the model forward, prefill, the
// denoising loop and the block commit.  Built as one translation unit so that
// the per-device error word is shared by every kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <utility>
#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/dg.h"
#include "attn.cuh"
#include "dg_common.cuh"
#include "gemm.cuh"
#include "kvcommit.cuh"
#include "norm.cuh"
#include "quant.cuh"
#include "unembed.cuh"
#include "sampler.cuh"
#include "selftest.cuh"

namespace {

constexpr int kVersion = 1;
constexpr int kNumSMs = 148;

thread_local char g_last_error[512] = "";
std::atomic<unsigned long long> g_launches{0};
inline void count_launch(unsigned long long n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// Programmatic dependent launch is on unless DG_PDL=0 is set in the environment.
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("DG_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

// The denoising loop replays each step as a CUDA graph unless DG_GRAPHS=0.
bool graphs_enabled() {
  static const bool on = [] {
    const char* e = getenv("DG_GRAPHS");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Launch with programmatic stream serialization (the kernel must call
// griddep_wait before touching its predecessors' data) and an optional
// cluster shape along z.
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t s, dim3 cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster.x * cluster.y * cluster.z > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster.x;
    attr[n].val.clusterDim.y = cluster.y;
    attr[n].val.clusterDim.z = cluster.z;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t s, int cluster_z, Args&&... args) {
  return launch_cluster(kernel, grid, block, smem, s, dim3(1, 1, cluster_z),
                        std::forward<Args>(args)...);
}

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

#define DG_CUDA(expr)                                                                     \
  do {                                                                                    \
    cudaError_t e_ = (expr);                                                              \
    if (e_ != cudaSuccess)                                                                \
      return fail(DG_ERR_CUDA, "%s failed: %s (%s:%d)", #expr, cudaGetErrorString(e_),    \
                  __FILE__, __LINE__);                                                    \
  } while (0)

#define DG_TRY(expr)              \
  do {                            \
    int s_ = (expr);              \
    if (s_ != DG_OK) return s_;   \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched through the runtime)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
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

// 2-D bf16 map over rows of `inner` elements, `row_stride` bytes apart; box
// {64, box_rows} with 128-byte swizzle (one box row = one 128-byte line).
int make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
              uint64_t row_stride_bytes, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (!aligned16(base) || (row_stride_bytes & 15u))
    return fail(DG_ERR_ALIGNMENT, "tensor map base %p / stride %llu not 16-byte aligned", base,
                (unsigned long long)row_stride_bytes);
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) inner=%llu rows=%llu", (int)r,
                (unsigned long long)inner, (unsigned long long)rows);
  return DG_OK;
}

// The same for 8-bit elements: box {128, box_rows} (one 128-byte line per row).
int make_tmap_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                 uint64_t row_stride_bytes, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (!aligned16(base) || (row_stride_bytes & 15u))
    return fail(DG_ERR_ALIGNMENT, "tensor map base %p / stride %llu not 16-byte aligned", base,
                (unsigned long long)row_stride_bytes);
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (u8) failed (%d) inner=%llu rows=%llu",
                (int)r, (unsigned long long)inner, (unsigned long long)rows);
  return DG_OK;
}

// Dequantisation scales of e4m3 unembedding operands (null: bf16 operands).
struct Fp8Scales {
  const float* tok;  // [M] per-token scale of the activations
  const float* w;    // the weight tensor's scale (device scalar)
};

// ---------------------------------------------------------------------------
// GEMM
// ---------------------------------------------------------------------------
struct GemmPlan {
  int splits, kb_per_split, bn;
  int ring_kb = 192;  // 192: one CTA per SM; 96: two CTAs per SM
};

// Choose the token tile (128 or 256) and the K split (cluster of 1, 2 or 4)
// that puts the most CTAs on the SMs in a single wave, preferring fewer splits
// and then wider tiles; each split keeps >= 4 k-blocks.  Shapes with more
// tiles than SMs use 256-token tiles without splitting.
GemmPlan plan_gemm(int M, int N, int K, int kb_elems = dg::gemm::BK) {
  const int kb = K / kb_elems;
  const int ft = N / dg::gemm::BM;
  GemmPlan best{1, kb, 256};
  int best_ctas = -1;
  for (int s : {1, 2, 4}) {
    for (int bn : {256, 128}) {
      if (kb % s || kb / s < 4) continue;
      const int ctas = ft * cdiv(M, bn) * s;
      if (ctas > kNumSMs) continue;
      if (ctas > best_ctas) {
        best = GemmPlan{s, kb / s, bn};
        best_ctas = ctas;
      }
    }
  }
  return best;
}

// "Kernel attributes are set" flags.  A kernel's attributes belong to one
// device's context, so the flag is kept per device (a device beyond the
// table re-sets them on every call).
struct PerDeviceFlag {
  bool done[64] = {};
  bool spare = false;
  bool& operator()() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return spare = false;
    return done[dev];
  }
};

PerDeviceFlag gemm_attr_done;

// Epilogue operands of one GEMM launch (see gemm.cuh).
struct GemmEpi {
  int epi = dg::gemm::EPI_F32;
  float* out_f32 = nullptr;
  __nv_bfloat16* out_bf16 = nullptr;
  float* x = nullptr;
  const float* ssq_in = nullptr;
  int n_ssq_in = 0;
  float inv_k = 0.f;
  float eps = 0.f;
  float* ssq_out = nullptr;
  unsigned long long* trace = nullptr;
};

// The GEMM instantiations: (split count, token tile, ring KB).
#define DG_GEMM_VARIANTS(X)                                                              \
  X(1, 256, 192) X(2, 256, 192) X(4, 256, 192) X(1, 128, 192) X(2, 128, 192)           \
  X(4, 128, 192) X(1, 128, 96) X(2, 128, 96) X(4, 128, 96) X(8, 128, 96) X(1, 64, 96)   \
  X(2, 64, 96) X(4, 64, 96) X(8, 64, 96)

template <int S, int BN, bool F8, int R>
cudaError_t launch_gemm_t(dim3 grid, cudaStream_t s, const CUtensorMap& tw, const CUtensorMap& tx,
                          const dg::gemm::Params& p) {
  return launch_ex(dg::gemm::gemm_kernel<S, BN, F8, R>, grid, dim3(dg::gemm::THREADS),
                   dg::gemm::smem_bytes(R), s, S, tw, tx, p);
}

template <int S, int BN, bool F8, int R>
cudaError_t gemm_set_attr() {
  return cudaFuncSetAttribute(dg::gemm::gemm_kernel<S, BN, F8, R>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              dg::gemm::smem_bytes(R));
}

template <bool F8>
cudaError_t gemm_set_attrs() {
  cudaError_t e;
#define DG_X(S_, BN_, R_) \
  if ((e = gemm_set_attr<S_, BN_, F8, R_>()) != cudaSuccess) return e;
  DG_GEMM_VARIANTS(DG_X)
#undef DG_X
  return cudaSuccess;
}

template <bool F8>
cudaError_t launch_gemm_plan(const GemmPlan& pl, dim3 grid, cudaStream_t s, const CUtensorMap& tw,
                             const CUtensorMap& tx, const dg::gemm::Params& p) {
#define DG_X(S_, BN_, R_)                                    \
  if (pl.splits == S_ && pl.bn == BN_ && pl.ring_kb == R_) \
    return launch_gemm_t<S_, BN_, F8, R_>(grid, s, tw, tx, p);
  DG_GEMM_VARIANTS(DG_X)
#undef DG_X
  return cudaErrorInvalidValue;
}

// x [M, K] and w [N, K]: bf16, or e4m3 codes with their scales when f8 is set.
int launch_gemm(const void* x, const void* w, int M, int N, int K, const GemmPlan& pl,
                const GemmEpi& e, cudaStream_t s, const Fp8Scales* f8 = nullptr) {
  if (!gemm_attr_done()) {
    DG_CUDA(gemm_set_attrs<false>());
    DG_CUDA(gemm_set_attrs<true>());
    gemm_attr_done() = true;
  }
  CUtensorMap tw, tx;
  if (f8) {
    DG_TRY(make_tmap_u8(&tw, w, K, N, (uint64_t)K, dg::gemm::BM));
    DG_TRY(make_tmap_u8(&tx, x, K, M, (uint64_t)K, pl.bn));
  } else {
    DG_TRY(make_tmap(&tw, w, K, N, (uint64_t)K * 2, dg::gemm::BM));
    DG_TRY(make_tmap(&tx, x, K, M, (uint64_t)K * 2, pl.bn));
  }
  dg::gemm::Params p;
  p.M = M; p.N = N; p.K = K;
  p.kb_per_split = pl.kb_per_split;
  p.splits = pl.splits;
  p.epi = e.epi;
  p.out_f32 = e.out_f32;
  p.out_bf16 = e.out_bf16;
  p.x = e.x;
  p.ssq_in = e.ssq_in;
  p.n_ssq_in = e.n_ssq_in;
  p.inv_k = e.inv_k;
  p.eps = e.eps;
  p.ssq_out = e.ssq_out;
  p.trace = e.trace;
  p.tok_scale = f8 ? f8->tok : nullptr;
  p.w_scale = f8 ? f8->w : nullptr;
  const dim3 grid(cdiv(M, pl.bn), N / dg::gemm::BM, pl.splits);
  const cudaError_t err = f8 ? launch_gemm_plan<true>(pl, grid, s, tw, tx, p)
                             : launch_gemm_plan<false>(pl, grid, s, tw, tx, p);
  if (err != cudaSuccess)
    return fail(DG_ERR_CUDA, "gemm launch (S=%d, BN=%d, ring %d KB) failed: %s", pl.splits,
                pl.bn, pl.ring_kb, cudaGetErrorString(err));
  count_launch();
  return DG_OK;
}

// Projections with many tokens run on the persistent CTA-pair pipeline
// (unembed.cuh, 256 x 256 tiles, double-buffered accumulators); fewer tokens
// take the split-K GEMM.
bool proj_use_pair(int M, int N, int K, bool f8) {
  const int kbe = f8 ? 128 : dg::gemm::BK;
  if (N % dg::unembed::TILE || K % kbe || K / kbe < 4) return false;
  // a full wave of pairs, or 48..73 tiles where the many-token shapes
  // measured faster than the split-K plans (M >= 1536)
  const int tiles = (N / dg::unembed::TILE) * cdiv(M, dg::unembed::TILE);
  return tiles >= kNumSMs / 2 || (tiles >= 48 && M >= 1536);
}

PerDeviceFlag proj_attr_done;

template <int KPS, bool F8>
cudaError_t proj_set_attrs() {
  namespace ue = dg::unembed;
  namespace gm = dg::gemm;
  cudaError_t e;
  const int smem = ue::SMEM_BYTES;
  const auto a = cudaFuncAttributeMaxDynamicSharedMemorySize;
  if ((e = cudaFuncSetAttribute(ue::proj_pair_kernel<KPS, F8, gm::EPI_F32>, a, smem))) return e;
  if ((e = cudaFuncSetAttribute(ue::proj_pair_kernel<KPS, F8, gm::EPI_BF16>, a, smem))) return e;
  if ((e = cudaFuncSetAttribute(ue::proj_pair_kernel<KPS, F8, gm::EPI_GELU>, a, smem))) return e;
  return cudaFuncSetAttribute(ue::proj_pair_kernel<KPS, F8, gm::EPI_RESID>, a, smem);
}

template <int KPS, bool F8>
decltype(&dg::unembed::proj_pair_kernel<1, false, 0>) proj_kernel(int epi) {
  namespace ue = dg::unembed;
  namespace gm = dg::gemm;
  switch (epi) {
    case gm::EPI_F32: return ue::proj_pair_kernel<KPS, F8, gm::EPI_F32>;
    case gm::EPI_GELU: return ue::proj_pair_kernel<KPS, F8, gm::EPI_GELU>;
    case gm::EPI_RESID: return ue::proj_pair_kernel<KPS, F8, gm::EPI_RESID>;
    default: return ue::proj_pair_kernel<KPS, F8, gm::EPI_BF16>;
  }
}

int launch_proj_pair(const void* x, const void* w, int M, int N, int K, const GemmEpi& e,
                     cudaStream_t s, const Fp8Scales* f8) {
  namespace ue = dg::unembed;
  if (!proj_attr_done()) {
    DG_CUDA((proj_set_attrs<1, false>()));
    DG_CUDA((proj_set_attrs<1, true>()));
    proj_attr_done() = true;
  }
  CUtensorMap tw, tx;
  if (f8) {
    DG_TRY(make_tmap_u8(&tw, w, K, N, (uint64_t)K, ue::HALF));
    DG_TRY(make_tmap_u8(&tx, x, K, M, (uint64_t)K, ue::HALF));
  } else {
    DG_TRY(make_tmap(&tw, w, K, N, (uint64_t)K * 2, ue::HALF));
    DG_TRY(make_tmap(&tx, x, K, M, (uint64_t)K * 2, ue::HALF));
  }
  ue::ProjParams p;
  p.M = M; p.N = N; p.K = K;
  p.n_ttiles = cdiv(M, ue::TILE);
  p.n_tiles = (N / ue::TILE) * p.n_ttiles;
  p.n_pairs = std::min(kNumSMs / 2, p.n_tiles);
  p.epi = e.epi;
  p.out_f32 = e.out_f32;
  p.out_bf16 = e.out_bf16;
  p.x = e.x;
  p.ssq_in = e.ssq_in; p.n_ssq_in = e.n_ssq_in; p.inv_k = e.inv_k; p.eps = e.eps;
  p.ssq_out = e.ssq_out;
  p.tok_scale = f8 ? f8->tok : nullptr;
  p.w_scale = f8 ? f8->w : nullptr;
  // one k-block per stage (two, 256 bytes per row request, measured the same
  // here, unlike the unembedding's weight stream)
  auto* kern = f8 ? proj_kernel<1, true>(e.epi) : proj_kernel<1, false>(e.epi);
  DG_CUDA(launch_cluster(kern, dim3(2 * p.n_pairs), dim3(ue::threads_for(ue::PROJ_EPI_WARPS)),
                         ue::SMEM_BYTES, s, dim3(2, 1, 1), tw, tx, p));
  count_launch();
  return DG_OK;
}

// y = epilogue(x w^T) with the plan chosen for this shape (e4m3 operands with
// their scales when f8 is set: 128-element k-blocks).  An EPI_RESID with
// ssq_out writes its sums of squares per 128 features on the split-K GEMM
// and per 32 on the pair pipeline.
int linear(const void* x, const void* w, int M, int N, int K, const GemmEpi& e,
           cudaStream_t s, const Fp8Scales* f8 = nullptr) {
  if (proj_use_pair(M, N, K, f8 != nullptr))
    return launch_proj_pair(x, w, M, N, K, e, s, f8);
  return launch_gemm(x, w, M, N, K, plan_gemm(M, N, K, f8 ? 128 : dg::gemm::BK), e, s, f8);
}

// Whether both residual projections of a forward pass over M tokens (the
// output projection, K = Hq hd, and the MLP down projection, K = F) run on
// the pair pipeline.  Each projection picks its plan from its own shape.
bool resid_on_pair(const dg_model_cfg& c, int M, bool f8) {
  return proj_use_pair(M, c.d, c.n_q_heads * c.head_dim, f8) &&
         proj_use_pair(M, c.d, c.ffn, f8);
}

// logits = rs * (h w_u^T).  Vocabularies that are a multiple of 256 run on
// the persistent CTA-pair kernel (unembed.cuh); others on the single-CTA GEMM.
PerDeviceFlag unembed_attr_done;

int launch_unembed(const void* h, const void* w_u, float* logits, int M, int d, int V,
                   const float* ssq_in, int n_ssq_in, float inv_k, float eps, cudaStream_t s,
                   const Fp8Scales* f8 = nullptr) {
  namespace ue = dg::unembed;
  if (f8 == nullptr && V % ue::TILE != 0) {
    GemmEpi e;
    e.epi = dg::gemm::EPI_F32;
    e.out_f32 = logits;
    e.ssq_in = ssq_in; e.n_ssq_in = n_ssq_in; e.inv_k = inv_k; e.eps = eps;
    return launch_gemm(h, w_u, M, V, d, GemmPlan{1, d / dg::gemm::BK, 256}, e, s);
  }
  if (!unembed_attr_done()) {
    DG_CUDA(cudaFuncSetAttribute(ue::unembed_pair_kernel<1, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, ue::SMEM_BYTES));
    DG_CUDA(cudaFuncSetAttribute(ue::unembed_pair_kernel<1, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, ue::SMEM_BYTES));
    unembed_attr_done() = true;
  }
  CUtensorMap tw, tx;
  if (f8) {
    DG_TRY(make_tmap_u8(&tw, w_u, d, V, (uint64_t)d, ue::HALF));
    DG_TRY(make_tmap_u8(&tx, h, d, M, (uint64_t)d, ue::HALF));
  } else {
    DG_TRY(make_tmap(&tw, w_u, d, V, (uint64_t)d * 2, ue::HALF));
    DG_TRY(make_tmap(&tx, h, d, M, (uint64_t)d * 2, ue::HALF));
  }
  ue::Params p;
  p.M = M; p.N = V; p.K = d;
  p.n_ttiles = cdiv(M, ue::TILE);
  p.n_tiles = (V / ue::TILE) * p.n_ttiles;
  p.n_pairs = std::min(kNumSMs / 2, p.n_tiles);
  p.logits = logits;
  p.ssq_in = ssq_in; p.n_ssq_in = n_ssq_in; p.inv_k = inv_k; p.eps = eps;
  p.tok_scale = f8 ? f8->tok : nullptr;
  p.w_scale = f8 ? f8->w : nullptr;
  // one k-block per stage: with the logits written this launch is bound by
  // HBM, and deeper single-block stages measured marginally faster
  DG_CUDA(launch_cluster(f8 ? ue::unembed_pair_kernel<1, true> : ue::unembed_pair_kernel<1, false>,
                         dim3(2 * p.n_pairs),
                         dim3(ue::threads_for(ue::STORE_EPI_WARPS)),
                         ue::SMEM_BYTES, s, dim3(2, 1, 1), tw, tx, p));
  count_launch();
  return DG_OK;
}

// ---------------------------------------------------------------------------
// Attention
// ---------------------------------------------------------------------------
// CTAs before splitting the key range: pairs of 128-row query tiles per kv head.
int attn_pairs(int Hq, int Hkv, int Lq) {
  return cdiv((Hq / Hkv) * cdiv(Lq, dg::attn::BQ), 2);
}

// The split count depends on the shape only (it sets the summation order,
// so a shape always gives the same bits).
int attn_splits(int B, int Hq, int Hkv, int Lq, int max_prefix) {
  const int units = B * Hkv * attn_pairs(Hq, Hkv, Lq);
  const int tmax = cdiv(max_prefix, dg::attn::BKV) + cdiv(Lq, dg::attn::BKV);
  int s = std::max(1, kNumSMs / std::max(1, units));
  s = std::min(s, std::max(1, tmax / 2));
  return std::min(s, dg::attn::MAX_SPLITS);
}

size_t attn_ws_bytes(int B, int Hq, int Hkv, int Lq, int hd, int max_prefix) {
  const int S = attn_splits(B, Hq, Hkv, Lq, max_prefix);
  if (S == 1) return 0;
  const size_t rows = (size_t)S * B * Hq * Lq;
  return align_up(rows * hd * 2, 256) + align_up(rows * sizeof(float), 256);
}

PerDeviceFlag attn_attr_done[2];

int launch_attn(const void* q, int ldq, const void* k_new, const void* v_new, int ldkv,
                const void* k_cache, const void* v_cache, const int32_t* cache_len,
                int max_prefix, int lmax, void* out, int ldo, float* lse, int B, int Hq, int Hkv,
                int Lq, int hd, float scale, int mask, void* ws, cudaStream_t s) {
  const int S = attn_splits(B, Hq, Hkv, Lq, max_prefix);
  CUtensorMap tq, tkn, tvn, tkc, tvc;
  DG_TRY(make_tmap(&tq, q, (uint64_t)Hq * hd, (uint64_t)B * Lq, (uint64_t)ldq * 2, 128));
  DG_TRY(make_tmap(&tkn, k_new, (uint64_t)Hkv * hd, (uint64_t)B * Lq, (uint64_t)ldkv * 2, 128));
  DG_TRY(make_tmap(&tvn, v_new, (uint64_t)Hkv * hd, (uint64_t)B * Lq, (uint64_t)ldkv * 2, 128));
  DG_TRY(make_tmap(&tkc, k_cache, hd, (uint64_t)B * Hkv * lmax, (uint64_t)hd * 2, 128));
  DG_TRY(make_tmap(&tvc, v_cache, hd, (uint64_t)B * Hkv * lmax, (uint64_t)hd * 2, 128));
  dg::attn::Params p;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.lmax = lmax; p.group = Hq / Hkv;
  p.n_rt = cdiv(Lq, dg::attn::BQ);
  p.n_pairs = attn_pairs(Hq, Hkv, Lq);
  p.n_splits = S;
  p.causal = mask == DG_MASK_CAUSAL ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.cache_len = cache_len;
  p.out = (__nv_bfloat16*)out;
  p.ldo = ldo;
  p.lse = lse;
  p.part_o = nullptr;
  p.part_lse = nullptr;
  p.q_scale = p.k_scale = p.v_scale = nullptr;
  if (S > 1) {
    const size_t rows = (size_t)S * B * Hq * Lq;
    p.part_o = (__nv_bfloat16*)ws;
    p.part_lse = (float*)((char*)ws + align_up(rows * hd * 2, 256));
  }
  dim3 grid(B * Hkv * p.n_pairs, S);
  if (hd == 128) {
    if (!attn_attr_done[1]()) {
      DG_CUDA(cudaFuncSetAttribute(dg::attn::attn_kernel<128>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   dg::attn::Cfg<128>::SMEM_BYTES));
      attn_attr_done[1]() = true;
    }
    DG_CUDA(launch_ex(dg::attn::attn_kernel<128>, grid, dim3(dg::attn::THREADS),
                      dg::attn::Cfg<128>::SMEM_BYTES, s, 1, tq, tkn, tvn, tkc, tvc, p));
    count_launch();
  } else {
    if (!attn_attr_done[0]()) {
      DG_CUDA(cudaFuncSetAttribute(dg::attn::attn_kernel<64>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   dg::attn::Cfg<64>::SMEM_BYTES));
      attn_attr_done[0]() = true;
    }
    DG_CUDA(launch_ex(dg::attn::attn_kernel<64>, grid, dim3(dg::attn::THREADS),
                      dg::attn::Cfg<64>::SMEM_BYTES, s, 1, tq, tkn, tvn, tkc, tvc, p));
    count_launch();
  }
  DG_CUDA(cudaGetLastError());
  if (S > 1) {
    const int rows = B * Hq * Lq;
    const int threads = dg::attn::COMBINE_THREADS;
    const int blocks = cdiv(rows * 32, threads);  // a warp per row
    if (hd == 128)
      DG_CUDA(launch_ex(dg::attn::attn_combine_kernel<128>, dim3(blocks), dim3(threads), 0, s, 1,
                        (const __nv_bfloat16*)p.part_o, (const float*)p.part_lse, S, B, Hq, Lq,
                        (__nv_bfloat16*)out, ldo, lse));
    else
      DG_CUDA(launch_ex(dg::attn::attn_combine_kernel<64>, dim3(blocks), dim3(threads), 0, s, 1,
                        (const __nv_bfloat16*)p.part_o, (const float*)p.part_lse, S, B, Hq, Lq,
                        (__nv_bfloat16*)out, ldo, lse));
    count_launch();
    DG_CUDA(cudaGetLastError());
  }
  return DG_OK;
}

PerDeviceFlag attn_f8_attr_done;

// The e4m3 variant (hd = 128): the same plan, split count and merge; 8-bit
// tensor maps (one 128-byte swizzle row per box row) over Q, K and V^T.
int launch_attn_e4m3(const uint8_t* q, int ldq, const float* q_scale, const uint8_t* k_new,
                     int ldkv, const uint8_t* vt_new, int ldvt, const uint8_t* k_cache,
                     const uint8_t* vt_cache, const float* k_scale, const float* v_scale,
                     const int32_t* cache_len, int max_prefix, int lmax, void* out, int ldo,
                     float* lse, int B, int Hq, int Hkv, int Lq, float scale, int mask, void* ws,
                     cudaStream_t s) {
  constexpr int hd = 128;
  const int S = attn_splits(B, Hq, Hkv, Lq, max_prefix);
  CUtensorMap tq, tkn, tvn, tkc, tvc;
  DG_TRY(make_tmap_u8(&tq, q, (uint64_t)Hq * hd, (uint64_t)B * Lq, (uint64_t)ldq, 128));
  DG_TRY(make_tmap_u8(&tkn, k_new, (uint64_t)Hkv * hd, (uint64_t)B * Lq, (uint64_t)ldkv, 128));
  DG_TRY(make_tmap_u8(&tvn, vt_new, (uint64_t)Lq, (uint64_t)B * Hkv * hd, (uint64_t)ldvt, 128));
  DG_TRY(make_tmap_u8(&tkc, k_cache, hd, (uint64_t)B * Hkv * lmax, (uint64_t)hd, 128));
  DG_TRY(make_tmap_u8(&tvc, vt_cache, (uint64_t)lmax, (uint64_t)B * Hkv * hd, (uint64_t)lmax,
                      128));
  dg::attn::Params p;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.lmax = lmax; p.group = Hq / Hkv;
  p.n_rt = cdiv(Lq, dg::attn::BQ);
  p.n_pairs = attn_pairs(Hq, Hkv, Lq);
  p.n_splits = S;
  p.causal = mask == DG_MASK_CAUSAL ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.cache_len = cache_len;
  p.out = (__nv_bfloat16*)out;
  p.ldo = ldo;
  p.lse = lse;
  p.part_o = nullptr;
  p.part_lse = nullptr;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  if (S > 1) {
    const size_t rows = (size_t)S * B * Hq * Lq;
    p.part_o = (__nv_bfloat16*)ws;
    p.part_lse = (float*)((char*)ws + align_up(rows * hd * 2, 256));
  }
  using CF = dg::attn::Cfg<128, true>;
  if (!attn_f8_attr_done()) {
    DG_CUDA(cudaFuncSetAttribute(dg::attn::attn_kernel<128, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, CF::SMEM_BYTES));
    attn_f8_attr_done() = true;
  }
  DG_CUDA(launch_ex(dg::attn::attn_kernel<128, true>, dim3(B * Hkv * p.n_pairs, S),
                    dim3(dg::attn::THREADS), CF::SMEM_BYTES, s, 1, tq, tkn, tvn, tkc, tvc, p));
  count_launch();
  DG_CUDA(cudaGetLastError());
  if (S > 1) {
    const int rows = B * Hq * Lq;
    const int threads = dg::attn::COMBINE_THREADS;
    DG_CUDA(launch_ex(dg::attn::attn_combine_kernel<128>, dim3(cdiv(rows * 32, threads)),
                      dim3(threads), 0, s, 1, (const __nv_bfloat16*)p.part_o,
                      (const float*)p.part_lse, S, B, Hq, Lq, (__nv_bfloat16*)out, ldo, lse));
    count_launch();
    DG_CUDA(cudaGetLastError());
  }
  return DG_OK;
}

// ---------------------------------------------------------------------------
// Sampler
// ---------------------------------------------------------------------------
// Row pass chunks: >= 131072 elements (>= 512 per thread: the CTA's closing
// reduction and its first batches, raced before a best score is known, are
// then a small share of its work), at most 64 per row, in multiples of 4
// elements.  When the CTAs would be few (fewer than 16 per SM), up to twice as
// many chunks are taken if that spreads them more evenly over the SMs.  The
// plan depends on the shape only.
int sample_chunking(int rows, int V, int* chunk) {
  const int n0 = std::max(1, std::min(64, V / 131072));
  int nchunk = n0;
  if ((long)rows * n0 < 16L * kNumSMs) {
    double best = 0.0;
    for (int n = n0; n <= std::min(64, 2 * n0); ++n) {
      const long ctas = (long)rows * n;
      const double fill = (double)ctas / (double)(cdiv(ctas, (long)kNumSMs) * kNumSMs);
      if (fill > best + 1e-9) {
        best = fill;
        nchunk = n;
      }
    }
  }
  int c = cdiv(V, nchunk);
  c = (c + 3) / 4 * 4;
  nchunk = cdiv(V, c);
  *chunk = c;
  return nchunk;
}

size_t sample_ws_bytes(int B, int C, int V) {
  int chunk;
  const int nchunk = sample_chunking(B * C, V, &chunk);
  return align_up((size_t)B * C * nchunk * sizeof(dg::RowPartial), 256);
}

bool sampler_cfg_ok(const dg_sampler_cfg& c) {
  return c.max_steps >= 1 && c.commit_k >= 0 && c.t_start > 0.f && c.t_end > 0.f &&
         (c.unselected_policy == DG_UNSELECTED_KEEP ||
          c.unselected_policy == DG_UNSELECTED_RENOISE) &&
         (c.selection == DG_SELECT_TOP_K || c.selection == DG_SELECT_ENTROPY) &&
         c.entropy_bound >= 0.f;
}

dg::SampleParams make_sample_params(const dg_sampler_cfg& cfg, uint32_t seed, int block,
                                    const int32_t* step_ptr, int step, int B, int C, int V) {
  dg::SampleParams p;
  p.B = B; p.C = C; p.V = V;
  p.nchunk = sample_chunking(B * C, V, &p.chunk);
  p.seed = seed;
  p.block = block;
  p.step_ptr = step_ptr;
  p.step_val = step;
  p.max_steps = cfg.max_steps;
  p.t_start = cfg.t_start;
  p.t_end = cfg.t_end;
  p.commit_k = cfg.commit_k;
  p.log_tau = cfg.renoise_conf > 0.f ? (float)std::log((double)cfg.renoise_conf) : -INFINITY;
  p.stop_entropy = cfg.stop_entropy;
  p.policy = cfg.unselected_policy;
  p.selection = cfg.selection;
  p.entropy_bound = cfg.entropy_bound;
  p.near_ties = nullptr;
  return p;
}

PerDeviceFlag rowpass_attr_done;

int launch_sample(const float* logits, int32_t* tok, uint8_t* committed, int32_t* prev_argmax,
                  int32_t* seq_status, const dg::SampleParams& p, const dg_step_out* out,
                  void* ws, cudaStream_t s) {
  dg::RowPartial* part = (dg::RowPartial*)ws;
  if (!rowpass_attr_done()) {
    DG_CUDA(cudaFuncSetAttribute(dg::sample_rowpass_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, dg::RP_SMEM));
    rowpass_attr_done() = true;
  }
  DG_CUDA(launch_ex(dg::sample_rowpass_kernel, dim3(p.B * p.C * p.nchunk), dim3(dg::RP_THREADS),
                    dg::RP_SMEM, s, 1, logits, (const int32_t*)seq_status, p, part));
  count_launch();
  const int threads = (p.C + 31) / 32 * 32;
  dg::SampleParams pc = p;
  pc.near_ties = out ? out->near_ties : nullptr;
  DG_CUDA(launch_ex(dg::sample_commit_kernel, dim3(p.B), dim3(threads), 0, s, 1, logits,
                    (const dg::RowPartial*)part, (const dg::RowStats*)nullptr, pc, tok, committed,
                    prev_argmax, seq_status,
                    out ? out->x_hat : (int32_t*)nullptr, out ? out->argmax : (int32_t*)nullptr,
                    out ? out->logconf : (float*)nullptr, out ? out->entropy : (float*)nullptr,
                    out ? out->flags : (uint8_t*)nullptr));
  count_launch();
  return DG_OK;
}

// ---------------------------------------------------------------------------
// Unembedding fused with the sampler step (vocabularies that are a multiple
// of 256): unembed_sample_kernel -> sample_merge_kernel -> sample_commit_kernel
// ---------------------------------------------------------------------------
struct FusedPlan {
  int n_ttiles, segs, n_pairs, nparts;
};

// As many vocabulary segments per token tile as keep one wave of CTA pairs.
FusedPlan plan_fused(int M, int V) {
  FusedPlan f;
  f.n_ttiles = cdiv(M, dg::unembed::TILE);
  f.segs = std::max(1, std::min(V / dg::unembed::TILE, (kNumSMs / 2) / f.n_ttiles));
  f.n_pairs = f.segs * f.n_ttiles;
  f.nparts = dg::unembed::SAMPLE_SLOTS * f.segs;  // one partial per epilogue warp set
  return f;
}

size_t fused_ws_bytes(int B, int C, int V) {
  const int M = B * C;
  const FusedPlan f = plan_fused(M, V);
  return align_up((size_t)M * f.nparts * sizeof(dg::FusedPartial), 256) +
         align_up((size_t)M * sizeof(dg::RowStats), 256);
}

PerDeviceFlag fused_attr_done;

int launch_unembed_sample(const void* h, const void* w_u, int d, const float* ssq_in,
                          int n_ssq_in, float inv_k, float eps, int32_t* tok,
                          uint8_t* committed, int32_t* prev_argmax, int32_t* seq_status,
                          const dg::SampleParams& sp, const dg_step_out* out, void* ws,
                          cudaStream_t s, const Fp8Scales* f8 = nullptr) {
  namespace ue = dg::unembed;
  const int M = sp.B * sp.C, V = sp.V;
  const FusedPlan f = plan_fused(M, V);
  if (!fused_attr_done()) {
    DG_CUDA(cudaFuncSetAttribute(ue::unembed_sample_kernel<1, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, ue::SMEM_BYTES));
    DG_CUDA(cudaFuncSetAttribute(ue::unembed_sample_kernel<2, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, ue::SMEM_BYTES));
    DG_CUDA(cudaFuncSetAttribute(ue::unembed_sample_kernel<1, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, ue::SMEM_BYTES));
    DG_CUDA(cudaFuncSetAttribute(ue::unembed_sample_kernel<2, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, ue::SMEM_BYTES));
    fused_attr_done() = true;
  }
  dg::FusedPartial* part = (dg::FusedPartial*)ws;
  dg::RowStats* stats = (dg::RowStats*)((char*)ws + align_up((size_t)M * f.nparts *
                                                             sizeof(dg::FusedPartial), 256));
  CUtensorMap tx, tw;
  if (f8) {
    DG_TRY(make_tmap_u8(&tx, h, d, M, (uint64_t)d, ue::HALF));
    DG_TRY(make_tmap_u8(&tw, w_u, d, V, (uint64_t)d, ue::HALF));
  } else {
    DG_TRY(make_tmap(&tx, h, d, M, (uint64_t)d * 2, ue::HALF));
    DG_TRY(make_tmap(&tw, w_u, d, V, (uint64_t)d * 2, ue::HALF));
  }
  ue::SampleFusedParams p;
  p.M = M; p.N = V; p.K = d;
  p.n_vtiles = V / ue::TILE;
  p.segs = f.segs;
  p.n_pairs = f.n_pairs;
  p.ssq_in = ssq_in; p.n_ssq_in = n_ssq_in; p.inv_k = inv_k; p.eps = eps;
  p.tok_scale = f8 ? f8->tok : nullptr;
  p.w_scale = f8 ? f8->w : nullptr;
  p.sp = sp;
  p.tok = tok;
  p.part = part;
  // two k-blocks per stage (256 contiguous bytes of each weight row per
  // request: 4% faster than one) when the width allows
  const int nkb = f8 ? d / 128 : d / 64;  // 128-byte k-blocks per row
  auto* kern = f8 ? (nkb % 2 == 0 ? ue::unembed_sample_kernel<2, true>
                                  : ue::unembed_sample_kernel<1, true>)
                  : (nkb % 2 == 0 ? ue::unembed_sample_kernel<2, false>
                                  : ue::unembed_sample_kernel<1, false>);
  DG_CUDA(launch_cluster(kern, dim3(2 * f.n_pairs),
                         dim3(ue::threads_for(ue::SAMPLE_EPI_WARPS)), ue::SMEM_BYTES, s,
                         dim3(2, 1, 1), tx, tw, p));
  count_launch();
  DG_CUDA(launch_ex(dg::sample_merge_kernel, dim3(cdiv(M, dg::MERGE_WARPS)),
                    dim3(dg::MERGE_WARPS * 32), 0, s, 1, (const dg::FusedPartial*)part, f.nparts,
                    (const uint8_t*)committed, sp, stats));
  count_launch();
  const int threads = (sp.C + 31) / 32 * 32;
  dg::SampleParams pc = sp;
  pc.near_ties = out ? out->near_ties : nullptr;
  DG_CUDA(launch_ex(dg::sample_commit_kernel, dim3(sp.B), dim3(threads), 0, s, 1,
                    (const float*)nullptr, (const dg::RowPartial*)nullptr,
                    (const dg::RowStats*)stats, pc, tok, committed, prev_argmax, seq_status,
                    out ? out->x_hat : (int32_t*)nullptr, out ? out->argmax : (int32_t*)nullptr,
                    out ? out->logconf : (float*)nullptr, out ? out->entropy : (float*)nullptr,
                    out ? out->flags : (uint8_t*)nullptr));
  count_launch();
  return DG_OK;
}

// ---------------------------------------------------------------------------
// KV commit
// ---------------------------------------------------------------------------
int launch_kv_commit(const void* const* k_blk, const void* const* v_blk, int ld_blk,
                     void* const* k_cache, void* const* v_cache, const int32_t* cache_len,
                     int n_layers, int B, int Hkv, int C, int hd, int lmax, cudaStream_t s) {
  dg::KVTables tab;
  memset(&tab, 0, sizeof(tab));
  for (int l = 0; l < n_layers; ++l) {
    tab.k_blk[l] = (const __nv_bfloat16*)k_blk[l];
    tab.v_blk[l] = (const __nv_bfloat16*)v_blk[l];
    tab.k_cache[l] = (__nv_bfloat16*)k_cache[l];
    tab.v_cache[l] = (__nv_bfloat16*)v_cache[l];
  }
  dg::KVParams p{n_layers, B, Hkv, C, hd, lmax, ld_blk, cache_len};
  // one grid row per (layer, K or V, sequence, kv head); x covers its vectors
  const int groups = n_layers * 2 * B * Hkv;
  const int nvec = C * (hd / 8);
  const int bx = std::max(1, std::min(cdiv(nvec, dg::KV_THREADS * dg::KV_UNROLL),
                                      cdiv(8 * kNumSMs, std::max(1, groups))));
  if (groups > 65535) return fail(DG_ERR_UNSUPPORTED_SHAPE, "kv commit: too many row groups");
  dg::kv_commit_kernel<<<dim3(bx, groups), dg::KV_THREADS, 0, s>>>(tab, p);
  count_launch();
  DG_CUDA(cudaGetLastError());
  return DG_OK;
}

// ---------------------------------------------------------------------------
// Model forward
// ---------------------------------------------------------------------------
int check_model(const dg_model* m) {
  if (!m || !m->embed || !m->unembed || !m->layers)
    return fail(DG_ERR_INVALID_ARG, "model: null pointer");
  const dg_model_cfg& c = m->cfg;
  if (c.d <= 0 || c.n_layers <= 0 || c.n_layers > dg::KV_MAX_LAYERS || c.n_q_heads <= 0 ||
      c.n_kv_heads <= 0 || c.n_q_heads % c.n_kv_heads != 0 || c.ffn <= 0 || c.vocab <= 0)
    return fail(DG_ERR_INVALID_ARG, "model: bad configuration");
  if (c.head_dim != 64 && c.head_dim != 128)
    return fail(DG_ERR_UNSUPPORTED_SHAPE, "head_dim %d not in {64,128}", c.head_dim);
  if (c.d % 128 || c.ffn % 128 || c.vocab % 128 || (c.n_q_heads * c.head_dim) % 128 ||
      ((c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim) % 128)
    return fail(DG_ERR_UNSUPPORTED_SHAPE,
                "d, ffn, vocab, Hq*hd and (Hq+2Hkv)*hd must be multiples of 128");
  if (!aligned16(m->embed) || !aligned16(m->unembed))
    return fail(DG_ERR_ALIGNMENT, "model: embed/unembed not 16-byte aligned");
  if ((m->unembed_e4m3 != nullptr) != (m->unembed_scale != nullptr))
    return fail(DG_ERR_INVALID_ARG, "model: unembed_e4m3 and unembed_scale go together");
  if (m->unembed_e4m3 && (!aligned16(m->unembed_e4m3) || c.vocab % dg::unembed::TILE))
    return fail(DG_ERR_UNSUPPORTED_SHAPE,
                "model: the e4m3 unembedding needs vocab %% 256 == 0 and 16-byte alignment");
  if (m->layers_e4m3) {
    for (int l = 0; l < c.n_layers; ++l) {
      const dg_layer_weights_e4m3& q = m->layers_e4m3[l];
      if (!q.w_qkv || !q.w_o || !q.w_up || !q.w_down || !q.scales)
        return fail(DG_ERR_INVALID_ARG, "model: e4m3 layer %d has a null pointer", l);
      if (!aligned16(q.w_qkv) || !aligned16(q.w_o) || !aligned16(q.w_up) || !aligned16(q.w_down))
        return fail(DG_ERR_ALIGNMENT, "model: e4m3 layer %d weight not 16-byte aligned", l);
    }
  }
  for (int l = 0; l < c.n_layers; ++l) {
    const dg_layer_weights& w = m->layers[l];
    if (!w.w_qkv || !w.w_o || !w.w_up || !w.w_down)
      return fail(DG_ERR_INVALID_ARG, "model: layer %d has a null weight", l);
    if (!aligned16(w.w_qkv) || !aligned16(w.w_o) || !aligned16(w.w_up) || !aligned16(w.w_down))
      return fail(DG_ERR_ALIGNMENT, "model: layer %d weight not 16-byte aligned", l);
  }
  return DG_OK;
}

int check_state(const dg_state* st, const dg_model_cfg& c, bool need_canvas) {
  if (!st || !st->k_cache || !st->v_cache || !st->cache_len)
    return fail(DG_ERR_INVALID_ARG, "state: null pointer");
  if (st->batch <= 0 || st->lmax <= 0) return fail(DG_ERR_INVALID_ARG, "state: bad batch/lmax");
  if (need_canvas) {
    if (!st->tok || !st->committed || !st->prev_argmax || !st->seq_status || !st->step)
      return fail(DG_ERR_INVALID_ARG, "state: null canvas pointer");
    if (st->canvas <= 0 || st->canvas > 1024)
      return fail(DG_ERR_UNSUPPORTED_SHAPE, "canvas %d not in [1, 1024]", st->canvas);
  }
  for (int l = 0; l < c.n_layers; ++l)
    if (!st->k_cache[l] || !st->v_cache[l] || !aligned16(st->k_cache[l]) ||
        !aligned16(st->v_cache[l]))
      return fail(DG_ERR_ALIGNMENT, "state: cache of layer %d null or misaligned", l);
  return DG_OK;
}

// Workspace carve-up for a forward over M = B * Lq rows.
struct FwdLayout {
  size_t x, xn, qkv, ao, up, attn, logits, spart, flag, aq, as, total;
};

FwdLayout fwd_layout(const dg_model_cfg& c, int B, int Lq, int max_prefix, bool logits) {
  FwdLayout L;
  const int M = B * Lq;
  const int nqkv = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim;
  const int hqd = c.n_q_heads * c.head_dim;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.x = take((size_t)M * c.d * 4);
  L.xn = take((size_t)M * c.d * 2);
  L.qkv = take((size_t)M * nqkv * 2);
  L.ao = take((size_t)M * hqd * 2);
  L.up = take((size_t)M * c.ffn * 2);
  L.attn = take(attn_ws_bytes(B, c.n_q_heads, c.n_kv_heads, Lq, c.head_dim, max_prefix));
  L.logits = take(logits ? (size_t)M * c.vocab * 4 : 0);
  L.spart = take(logits ? std::max(sample_ws_bytes(B, Lq, c.vocab),
                                    c.vocab % dg::unembed::TILE == 0
                                        ? fused_ws_bytes(B, Lq, c.vocab) : (size_t)0)
                         : 0);
  L.flag = take(logits ? 16 : 0);
  // e4m3 codes and per-token scales of the input of the next FP8 projection
  // (or of the final hidden states for the FP8 unembedding)
  L.aq = take((size_t)M * std::max(std::max(c.d, hqd), c.ffn));
  L.as = take((size_t)M * sizeof(float));
  L.total = off;
  return L;
}

struct Fwd {
  const dg_model* m;
  int B, Lq, max_prefix, lmax, mask;
  const int32_t* cache_len;
  void* const* k_cache;
  void* const* v_cache;
  bool commit_kv;   // write each layer's new K/V into the cache at cache_len
  bool want_logits;  // run the whole stack and (unless unembed_elsewhere) the unembedding
  char* ws;
  FwdLayout L;
  bool unembed_elsewhere = false;  // the caller fuses the unembedding into its sampler step
};

// A bf16 activation [B*Lq, cols] quantised per token to e4m3 codes (L.aq)
// and scales (L.as): the normalised residual stream, the attention output or
// the GELU output, as stored in bf16.
int quantize_act(const Fwd& f, const void* in, int cols, cudaStream_t s) {
  DG_CUDA(launch_ex(dg::quant::quantize_rows_kernel, dim3(f.B * f.Lq), dim3(dg::quant::THREADS),
                    0, s, 1, (const __nv_bfloat16*)in, f.B * f.Lq, cols,
                    (uint8_t*)(f.ws + f.L.aq), (float*)(f.ws + f.L.as)));
  count_launch();
  return DG_OK;
}

// The final normalised hidden states, quantised for the FP8 unembedding.
int quantize_hidden(const Fwd& f, cudaStream_t s) {
  return quantize_act(f, f.ws + f.L.xn, f.m->cfg.d, s);
}

int run_forward(const Fwd& f, const int32_t* tok, float* logits, cudaStream_t s) {
  const dg_model_cfg& c = f.m->cfg;
  const int M = f.B * f.Lq;
  const int hd = c.head_dim, hq = c.n_q_heads, hkv = c.n_kv_heads;
  const int nqkv = (hq + 2 * hkv) * hd;
  float* x = (float*)(f.ws + f.L.x);                      // residual stream, fp32
  __nv_bfloat16* xn = (__nv_bfloat16*)(f.ws + f.L.xn);    // bf16(RMSNorm(x)), the next input
  __nv_bfloat16* qkv = (__nv_bfloat16*)(f.ws + f.L.qkv);
  __nv_bfloat16* ao = (__nv_bfloat16*)(f.ws + f.L.ao);
  __nv_bfloat16* up = (__nv_bfloat16*)(f.ws + f.L.up);
  void* aws = f.ws + f.L.attn;
  const float scale = 1.0f / std::sqrt((float)hd);
  // xn = bf16(RMSNorm(x)) after each residual update: a warp per row while
  // the row fits in its registers
  auto norm = [&]() -> int {
    namespace nm = dg::norm;
    const dim3 rows_grid(cdiv(M, nm::ROW_WARPS)), rows_block(nm::ROW_WARPS * 32);
    const float inv_d = 1.f / c.d;
    cudaError_t e;
    switch (c.d % 128 == 0 && c.d <= nm::ROW_MAX_D ? c.d / 128 : 0) {
      case 1: e = launch_ex(nm::rmsnorm_rows_kernel<1>, rows_grid, rows_block, 0, s, 1,
                            (const float*)x, M, c.d, inv_d, c.eps, xn); break;
      case 2: e = launch_ex(nm::rmsnorm_rows_kernel<2>, rows_grid, rows_block, 0, s, 1,
                            (const float*)x, M, c.d, inv_d, c.eps, xn); break;
      case 4: e = launch_ex(nm::rmsnorm_rows_kernel<4>, rows_grid, rows_block, 0, s, 1,
                            (const float*)x, M, c.d, inv_d, c.eps, xn); break;
      case 8: e = launch_ex(nm::rmsnorm_rows_kernel<8>, rows_grid, rows_block, 0, s, 1,
                            (const float*)x, M, c.d, inv_d, c.eps, xn); break;
      case 16: e = launch_ex(nm::rmsnorm_rows_kernel<16>, rows_grid, rows_block, 0, s, 1,
                             (const float*)x, M, c.d, inv_d, c.eps, xn); break;
      case 32: e = launch_ex(nm::rmsnorm_rows_kernel<32>, rows_grid, rows_block, 0, s, 1,
                             (const float*)x, M, c.d, inv_d, c.eps, xn); break;
      default: e = launch_ex(nm::rmsnorm_kernel, dim3(M), dim3(nm::NORM_THREADS), 0, s, 1,
                             (const float*)x, c.d, inv_d, c.eps, xn); break;
    }
    DG_CUDA(e);
    count_launch();
    return DG_OK;
  };

  DG_CUDA(launch_ex(dg::norm::embed_norm_kernel, dim3(M), dim3(dg::norm::NORM_THREADS), 0, s, 1,
                    tok, (const __nv_bfloat16*)f.m->embed, c.vocab, c.d, 1.f / c.d, c.eps, x,
                    xn));
  count_launch();
  for (int l = 0; l < c.n_layers; ++l) {
    const dg_layer_weights& w = f.m->layers[l];
    const bool last = l == c.n_layers - 1;
    const dg_layer_weights_e4m3* q8 = f.m->layers_e4m3 ? &f.m->layers_e4m3[l] : nullptr;
    // y = epilogue(in w^T): bf16, or e4m3 with the input quantised per token
    auto proj = [&](const void* in, const void* wb, const uint8_t* wq, int widx, int N, int K,
                    const GemmEpi& e) -> int {
      if (!q8) return linear(in, wb, M, N, K, e, s, nullptr);
      DG_TRY(quantize_act(f, in, K, s));
      const Fp8Scales f8{(const float*)(f.ws + f.L.as), q8->scales + widx};
      return linear(f.ws + f.L.aq, wq, M, N, K, e, s, &f8);
    };
    GemmEpi eq;  // QKV of RMSNorm(x)
    eq.epi = dg::gemm::EPI_BF16;
    eq.out_bf16 = qkv;
    DG_TRY(proj(xn, w.w_qkv, q8 ? q8->w_qkv : nullptr, 0, nqkv, c.d, eq));
    if (f.commit_kv) {
      const void* kb = qkv + hq * hd;
      const void* vb = qkv + (hq + hkv) * hd;
      DG_TRY(launch_kv_commit(&kb, &vb, nqkv, &f.k_cache[l], &f.v_cache[l], f.cache_len, 1,
                              f.B, hkv, f.Lq, hd, f.lmax, s));
    }
    if (last && !f.want_logits) break;
    DG_TRY(launch_attn(qkv, nqkv, qkv + hq * hd, qkv + (hq + hkv) * hd, nqkv, f.k_cache[l],
                       f.v_cache[l], f.cache_len, f.max_prefix, f.lmax, ao, hq * hd, nullptr,
                       f.B, hq, hkv, f.Lq, hd, scale, f.mask, aws, s));
    GemmEpi eo;  // h = x + O w_o^T
    eo.epi = dg::gemm::EPI_RESID;
    eo.x = x;
    DG_TRY(proj(ao, w.w_o, q8 ? q8->w_o : nullptr, 1, c.d, hq * hd, eo));
    DG_TRY(norm());
    GemmEpi eu;  // gelu(RMSNorm(h) w_up^T)
    eu.epi = dg::gemm::EPI_GELU;
    eu.out_bf16 = up;
    DG_TRY(proj(xn, w.w_up, q8 ? q8->w_up : nullptr, 2, c.ffn, c.d, eu));
    GemmEpi ed;  // x = h + u w_down^T
    ed.epi = dg::gemm::EPI_RESID;
    ed.x = x;
    DG_TRY(proj(up, w.w_down, q8 ? q8->w_down : nullptr, 3, c.d, c.ffn, ed));
    DG_TRY(norm());  // the next layer's input, or the unembedding's after the last layer
  }
  if (f.want_logits && !f.unembed_elsewhere) {
    // logits of RMSNorm(x), on e4m3 operands when the model carries them
    if (f.m->unembed_e4m3) {
      DG_TRY(quantize_hidden(f, s));
      const Fp8Scales f8{(const float*)(f.ws + f.L.as), f.m->unembed_scale};
      DG_TRY(launch_unembed(f.ws + f.L.aq, f.m->unembed_e4m3, logits, M, c.d, c.vocab, nullptr,
                            0, 1.f / c.d, c.eps, s, &f8));
    } else {
      DG_TRY(launch_unembed(xn, f.m->unembed, logits, M, c.d, c.vocab, nullptr, 0, 1.f / c.d,
                            c.eps, s));
    }
  }
  return DG_OK;
}

// ---------------------------------------------------------------------------
// dg_sample_commit_noalloc: the sampler step with its scratch in a fixed
// device array instead of a caller-supplied workspace.
//
// For callers that cannot allocate device memory: a plugin whose host
// application owns every device allocation, or code that enqueues work while
// a stream is being captured, where cudaMalloc is not allowed.  The row
// partials live in kNoallocScratchBytes of static device memory that every
// GPU loading this library keeps until the process exits.  Host code may not
// hand the array's name to a kernel (in host code it is only a stand-in for
// the device symbol), so the device address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the
// first call there.
// ---------------------------------------------------------------------------
constexpr size_t kNoallocScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

int noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  DG_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(DG_ERR_INVALID_ARG, "device ordinal %d >= 64", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(DG_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed on device %d: %s", dev,
                  cudaGetErrorString(e));
    addr[dev] = p;
  }
  *out = addr[dev];
  return DG_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
// A captured denoising step: the launches are recorded on a private stream
// (launch counts included) and replayed with cudaGraphLaunch on the caller's
// stream.  A failed capture leaves exec null and the caller launches directly.
struct StepGraph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  unsigned long long launches = 0;  // kernels per replay
  ~StepGraph() {
    if (exec) cudaGraphExecDestroy(exec);
    if (graph) cudaGraphDestroy(graph);
  }
  template <class F>
  int capture(F&& enqueue) {
    static cudaStream_t streams[64] = {};  // one private capture stream per device
    int dev = 0;
    DG_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return DG_OK;  // no capture: launch the steps directly
    if (!streams[dev]) DG_CUDA(cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking));
    cudaStream_t cs = streams[dev];
    const unsigned long long c0 = g_launches.load(std::memory_order_relaxed);
    DG_CUDA(cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal));
    const int rc = enqueue(cs);
    const cudaError_t end = cudaStreamEndCapture(cs, &graph);
    launches = g_launches.load(std::memory_order_relaxed) - c0;
    g_launches.fetch_sub(launches, std::memory_order_relaxed);  // recorded, not run
    if (rc != DG_OK) return rc;
    if (end != cudaSuccess || cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) {
      (void)cudaGetLastError();
      exec = nullptr;  // launch the steps directly instead
    }
    return DG_OK;
  }
  int launch(cudaStream_t s) {
    DG_CUDA(cudaGraphLaunch(exec, s));
    count_launch(launches);
    return DG_OK;
  }
};

extern "C" {

const char* dg_status_string(int status) {
  switch (status) {
    case DG_OK: return "DG_OK";
    case DG_ERR_INVALID_ARG: return "DG_ERR_INVALID_ARG";
    case DG_ERR_UNSUPPORTED_SHAPE: return "DG_ERR_UNSUPPORTED_SHAPE";
    case DG_ERR_ALIGNMENT: return "DG_ERR_ALIGNMENT";
    case DG_ERR_WORKSPACE_TOO_SMALL: return "DG_ERR_WORKSPACE_TOO_SMALL";
    case DG_ERR_CUDA: return "DG_ERR_CUDA";
    case DG_ERR_TIMEOUT: return "DG_ERR_TIMEOUT";
    case DG_ERR_DEVICE_CHECK: return "DG_ERR_DEVICE_CHECK";
    default: return "DG_ERR_UNKNOWN";
  }
}

const char* dg_last_error(void) { return g_last_error; }

int dg_version(void) { return kVersion; }

unsigned long long dg_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void dg_sampler_defaults(dg_sampler_cfg* cfg) {
  if (!cfg) return;
  cfg->max_steps = 48;
  cfg->t_start = 0.8f;
  cfg->t_end = 0.4f;
  cfg->commit_k = 16;
  cfg->renoise_conf = 0.05f;
  cfg->stop_entropy = 0.005f;
  cfg->unselected_policy = DG_UNSELECTED_KEEP;
  cfg->selection = DG_SELECT_TOP_K;
  cfg->entropy_bound = 0.1f;
}

int dg_check_device_errors(void* stream, uint32_t* code_out) {
  cudaStream_t s = (cudaStream_t)stream;
  DG_CUDA(cudaStreamSynchronize(s));
  uint32_t w[4];
  DG_CUDA(cudaMemcpyFromSymbol(w, dg::g_err, sizeof(w)));
  if (code_out) *code_out = w[0];
  if (w[0] == 0) return DG_OK;
  const uint32_t zero[4] = {0, 0, 0, 0};
  DG_CUDA(cudaMemcpyToSymbol(dg::g_err, zero, sizeof(zero)));
  if (w[0] & dg::ERR_TIMEOUT)
    return fail(DG_ERR_TIMEOUT, "device wait expired (site 0x%x, detail %u, %u errors)",
                w[0] & 0xFFFFu, w[2], w[1]);
  return fail(DG_ERR_DEVICE_CHECK, "device check failed (site 0x%x, detail %u, %u errors)",
              w[0] & 0xFFFFu, w[2], w[1]);
}

size_t dg_canvas_attn_workspace_bytes(int B, int Hq, int Hkv, int Lq, int hd, int max_prefix) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Lq <= 0 || (hd != 64 && hd != 128) ||
      max_prefix < 0)
    return 0;
  return attn_ws_bytes(B, Hq, Hkv, Lq, hd, max_prefix);
}

int dg_canvas_attn(const void* q, int ldq, const void* k_new, const void* v_new, int ldkv,
                   const void* k_cache, const void* v_cache, const int32_t* cache_len,
                   int max_prefix, int lmax, void* out, int ldo, float* lse, int B, int Hq,
                   int Hkv, int Lq, int hd, float scale, int mask_mode, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !cache_len || !out)
    return fail(DG_ERR_INVALID_ARG, "dg_canvas_attn: null pointer");
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Hq % Hkv || max_prefix < 0 || lmax < 1 ||
      max_prefix > lmax || (mask_mode != DG_MASK_BIDIR && mask_mode != DG_MASK_CAUSAL))
    return fail(DG_ERR_INVALID_ARG, "dg_canvas_attn: bad sizes or mask");
  if (hd != 64 && hd != 128)
    return fail(DG_ERR_UNSUPPORTED_SHAPE, "dg_canvas_attn: head_dim %d not in {64,128}", hd);
  if (ldq % 8 || ldkv % 8 || ldo % 8 || ldq < Hq * hd || ldkv < Hkv * hd || ldo < Hq * hd)
    return fail(DG_ERR_ALIGNMENT, "dg_canvas_attn: leading dimensions");
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(out))
    return fail(DG_ERR_ALIGNMENT, "dg_canvas_attn: pointers must be 16-byte aligned");
  const size_t need = attn_ws_bytes(B, Hq, Hkv, Lq, hd, max_prefix);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(DG_ERR_WORKSPACE_TOO_SMALL, "dg_canvas_attn: workspace needs %zu bytes", need);
  return launch_attn(q, ldq, k_new, v_new, ldkv, k_cache, v_cache, cache_len, max_prefix, lmax,
                     out, ldo, lse, B, Hq, Hkv, Lq, hd, scale, mask_mode, workspace,
                     (cudaStream_t)stream);
}

int dg_canvas_attn_e4m3(const uint8_t* q, int ldq, const float* q_scale, const uint8_t* k_new,
                        int ldkv, const uint8_t* vt_new, int ldvt, const uint8_t* k_cache,
                        const uint8_t* vt_cache, const float* k_scale, const float* v_scale,
                        const int32_t* cache_len, int max_prefix, int lmax, void* out, int ldo,
                        float* lse, int B, int Hq, int Hkv, int Lq, int hd, float scale,
                        int mask_mode, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !q_scale || !k_new || !vt_new || !k_cache || !vt_cache || !k_scale || !v_scale ||
      !cache_len || !out)
    return fail(DG_ERR_INVALID_ARG, "dg_canvas_attn_e4m3: null pointer");
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Hq % Hkv || max_prefix < 0 || lmax < 1 ||
      max_prefix > lmax || (mask_mode != DG_MASK_BIDIR && mask_mode != DG_MASK_CAUSAL))
    return fail(DG_ERR_INVALID_ARG, "dg_canvas_attn_e4m3: bad sizes or mask");
  if (hd != 128)
    return fail(DG_ERR_UNSUPPORTED_SHAPE, "dg_canvas_attn_e4m3: head_dim %d is not 128", hd);
  if (ldq % 16 || ldkv % 16 || ldvt % 16 || lmax % 16 || ldo % 8 || ldq < Hq * hd ||
      ldkv < Hkv * hd || ldvt < Lq || ldo < Hq * hd)
    return fail(DG_ERR_ALIGNMENT, "dg_canvas_attn_e4m3: leading dimensions");
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(vt_new) || !aligned16(k_cache) ||
      !aligned16(vt_cache) || !aligned16(out))
    return fail(DG_ERR_ALIGNMENT, "dg_canvas_attn_e4m3: pointers must be 16-byte aligned");
  const size_t need = attn_ws_bytes(B, Hq, Hkv, Lq, hd, max_prefix);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(DG_ERR_WORKSPACE_TOO_SMALL, "dg_canvas_attn_e4m3: workspace needs %zu bytes",
                need);
  return launch_attn_e4m3(q, ldq, q_scale, k_new, ldkv, vt_new, ldvt, k_cache, vt_cache, k_scale,
                          v_scale, cache_len, max_prefix, lmax, out, ldo, lse, B, Hq, Hkv, Lq,
                          scale, mask_mode, workspace, (cudaStream_t)stream);
}

int dg_unembed(const void* h, const void* w_u, float* logits, int M, int d, int V,
               void* workspace, size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (!h || !w_u || !logits) return fail(DG_ERR_INVALID_ARG, "dg_unembed: null pointer");
  if (M <= 0 || d <= 0 || V <= 0) return fail(DG_ERR_INVALID_ARG, "dg_unembed: bad sizes");
  if (V % 128 || d % 64)
    return fail(DG_ERR_UNSUPPORTED_SHAPE, "dg_unembed: V %% 128 and d %% 64 must be 0");
  if (!aligned16(h) || !aligned16(w_u) || !aligned16(logits))
    return fail(DG_ERR_ALIGNMENT, "dg_unembed: pointers must be 16-byte aligned");
  return launch_unembed(h, w_u, logits, M, d, V, nullptr, 0, 0.f, 0.f, (cudaStream_t)stream);
}

int dg_linear_plan_of(int M, int N, int K, int e4m3) {
  const int kbe = e4m3 ? 128 : dg::gemm::BK;
  if (M <= 0 || N <= 0 || K <= 0 || N % 128 || K % kbe) return -1;
  return proj_use_pair(M, N, K, e4m3 != 0) ? DG_PLAN_PAIRS : DG_PLAN_SPLIT_K;
}

int dg_model_residual_on_pairs(const dg_model_cfg* cfg, int M, int e4m3) {
  if (!cfg || M < 1) return -1;
  return resid_on_pair(*cfg, M, e4m3 != 0) ? 1 : 0;
}

size_t dg_linear_workspace_bytes(int M, int N, int K) {
  (void)M;
  (void)N;
  (void)K;
  return 0;  // split-K partial sums stay in the cluster's shared memory
}

int dg_linear(const void* x, const void* w, void* out, int M, int N, int K, int epilogue,
              void* workspace, size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (!x || !w || !out) return fail(DG_ERR_INVALID_ARG, "dg_linear: null pointer");
  if (M <= 0 || N <= 0 || K <= 0 || epilogue < 0 || epilogue > DG_EPI_RESID_F32)
    return fail(DG_ERR_INVALID_ARG, "dg_linear: bad sizes or epilogue");
  if (N % 128 || K % 64)
    return fail(DG_ERR_UNSUPPORTED_SHAPE, "dg_linear: N %% 128 and K %% 64 must be 0");
  if (!aligned16(x) || !aligned16(w) || !aligned16(out))
    return fail(DG_ERR_ALIGNMENT, "dg_linear: pointers must be 16-byte aligned");
  GemmEpi e;
  if (epilogue == DG_EPI_F32) {
    e.epi = dg::gemm::EPI_F32;
    e.out_f32 = (float*)out;
  } else if (epilogue == DG_EPI_BF16) {
    e.epi = dg::gemm::EPI_BF16;
    e.out_bf16 = (__nv_bfloat16*)out;
  } else if (epilogue == DG_EPI_GELU_BF16) {
    e.epi = dg::gemm::EPI_GELU;
    e.out_bf16 = (__nv_bfloat16*)out;
  } else {
    e.epi = dg::gemm::EPI_RESID;
    e.x = (float*)out;
  }
  return linear(x, w, M, N, K, e, (cudaStream_t)stream);
}

int dg_linear_e4m3(const uint8_t* x_q, const float* x_scale, const uint8_t* w_q,
                   const float* w_scale, void* out, int M, int N, int K, int epilogue,
                   void* stream) {
  if (!x_q || !x_scale || !w_q || !w_scale || !out)
    return fail(DG_ERR_INVALID_ARG, "dg_linear_e4m3: null pointer");
  if (M <= 0 || N <= 0 || K <= 0 || epilogue < 0 || epilogue > DG_EPI_RESID_F32)
    return fail(DG_ERR_INVALID_ARG, "dg_linear_e4m3: bad sizes or epilogue");
  if (N % 128 || K % 128)
    return fail(DG_ERR_UNSUPPORTED_SHAPE, "dg_linear_e4m3: N %% 128 and K %% 128 must be 0");
  if (!aligned16(x_q) || !aligned16(w_q) || !aligned16(out))
    return fail(DG_ERR_ALIGNMENT, "dg_linear_e4m3: pointers must be 16-byte aligned");
  GemmEpi e;
  if (epilogue == DG_EPI_F32) {
    e.epi = dg::gemm::EPI_F32;
    e.out_f32 = (float*)out;
  } else if (epilogue == DG_EPI_BF16) {
    e.epi = dg::gemm::EPI_BF16;
    e.out_bf16 = (__nv_bfloat16*)out;
  } else if (epilogue == DG_EPI_GELU_BF16) {
    e.epi = dg::gemm::EPI_GELU;
    e.out_bf16 = (__nv_bfloat16*)out;
  } else {
    e.epi = dg::gemm::EPI_RESID;
    e.x = (float*)out;
  }
  const Fp8Scales f8{x_scale, w_scale};
  return linear(x_q, w_q, M, N, K, e, (cudaStream_t)stream, &f8);
}

size_t dg_sample_commit_workspace_bytes(int B, int C, int V) {
  if (B <= 0 || C <= 0 || V <= 0) return 0;
  return sample_ws_bytes(B, C, V);
}

int dg_sample_commit(const float* logits, int32_t* tok, uint8_t* committed,
                     int32_t* prev_argmax, int32_t* seq_status, const dg_sampler_cfg* cfg,
                     uint32_t seed, int block, int step, int B, int C, int V,
                     const dg_step_out* out, void* workspace, size_t workspace_bytes,
                     void* stream) {
  if (!logits || !tok || !committed || !prev_argmax || !seq_status || !cfg)
    return fail(DG_ERR_INVALID_ARG, "dg_sample_commit: null pointer");
  if (B <= 0 || C <= 0 || C > 1024 || V <= 0 || V % 4 || step < 0 || block < 0)
    return fail(DG_ERR_UNSUPPORTED_SHAPE, "dg_sample_commit: need C <= 1024, V %% 4 == 0");
  if (!sampler_cfg_ok(*cfg))
    return fail(DG_ERR_INVALID_ARG, "dg_sample_commit: bad sampler settings");
  if (!aligned16(logits)) return fail(DG_ERR_ALIGNMENT, "dg_sample_commit: logits alignment");
  const size_t need = sample_ws_bytes(B, C, V);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(DG_ERR_WORKSPACE_TOO_SMALL, "dg_sample_commit: workspace needs %zu bytes", need);
  const dg::SampleParams p = make_sample_params(*cfg, seed, block, nullptr, step, B, C, V);
  return launch_sample(logits, tok, committed, prev_argmax, seq_status, p, out, workspace,
                       (cudaStream_t)stream);
}

size_t dg_unembed_sample_commit_workspace_bytes(int B, int C, int V) {
  if (B <= 0 || C <= 0 || V <= 0 || V % dg::unembed::TILE) return 0;
  return fused_ws_bytes(B, C, V);
}

int dg_unembed_sample_commit(const void* h, const void* w_u, int d, int32_t* tok,
                             uint8_t* committed, int32_t* prev_argmax, int32_t* seq_status,
                             const dg_sampler_cfg* cfg, uint32_t seed, int block, int step,
                             int B, int C, int V, const dg_step_out* out, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (!h || !w_u || !tok || !committed || !prev_argmax || !seq_status || !cfg)
    return fail(DG_ERR_INVALID_ARG, "dg_unembed_sample_commit: null pointer");
  if (B <= 0 || C <= 0 || C > 1024 || V <= 0 || V % dg::unembed::TILE || d <= 0 || d % 64 ||
      step < 0 || block < 0)
    return fail(DG_ERR_UNSUPPORTED_SHAPE,
                "dg_unembed_sample_commit: need C <= 1024, V %% 256 == 0, d %% 64 == 0");
  if (!sampler_cfg_ok(*cfg))
    return fail(DG_ERR_INVALID_ARG, "dg_unembed_sample_commit: bad sampler settings");
  if (!aligned16(h) || !aligned16(w_u))
    return fail(DG_ERR_ALIGNMENT, "dg_unembed_sample_commit: pointers must be 16-byte aligned");
  const size_t need = fused_ws_bytes(B, C, V);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(DG_ERR_WORKSPACE_TOO_SMALL,
                "dg_unembed_sample_commit: workspace needs %zu bytes", need);
  const dg::SampleParams p = make_sample_params(*cfg, seed, block, nullptr, step, B, C, V);
  return launch_unembed_sample(h, w_u, d, nullptr, 0, 0.f, 0.f, tok, committed, prev_argmax,
                               seq_status, p, out, workspace, (cudaStream_t)stream);
}

int dg_quantize_e4m3(const void* in, int rows, int cols, int per_row, uint8_t* out,
                     float* scales, void* stream) {
  if (!in || !out || !scales) return fail(DG_ERR_INVALID_ARG, "dg_quantize_e4m3: null pointer");
  if (rows <= 0 || cols <= 0 || cols % 8)
    return fail(DG_ERR_UNSUPPORTED_SHAPE, "dg_quantize_e4m3: need cols %% 8 == 0");
  if (!aligned16(in) || !aligned16(out))
    return fail(DG_ERR_ALIGNMENT, "dg_quantize_e4m3: pointers must be 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  namespace qt = dg::quant;
  if (per_row) {
    DG_CUDA(launch_ex(qt::quantize_rows_kernel, dim3(rows), dim3(qt::THREADS), 0, s, 1,
                      (const __nv_bfloat16*)in, rows, cols, out, scales));
    count_launch();
    return DG_OK;
  }
  const size_t n = (size_t)rows * cols;
  const int blocks = (int)std::min<size_t>(4 * kNumSMs, (n / 8 + qt::THREADS - 1) / qt::THREADS);
  DG_CUDA(cudaMemsetAsync(scales, 0, sizeof(float), s));
  qt::absmax_kernel<<<blocks, qt::THREADS, 0, s>>>((const __nv_bfloat16*)in, n,
                                                   (unsigned int*)scales);
  qt::quantize_tensor_kernel<<<blocks, qt::THREADS, 0, s>>>(
      (const __nv_bfloat16*)in, n, out, (const unsigned int*)scales);
  qt::amax_to_scale_kernel<<<1, 1, 0, s>>>((unsigned int*)scales);
  count_launch(3);
  DG_CUDA(cudaGetLastError());
  return DG_OK;
}

int dg_unembed_e4m3(const uint8_t* h_q, const float* h_scale, const uint8_t* w_q,
                    const float* w_scale, float* logits, int M, int d, int V, void* stream) {
  if (!h_q || !h_scale || !w_q || !w_scale || !logits)
    return fail(DG_ERR_INVALID_ARG, "dg_unembed_e4m3: null pointer");
  if (M <= 0 || d <= 0 || V <= 0 || V % dg::unembed::TILE || d % 128)
    return fail(DG_ERR_UNSUPPORTED_SHAPE, "dg_unembed_e4m3: need V %% 256 == 0, d %% 128 == 0");
  if (!aligned16(h_q) || !aligned16(w_q) || !aligned16(logits))
    return fail(DG_ERR_ALIGNMENT, "dg_unembed_e4m3: pointers must be 16-byte aligned");
  const Fp8Scales f8{h_scale, w_scale};
  return launch_unembed(h_q, w_q, logits, M, d, V, nullptr, 0, 0.f, 0.f, (cudaStream_t)stream,
                        &f8);
}

int dg_unembed_sample_commit_e4m3(const uint8_t* h_q, const float* h_scale, const uint8_t* w_q,
                                  const float* w_scale, int d, int32_t* tok, uint8_t* committed,
                                  int32_t* prev_argmax, int32_t* seq_status,
                                  const dg_sampler_cfg* cfg, uint32_t seed, int block, int step,
                                  int B, int C, int V, const dg_step_out* out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (!h_q || !h_scale || !w_q || !w_scale || !tok || !committed || !prev_argmax ||
      !seq_status || !cfg)
    return fail(DG_ERR_INVALID_ARG, "dg_unembed_sample_commit_e4m3: null pointer");
  if (B <= 0 || C <= 0 || C > 1024 || V <= 0 || V % dg::unembed::TILE || d <= 0 || d % 128 ||
      step < 0 || block < 0)
    return fail(DG_ERR_UNSUPPORTED_SHAPE,
                "dg_unembed_sample_commit_e4m3: need C <= 1024, V %% 256 == 0, d %% 128 == 0");
  if (!sampler_cfg_ok(*cfg))
    return fail(DG_ERR_INVALID_ARG, "dg_unembed_sample_commit_e4m3: bad sampler settings");
  if (!aligned16(h_q) || !aligned16(w_q))
    return fail(DG_ERR_ALIGNMENT,
                "dg_unembed_sample_commit_e4m3: pointers must be 16-byte aligned");
  const size_t need = fused_ws_bytes(B, C, V);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(DG_ERR_WORKSPACE_TOO_SMALL,
                "dg_unembed_sample_commit_e4m3: workspace needs %zu bytes", need);
  const dg::SampleParams p = make_sample_params(*cfg, seed, block, nullptr, step, B, C, V);
  const Fp8Scales f8{h_scale, w_scale};
  return launch_unembed_sample(h_q, w_q, d, nullptr, 0, 0.f, 0.f, tok, committed, prev_argmax,
                               seq_status, p, out, workspace, (cudaStream_t)stream, &f8);
}

int dg_sample_commit_noalloc(const float* logits, int32_t* tok, uint8_t* committed,
                             int32_t* prev_argmax, int32_t* seq_status, const dg_sampler_cfg* cfg,
                             uint32_t seed, int block, int step, int B, int C, int V,
                             const dg_step_out* out, void* stream) {
  if (!logits || !tok || !committed || !prev_argmax || !seq_status || !cfg)
    return fail(DG_ERR_INVALID_ARG, "dg_sample_commit_noalloc: null pointer");
  if (B <= 0 || C <= 0 || C > 1024 || V <= 0 || V % 4 || step < 0 || block < 0)
    return fail(DG_ERR_UNSUPPORTED_SHAPE,
                "dg_sample_commit_noalloc: need C <= 1024, V %% 4 == 0");
  if (!sampler_cfg_ok(*cfg))
    return fail(DG_ERR_INVALID_ARG, "dg_sample_commit_noalloc: bad sampler settings");
  if (!aligned16(logits))
    return fail(DG_ERR_ALIGNMENT, "dg_sample_commit_noalloc: logits alignment");
  const size_t need = sample_ws_bytes(B, C, V);
  if (need > kNoallocScratchBytes)
    return fail(DG_ERR_UNSUPPORTED_SHAPE,
                "dg_sample_commit_noalloc: B=%d C=%d V=%d needs %zu bytes of scratch, above the "
                "fixed %zu; use dg_sample_commit with a workspace",
                B, C, V, need, kNoallocScratchBytes);
  void* scratch = nullptr;
  DG_TRY(noalloc_scratch(&scratch));
  const dg::SampleParams p = make_sample_params(*cfg, seed, block, nullptr, step, B, C, V);
  return launch_sample(logits, tok, committed, prev_argmax, seq_status, p, out, scratch,
                       (cudaStream_t)stream);
}

int dg_kv_block_commit(const void* const* k_blk, const void* const* v_blk, int ld_blk,
                       void* const* k_cache, void* const* v_cache, int32_t* cache_len,
                       int n_layers, int B, int Hkv, int C, int hd, int lmax, void* stream) {
  if (!k_blk || !v_blk || !k_cache || !v_cache || !cache_len)
    return fail(DG_ERR_INVALID_ARG, "dg_kv_block_commit: null pointer");
  if (n_layers <= 0 || n_layers > dg::KV_MAX_LAYERS || B <= 0 || Hkv <= 0 || C <= 0 || lmax <= 0)
    return fail(DG_ERR_INVALID_ARG, "dg_kv_block_commit: bad sizes (n_layers <= %d)",
                dg::KV_MAX_LAYERS);
  if (hd != 64 && hd != 128)
    return fail(DG_ERR_UNSUPPORTED_SHAPE, "dg_kv_block_commit: head_dim %d not in {64,128}", hd);
  if (ld_blk % 8 || ld_blk < Hkv * hd)
    return fail(DG_ERR_ALIGNMENT, "dg_kv_block_commit: ld_blk must be a multiple of 8, >= Hkv hd");
  for (int l = 0; l < n_layers; ++l)
    if (!aligned16(k_blk[l]) || !aligned16(v_blk[l]) || !aligned16(k_cache[l]) ||
        !aligned16(v_cache[l]) || !k_blk[l] || !v_blk[l] || !k_cache[l] || !v_cache[l])
      return fail(DG_ERR_ALIGNMENT, "dg_kv_block_commit: layer %d pointer null or misaligned", l);
  cudaStream_t s = (cudaStream_t)stream;
  DG_TRY(launch_kv_commit(k_blk, v_blk, ld_blk, k_cache, v_cache, cache_len, n_layers, B, Hkv, C,
                          hd, lmax, s));
  dg::cache_len_bump_kernel<<<1, 256, 0, s>>>(cache_len, B, C, lmax);
  count_launch();
  DG_CUDA(cudaGetLastError());
  return DG_OK;
}

size_t dg_prefill_workspace_bytes(const dg_model_cfg* cfg, int B, int P) {
  if (!cfg || B <= 0 || P <= 0) return 0;
  return fwd_layout(*cfg, B, P, 0, false).total;
}

int dg_prefill(const dg_model* m, dg_state* st, const int32_t* prompt, int P, void* workspace,
               size_t workspace_bytes, void* stream) {
  DG_TRY(check_model(m));
  DG_TRY(check_state(st, m->cfg, false));
  if (!prompt || P <= 0 || P > st->lmax)
    return fail(DG_ERR_INVALID_ARG, "dg_prefill: bad prompt (P=%d, lmax=%d)", P, st->lmax);
  const FwdLayout L = fwd_layout(m->cfg, st->batch, P, 0, false);
  if (!workspace || workspace_bytes < L.total || !aligned16(workspace))
    return fail(DG_ERR_WORKSPACE_TOO_SMALL, "dg_prefill: workspace needs %zu bytes", L.total);
  cudaStream_t s = (cudaStream_t)stream;
  dg::cache_len_set_kernel<<<1, 256, 0, s>>>(st->cache_len, st->batch, 0);
  count_launch();
  DG_CUDA(cudaGetLastError());
  Fwd f{m, st->batch, P, 0, st->lmax, DG_MASK_CAUSAL, st->cache_len, st->k_cache,
        st->v_cache, true, false, (char*)workspace, L};
  DG_TRY(run_forward(f, prompt, nullptr, s));
  dg::cache_len_set_kernel<<<1, 256, 0, s>>>(st->cache_len, st->batch, P);
  count_launch();
  DG_CUDA(cudaGetLastError());
  st->cache_len_host = P;
  return DG_OK;
}

size_t dg_denoise_block_workspace_bytes(const dg_model_cfg* cfg, int B, int C, int lmax) {
  if (!cfg || B <= 0 || C <= 0 || lmax <= 0) return 0;
  return fwd_layout(*cfg, B, C, lmax, true).total;
}

int dg_denoise_logits(const dg_model* m, const dg_state* st, float* logits, void* workspace,
                      size_t workspace_bytes, void* stream) {
  DG_TRY(check_model(m));
  DG_TRY(check_state(st, m->cfg, true));
  if (!logits || !aligned16(logits))
    return fail(DG_ERR_INVALID_ARG, "dg_denoise_logits: logits null or misaligned");
  if (st->cache_len_host < 0 || st->cache_len_host > st->lmax)
    return fail(DG_ERR_INVALID_ARG, "dg_denoise_logits: cache_len_host out of range");
  const FwdLayout L = fwd_layout(m->cfg, st->batch, st->canvas, st->lmax, true);
  if (!workspace || workspace_bytes < L.total || !aligned16(workspace))
    return fail(DG_ERR_WORKSPACE_TOO_SMALL, "dg_denoise_logits: workspace needs %zu bytes",
                L.total);
  Fwd f{m, st->batch, st->canvas, st->cache_len_host, st->lmax, DG_MASK_BIDIR, st->cache_len,
        st->k_cache, st->v_cache, false, true, (char*)workspace, L};
  return run_forward(f, st->tok, logits, (cudaStream_t)stream);
}

int dg_denoise_block(const dg_model* m, dg_state* st, const dg_sampler_cfg* cfg, uint32_t seed,
                     int block, int* steps_taken, void* workspace, size_t workspace_bytes,
                     void* stream) {
  DG_TRY(check_model(m));
  DG_TRY(check_state(st, m->cfg, true));
  if (!cfg || !sampler_cfg_ok(*cfg) || block < 0)
    return fail(DG_ERR_INVALID_ARG, "dg_denoise_block: bad sampler settings or block");
  if (m->cfg.vocab % 4) return fail(DG_ERR_UNSUPPORTED_SHAPE, "vocab must be a multiple of 4");
  if (st->cache_len_host < 0 || st->cache_len_host + st->canvas > st->lmax)
    return fail(DG_ERR_INVALID_ARG, "dg_denoise_block: cache full (%d + %d > %d)",
                st->cache_len_host, st->canvas, st->lmax);
  const FwdLayout L = fwd_layout(m->cfg, st->batch, st->canvas, st->lmax, true);
  if (!workspace || workspace_bytes < L.total || !aligned16(workspace))
    return fail(DG_ERR_WORKSPACE_TOO_SMALL, "dg_denoise_block: workspace needs %zu bytes",
                L.total);
  cudaStream_t s = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  const int B = st->batch, C = st->canvas, V = m->cfg.vocab;
  float* logits = (float*)(ws + L.logits);
  int32_t* running = (int32_t*)(ws + L.flag);

  dg::init_canvas_kernel<<<B, 256, 0, s>>>(B, C, V, seed, block, st->tok, st->committed,
                                            st->prev_argmax, st->seq_status, st->step);
  count_launch();
  DG_CUDA(cudaGetLastError());
  Fwd f{m, B, C, st->cache_len_host, st->lmax, DG_MASK_BIDIR, st->cache_len, st->k_cache,
        st->v_cache, false, true, ws, L};
  const dg::SampleParams sp = make_sample_params(*cfg, seed, block, st->step, 0, B, C, V);
  int steps = 0;
  // with a vocabulary of 256-entry tiles the sampler's row pass runs inside
  // the unembedding and the logits never reach memory
  const bool fused = V % dg::unembed::TILE == 0;
  const bool fp8 = m->unembed_e4m3 != nullptr;  // check_model: vocab % 256 == 0 then
  Fwd fl = f;
  fl.unembed_elsewhere = fused;
  // one denoising step: forward pass, unembedding + sampler, step advance
  auto enqueue_step = [&](cudaStream_t q) -> int {
    DG_TRY(run_forward(fl, st->tok, logits, q));
    if (fused && fp8) {
      // the hidden states quantised per token, then the e4m3 unembedding + sampler
      DG_TRY(quantize_hidden(fl, q));
      const Fp8Scales f8{(const float*)(ws + L.as), m->unembed_scale};
      DG_TRY(launch_unembed_sample(ws + L.aq, m->unembed_e4m3, m->cfg.d, nullptr, 0,
                                   1.f / m->cfg.d, m->cfg.eps, st->tok, st->committed,
                                   st->prev_argmax,
                                   st->seq_status, sp, nullptr, ws + L.spart, q, &f8));
    } else if (fused) {
      DG_TRY(launch_unembed_sample(ws + L.xn, m->unembed, m->cfg.d, nullptr, 0,
                                   1.f / m->cfg.d, m->cfg.eps, st->tok,
                                   st->committed, st->prev_argmax, st->seq_status, sp, nullptr,
                                   ws + L.spart, q));
    } else {
      DG_TRY(launch_sample(logits, st->tok, st->committed, st->prev_argmax, st->seq_status, sp,
                           nullptr, ws + L.spart, q));
    }
    dg::step_advance_kernel<<<1, 256, 0, q>>>(B, cfg->max_steps, st->seq_status, st->step,
                                              running);
    count_launch();
    DG_CUDA(cudaGetLastError());
    return DG_OK;
  };
  // Steps after the first replay one captured graph of the step's launches
  // (the step index lives on the device, so every replay is the next step):
  // the GPU dispatches a graph's kernels with less overhead than stream
  // launches.  Not when the caller's stream is itself being captured.
  StepGraph g;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  DG_CUDA(cudaStreamIsCapturing(s, &cap));
  const bool use_graph = graphs_enabled() && cap == cudaStreamCaptureStatusNone &&
                         cfg->max_steps > 2;
  for (int it = 0; it < cfg->max_steps; ++it) {
    if (use_graph && it == 1) DG_TRY(g.capture(enqueue_step));
    if (g.exec) {
      DG_TRY(g.launch(s));
    } else {
      DG_TRY(enqueue_step(s));
    }
    int32_t host_running = 0;
    DG_CUDA(cudaMemcpyAsync(&host_running, running, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
    DG_CUDA(cudaStreamSynchronize(s));
    steps = it + 1;
    if (!host_running) break;
  }
  // causal re-encode of the final block; each layer's K/V goes to rows
  // [cache_len, cache_len + C), then the length moves on
  Fwd r{m, B, C, st->cache_len_host, st->lmax, DG_MASK_CAUSAL, st->cache_len, st->k_cache,
        st->v_cache, true, false, ws, L};
  DG_TRY(run_forward(r, st->tok, nullptr, s));
  dg::cache_len_bump_kernel<<<1, 256, 0, s>>>(st->cache_len, B, C, st->lmax);
  count_launch();
  DG_CUDA(cudaGetLastError());
  st->cache_len_host += C;
  if (steps_taken) *steps_taken = steps;
  return DG_OK;
}

int dg_philox4x32_10(const uint32_t* in, uint32_t* out, int n, void* stream) {
  if (!in || !out || n < 0) return fail(DG_ERR_INVALID_ARG, "dg_philox4x32_10: bad arguments");
  if (n == 0) return DG_OK;
  dg::philox_kernel<<<cdiv(n, 256), 256, 0, (cudaStream_t)stream>>>(in, out, n);
  count_launch();
  DG_CUDA(cudaGetLastError());
  return DG_OK;
}

int dg_set_wait_limit_ns(uint64_t ns, void* stream) {
  if (ns != 0 && (ns < 1000ull || ns > 600000000000ull))
    return fail(DG_ERR_INVALID_ARG, "dg_set_wait_limit_ns: %llu ns is outside [1 us, 600 s]",
                (unsigned long long)ns);
  const uint64_t v = ns ? ns : dg::kWaitLimitDefaultNs;
  cudaStream_t s = (cudaStream_t)stream;
  DG_CUDA(cudaMemcpyToSymbolAsync(dg::g_wait_limit_ns, &v, sizeof(v), 0, cudaMemcpyHostToDevice,
                                  s));
  DG_CUDA(cudaStreamSynchronize(s));
  return DG_OK;
}

int dg_self_test_wait(int kind, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  if (kind == 0) {
    dg::wait_selftest_kernel<<<1, 32, 0, s>>>();
  } else if (kind == 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(32);
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    DG_CUDA(cudaLaunchKernelEx(&cfg, dg::wait_pair_selftest_kernel));
  } else {
    return fail(DG_ERR_INVALID_ARG, "dg_self_test_wait: kind %d is not 0 or 1", kind);
  }
  count_launch();
  DG_CUDA(cudaGetLastError());
  return DG_OK;
}

}  // extern "C"
