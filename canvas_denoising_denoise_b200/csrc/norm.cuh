// norm.cuh - the RMSNorm of the residual stream, stored as the bf16 input of
// the projection (or unembedding) that consumes it.
//
//   xn[t, :] = bf16(x[t, :] * rs[t]),   rs[t] = 1 / sqrt(mean_k x[t, k]^2 + eps)
//
// with unit gain.  Rounding the normalised row (not the raw one) is what a
// bf16 pipeline stores between the norm and the next product.  One CTA per
// token row; the row's sum of squares is taken in a fixed order (each
// thread's strided partial, the warp's butterfly, then the warps in index
// order), so the bits do not depend on scheduling.
#pragma once

#include "dg_common.cuh"

namespace dg {
namespace norm {

constexpr int NORM_THREADS = 256;

// Sum over the CTA of each thread's partial, in a fixed order (the warp's
// butterfly, then the warps in index order); every thread returns the total.
__device__ __forceinline__ float block_sum(float v, float* s_part) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = v;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < NORM_THREADS / 32; ++w) tot += s_part[w];
  return tot;
}

__device__ __forceinline__ float4 bf16x4_to_float4(uint2 raw) {
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  return make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
}

__device__ __forceinline__ void store_scaled_row(const float4* __restrict__ xr, int n4, float rs,
                                                 __nv_bfloat16* __restrict__ out) {
  uint2* o = reinterpret_cast<uint2*>(out);
  for (int i = threadIdx.x; i < n4; i += NORM_THREADS) {
    const float4 a = xr[i];
    uint2 w;
    w.x = pack_bf16x2(a.x * rs, a.y * rs);
    w.y = pack_bf16x2(a.z * rs, a.w * rs);
    o[i] = w;
  }
}

// x [M, d] fp32 -> xn [M, d] bf16; d % 4 == 0.  Grid: M CTAs.  (Rows wider
// than ROW_MAX_D; the warp-per-row kernel below takes the rest.)
__global__ void __launch_bounds__(NORM_THREADS)
    rmsnorm_kernel(const float* __restrict__ x, int d, float inv_d, float eps,
                   __nv_bfloat16* __restrict__ xn) {
  __shared__ float s_part[NORM_THREADS / 32];
  griddep_launch();
  griddep_wait();
  const size_t row = blockIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(x + row * d);
  const int n4 = d / 4;
  float ss = 0.f;
  for (int i = threadIdx.x; i < n4; i += NORM_THREADS) {
    const float4 a = xr[i];
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
  }
  const float rs = rsqrtf(block_sum(ss, s_part) * inv_d + eps);
  store_scaled_row(xr, n4, rs, xn + row * d);
}

// One warp per row for rows of up to ROW_MAX_D values (d % 128 == 0): the
// row sits in the warp's registers (lane k holds float4 groups k, k + 32, ...),
// so it is read once and reduced with shuffles alone.  The sum of squares is
// each lane's groups in order, then the butterfly: a fixed order.
constexpr int ROW_MAX_D = 4096;
constexpr int ROW_WARPS = 4;  // rows per CTA

template <int G>  // float4 groups per lane: d / 128
__global__ void __launch_bounds__(ROW_WARPS * 32)
    rmsnorm_rows_kernel(const float* __restrict__ x, int M, int d, float inv_d, float eps,
                        __nv_bfloat16* __restrict__ xn) {
  griddep_launch();
  griddep_wait();
  const int row = static_cast<int>(blockIdx.x) * ROW_WARPS + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;  // warp-uniform
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(row) * d);
  float4 v[G];
  float ss = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) v[g] = xr[g * 32 + lane];
#pragma unroll
  for (int g = 0; g < G; ++g) ss += v[g].x * v[g].x + v[g].y * v[g].y + v[g].z * v[g].z + v[g].w * v[g].w;
  const float rs = rsqrtf(warp_sum(ss) * inv_d + eps);
  uint2* o = reinterpret_cast<uint2*>(xn + static_cast<size_t>(row) * d);
#pragma unroll
  for (int g = 0; g < G; ++g)
    o[g * 32 + lane] = make_uint2(pack_bf16x2(v[g].x * rs, v[g].y * rs),
                                  pack_bf16x2(v[g].z * rs, v[g].w * rs));
}

// The embedding lookup and the first norm: x[t] = embed[tok[t]] (fp32, no
// scaling), xn[t] = bf16(RMSNorm(x[t])).  An out-of-range id is recorded in
// the error word and read as id 0.  Grid: M CTAs; d % 4 == 0.
__global__ void __launch_bounds__(NORM_THREADS)
    embed_norm_kernel(const int32_t* __restrict__ tok, const __nv_bfloat16* __restrict__ embed,
                      int V, int d, float inv_d, float eps, float* __restrict__ x,
                      __nv_bfloat16* __restrict__ xn) {
  __shared__ float s_part[NORM_THREADS / 32];
  // the successor (a projection) may launch and fetch its weights now; it
  // reads xn only after its own wait, which covers this kernel's completion
  griddep_launch();
  griddep_wait();
  const int t = blockIdx.x;
  int id = tok[t];
  if (id < 0 || id >= V) {
    if (threadIdx.x == 0) raise_error(ERR_CHECK | 0x201, static_cast<uint32_t>(t));
    id = 0;
  }
  const uint2* e = reinterpret_cast<const uint2*>(embed + static_cast<size_t>(id) * d);
  float4* xr = reinterpret_cast<float4*>(x + static_cast<size_t>(t) * d);
  const int n4 = d / 4;
  float ss = 0.f;
  for (int i = threadIdx.x; i < n4; i += NORM_THREADS) {
    const float4 a = bf16x4_to_float4(e[i]);
    xr[i] = a;
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
  }
  const float rs = rsqrtf(block_sum(ss, s_part) * inv_d + eps);
  uint2* o = reinterpret_cast<uint2*>(xn + static_cast<size_t>(t) * d);
  for (int i = threadIdx.x; i < n4; i += NORM_THREADS) {
    const float4 a = bf16x4_to_float4(e[i]);  // the embedding row again, not x
    uint2 w;
    w.x = pack_bf16x2(a.x * rs, a.y * rs);
    w.y = pack_bf16x2(a.z * rs, a.w * rs);
    o[i] = w;
  }
}

}  // namespace norm
}  // namespace dg
