// quant.cuh - e4m3 quantisation of bf16 matrices for the FP8 unembedding.
//
// Per row r (activations): s_r = max_k |x[r, k]| / 448, q = e4m3(x / s_r).
// Per tensor (weights): one s = max |x| / 448 for the whole matrix.
// 448 is the largest finite e4m3 value; the conversion rounds to the nearest
// value (ties to even) and saturates; an all-zero row or tensor takes s = 1.
// The divisions are IEEE fp32 (correctly rounded), so the scales and the codes
// are reproducible bit for bit.
#pragma once

#include <cuda_fp8.h>

#include "dg_common.cuh"

namespace dg {
namespace quant {

constexpr int THREADS = 256;

__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float scale_of(float amax) {
  return amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
}

// One CTA per row; cols a multiple of 8.  A thread holds up to REG_CHUNKS
// 8-element chunks of its row in registers (rows of up to 8192 bf16 are read
// once); longer rows are read again for the codes.
constexpr int REG_CHUNKS = 4;

__global__ void __launch_bounds__(THREADS) quantize_rows_kernel(
    const __nv_bfloat16* __restrict__ in, int rows, int cols, uint8_t* __restrict__ out,
    float* __restrict__ scales) {
  griddep_wait();
  griddep_launch();
  __shared__ float red[THREADS / 32];
  const int row = blockIdx.x;
  if (row >= rows) return;
  const size_t base = static_cast<size_t>(row) * cols;
  uint4 keep[REG_CHUNKS];
  float amax = 0.f;
  for (int i = 0, c = threadIdx.x * 8; c < cols; ++i, c += THREADS * 8) {
    const uint4 raw = *reinterpret_cast<const uint4*>(in + base + c);
    if (i < REG_CHUNKS) keep[i] = raw;
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      amax = fmaxf(amax, fabsf(__low2float(h[e])));
      amax = fmaxf(amax, fabsf(__high2float(h[e])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  float a = red[0];
#pragma unroll
  for (int w = 1; w < THREADS / 32; ++w) a = fmaxf(a, red[w]);
  const float s = scale_of(a);
  if (threadIdx.x == 0) scales[row] = s;
  for (int i = 0, c = threadIdx.x * 8; c < cols; ++i, c += THREADS * 8) {
    const uint4 raw = i < REG_CHUNKS ? keep[i] : *reinterpret_cast<const uint4*>(in + base + c);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = to_e4m3(__fdiv_rn(__low2float(h[e]), s));
      const uint32_t hi = to_e4m3(__fdiv_rn(__high2float(h[e]), s));
      w[e >> 1] |= (lo | (hi << 8)) << ((e & 1) * 16);
    }
    *reinterpret_cast<uint2*>(out + base + c) = make_uint2(w[0], w[1]);
  }
}

// max |x| of n values into *amax_bits (as the bits of a non-negative float,
// which order like unsigned integers); *amax_bits must start at 0.
__global__ void __launch_bounds__(THREADS) absmax_kernel(const __nv_bfloat16* __restrict__ in,
                                                         size_t n, unsigned int* amax_bits) {
  float amax = 0.f;
  for (size_t i = (static_cast<size_t>(blockIdx.x) * THREADS + threadIdx.x) * 8; i < n;
       i += static_cast<size_t>(gridDim.x) * THREADS * 8) {
    const uint4 raw = *reinterpret_cast<const uint4*>(in + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      amax = fmaxf(amax, fabsf(__low2float(h[e])));
      amax = fmaxf(amax, fabsf(__high2float(h[e])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(amax));
}

// The codes, with the scale taken from the amax bits absmax_kernel left.
__global__ void __launch_bounds__(THREADS) quantize_tensor_kernel(
    const __nv_bfloat16* __restrict__ in, size_t n, uint8_t* __restrict__ out,
    const unsigned int* __restrict__ amax_bits) {
  const float s = scale_of(__uint_as_float(*amax_bits));
  for (size_t i = (static_cast<size_t>(blockIdx.x) * THREADS + threadIdx.x) * 8; i < n;
       i += static_cast<size_t>(gridDim.x) * THREADS * 8) {
    const uint4 raw = *reinterpret_cast<const uint4*>(in + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = to_e4m3(__fdiv_rn(__low2float(h[e]), s));
      const uint32_t hi = to_e4m3(__fdiv_rn(__high2float(h[e]), s));
      w[e >> 1] |= (lo | (hi << 8)) << ((e & 1) * 16);
    }
    *reinterpret_cast<uint2*>(out + i) = make_uint2(w[0], w[1]);
  }
}

// amax bits -> scale, in place (one thread).
__global__ void amax_to_scale_kernel(unsigned int* amax_bits_then_scale) {
  const float s = scale_of(__uint_as_float(*amax_bits_then_scale));
  *reinterpret_cast<float*>(amax_bits_then_scale) = s;
}

}  // namespace quant
}  // namespace dg
