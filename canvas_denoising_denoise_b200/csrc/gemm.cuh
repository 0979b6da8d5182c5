// gemm.cuh - the projections of the stack and the unembedding on tcgen05.
//
//   y[t, f] = sum_k x[t, k] w[f, k]        x bf16 [M, K] (activations)
//                                          w bf16 [N, K] (weights, nn.Linear layout)
//
// The weight is the UMMA A operand (M side, 128 output features per tile) and
// the activations are the B operand (N side, up to 256 tokens per tile): one
// 128 x 256 x 16 instruction per k-step, the accumulator in TMEM.  At the
// canvas sizes (256 tokens per sequence) each weight tile is streamed from
// HBM exactly once and the activations come from L2.  Few output tiles at
// small widths are spread over the SMs by splitting K; the split partial sums
// (fp32) are reduced in a fixed order by a separate kernel that also applies
// the epilogue (bf16 store, GELU, residual add, residual add + RMSNorm).
//
// Warp roles (192 threads): warp 0 issues TMA loads into a ring of stages,
// warp 1 owns TMEM and one elected lane issues the MMAs, warps 2..5 drain
// the accumulator (TMEM -> registers -> global).
#pragma once

#include "dg_common.cuh"

namespace dg {
namespace gemm {

constexpr int BM = 128;  // output features per tile (UMMA M)
constexpr int BN = 256;  // tokens per tile (UMMA N)
constexpr int BK = 64;   // K per stage: one 128-byte swizzle row of bf16
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int STAGES = 4;
constexpr int THREADS = 192;
constexpr int TMEM_COLS = BN;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, false, false);

enum Epi : int {
  EPI_STORE_F32 = 0,   // out_f32[(split * M + t) * N + f] = acc
  EPI_BF16 = 1,        // out_bf16[t * N + f] = acc
  EPI_GELU_BF16 = 2,   // out_bf16[t * N + f] = gelu(acc)
  EPI_ADD_F32 = 3,     // out_f32[t * N + f] += acc
};

struct Params {
  int M, N, K;
  int kb_per_split;  // k-blocks (of 64) per split
  int epi;
  float* out_f32;
  __nv_bfloat16* out_bf16;
};

__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  const int f0 = blockIdx.x * BM;
  const int t0 = blockIdx.y * BN;
  const int split = blockIdx.z;
  const int kb_total = p.K / BK;
  const int kb_begin = split * p.kb_per_split;
  const int nkb = min(p.kb_per_split, kb_total - kb_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_holder;

  if (nkb > 0) {
    if (warp == 0) {
      if (lane == 0) {
        const uint64_t pol_w = l2_policy_evict_first();
        int issued = 0;
        for (int kb = 0; kb < nkb; ++kb) {
          const int st = kb % STAGES;
          if (kb >= STAGES &&
              !mbar_wait(&empty[st], ((kb / STAGES) - 1) & 1, abort_flag, 0x101))
            break;
          uint8_t* a = smem + st * STAGE_BYTES;
          uint8_t* bt = a + A_BYTES;
          mbar_expect_tx(&full[st], STAGE_BYTES);
          const int kx = (kb_begin + kb) * BK;
          tma_load_2d_hint(a, &tm_w, &full[st], kx, f0, pol_w);
          tma_load_2d(bt, &tm_x, &full[st], kx, t0);
          issued = kb + 1;
        }
        if (*abort_flag) {
          // let every load already in flight land before the CTA exits
          for (int kb = max(0, issued - STAGES); kb < issued; ++kb)
            mbar_wait(&full[kb % STAGES], (kb / STAGES) & 1, nullptr, 0x102);
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        for (int kb = 0; kb < nkb; ++kb) {
          const int st = kb % STAGES;
          if (!mbar_wait(&full[st], (kb / STAGES) & 1, abort_flag, 0x103)) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + st * STAGE_BYTES);
          const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(a_base + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b_base + kk * 32, 16, 1024);
            umma_ss(tmem_acc, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[st]);
        }
        umma_commit(acc_full);
        // all MMAs of this CTA retire before TMEM is released
        umma_commit(drain);
        mbar_wait(drain, 0, nullptr, 0x104);
      }
    } else {
      // epilogue warps 2..5 -> TMEM lane quarter (warp % 4)
      const int quarter = warp & 3;
      const int f = f0 + quarter * 32 + lane;
      if (__all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, 0x105))) {
        tc_fence_after();
        const uint32_t taddr = tmem_acc + (static_cast<uint32_t>(quarter * 32) << 16);
        for (int c = 0; c < BN / 32; ++c) {
          const int tb = t0 + c * 32;
          if (tb >= p.M) break;
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          const int nt = min(32, p.M - tb);
          if (p.epi == EPI_STORE_F32) {
            float* o = p.out_f32 + (static_cast<size_t>(split) * p.M + tb) * p.N + f;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nt) o[static_cast<size_t>(j) * p.N] = __uint_as_float(r[j]);
          } else if (p.epi == EPI_ADD_F32) {
            float* o = p.out_f32 + static_cast<size_t>(tb) * p.N + f;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nt) o[static_cast<size_t>(j) * p.N] += __uint_as_float(r[j]);
          } else if (p.epi == EPI_BF16) {
            __nv_bfloat16* o = p.out_bf16 + static_cast<size_t>(tb) * p.N + f;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nt) o[static_cast<size_t>(j) * p.N] = __float2bfloat16_rn(__uint_as_float(r[j]));
          } else {
            __nv_bfloat16* o = p.out_bf16 + static_cast<size_t>(tb) * p.N + f;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nt)
                o[static_cast<size_t>(j) * p.N] =
                    __float2bfloat16_rn(gelu_erf(__uint_as_float(r[j])));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Split-K reductions with the layer epilogues.  part: [S, M, N] fp32.
// ---------------------------------------------------------------------------
enum RedMode : int { RED_BF16 = 0, RED_GELU_BF16 = 1, RED_ADD_F32 = 2 };

__global__ void reduce_kernel(const float* __restrict__ part, int S, int M, int N, int mode,
                              __nv_bfloat16* __restrict__ out_bf16, float* __restrict__ out_f32) {
  const size_t n4 = static_cast<size_t>(M) * N / 4;
  const size_t stride = static_cast<size_t>(M) * N;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float4 a = reinterpret_cast<const float4*>(part)[i];
    for (int s = 1; s < S; ++s) {
      const float4 c = reinterpret_cast<const float4*>(part + s * stride)[i];
      a.x += c.x; a.y += c.y; a.z += c.z; a.w += c.w;
    }
    if (mode == RED_ADD_F32) {
      float4 o = reinterpret_cast<float4*>(out_f32)[i];
      o.x += a.x; o.y += a.y; o.z += a.z; o.w += a.w;
      reinterpret_cast<float4*>(out_f32)[i] = o;
    } else {
      if (mode == RED_GELU_BF16) {
        a.x = gelu_erf(a.x); a.y = gelu_erf(a.y); a.z = gelu_erf(a.z); a.w = gelu_erf(a.w);
      }
      uint2 v;
      v.x = pack_bf16x2(a.x, a.y);
      v.y = pack_bf16x2(a.z, a.w);
      reinterpret_cast<uint2*>(out_bf16)[i] = v;
    }
  }
}

// One CTA per token row: x[t] (+)= sum_s part[s][t], then xn[t] = bf16(x[t] / rms(x[t])).
// With S == 0 only the normalisation runs.
constexpr int NORM_THREADS = 256;

__global__ void __launch_bounds__(NORM_THREADS) add_norm_kernel(
    const float* __restrict__ part, int S, int M, int N, float eps, float* __restrict__ x,
    __nv_bfloat16* __restrict__ xn) {
  const int t = blockIdx.x;
  const size_t stride = static_cast<size_t>(M) * N;
  float* xr = x + static_cast<size_t>(t) * N;
  float ss = 0.f;
  for (int c = threadIdx.x * 4; c < N; c += NORM_THREADS * 4) {
    float4 a = *reinterpret_cast<float4*>(xr + c);
    for (int s = 0; s < S; ++s) {
      const float4 d = *reinterpret_cast<const float4*>(part + s * stride +
                                                        static_cast<size_t>(t) * N + c);
      a.x += d.x; a.y += d.y; a.z += d.z; a.w += d.w;
    }
    if (S > 0) *reinterpret_cast<float4*>(xr + c) = a;
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
  }
  __shared__ float red[NORM_THREADS / 32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < NORM_THREADS / 32; ++w) tot += red[w];
  const float inv = rsqrtf(tot / static_cast<float>(N) + eps);
  __nv_bfloat16* xo = xn + static_cast<size_t>(t) * N;
  for (int c = threadIdx.x * 4; c < N; c += NORM_THREADS * 4) {
    const float4 a = *reinterpret_cast<const float4*>(xr + c);
    uint2 v;
    v.x = pack_bf16x2(a.x * inv, a.y * inv);
    v.y = pack_bf16x2(a.z * inv, a.w * inv);
    *reinterpret_cast<uint2*>(xo + c) = v;
  }
}

// One CTA per token row: x[t] = embed[tok[t]] (fp32), xn[t] = bf16(rmsnorm(x[t])).
__global__ void __launch_bounds__(NORM_THREADS) embed_norm_kernel(
    const int32_t* __restrict__ tok, const __nv_bfloat16* __restrict__ embed, int V, int d,
    float eps, float* __restrict__ x, __nv_bfloat16* __restrict__ xn) {
  const int t = blockIdx.x;
  int id = tok[t];
  if (id < 0 || id >= V) {
    raise_error(ERR_CHECK | 0x201, static_cast<uint32_t>(t));
    id = 0;
  }
  const __nv_bfloat16* e = embed + static_cast<size_t>(id) * d;
  float* xr = x + static_cast<size_t>(t) * d;
  float ss = 0.f;
  for (int c = threadIdx.x * 4; c < d; c += NORM_THREADS * 4) {
    const uint2 raw = *reinterpret_cast<const uint2*>(e + c);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
    const float4 a = make_float4(__low2float(lo), __high2float(lo), __low2float(hi),
                                 __high2float(hi));
    *reinterpret_cast<float4*>(xr + c) = a;
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
  }
  __shared__ float red[NORM_THREADS / 32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < NORM_THREADS / 32; ++w) tot += red[w];
  const float inv = rsqrtf(tot / static_cast<float>(d) + eps);
  __nv_bfloat16* xo = xn + static_cast<size_t>(t) * d;
  for (int c = threadIdx.x * 4; c < d; c += NORM_THREADS * 4) {
    const float4 a = *reinterpret_cast<const float4*>(xr + c);
    uint2 v;
    v.x = pack_bf16x2(a.x * inv, a.y * inv);
    v.y = pack_bf16x2(a.z * inv, a.w * inv);
    *reinterpret_cast<uint2*>(xo + c) = v;
  }
}

}  // namespace gemm
}  // namespace dg
