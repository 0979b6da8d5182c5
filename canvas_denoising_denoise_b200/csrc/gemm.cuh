// gemm.cuh - the projections of the stack and the unembedding on tcgen05.
//
//   y[t, f] = rs[t] * sum_k x[t, k] w[f, k]     x bf16 [M, K] (activations)
//                                               w bf16 [N, K] (weights, [out, in])
//
// The weight is the UMMA A operand (128 output features per tile) and the
// tokens are the B operand (up to 256 per tile): one 128 x 256 x 16
// tcgen05.mma per k-step, fp32 accumulator in TMEM, a 4-stage TMA ring.
//
// When there are too few output tiles to occupy the SMs (the layer
// projections of one 256-token canvas), K is split over S CTAs that form one
// thread-block cluster.  Each CTA stages its partial tile in its own shared
// memory; after a cluster barrier, CTA r sums token rows [r*256/S, (r+1)*256/S)
// of all S partials through distributed shared memory and applies the
// epilogue.  Partial sums never leave the cluster.
//
// The epilogue can scale each token's row by rs[t] = 1/sqrt(mean_k x[t,k]^2 +
// eps), computed from per-column-group sums of squares of the input (a
// standalone use of dg_linear with row scales; the model's forward pass feeds
// the projections rows that are already normalised, see norm.cuh).

// With e4m3 operands (F8: x and w as codes, x scaled per token by sx[t], w
// per tensor by sw) the MMA is kind::f8f6f4 and every epilogue takes acc as
// sx[t] * sw * (sum of code products): a k-block is 128 codes, still one
// 128-byte swizzle row.
//
// Epilogues:
//   EPI_F32    out_f32[t, f]  = rs * acc
//   EPI_BF16   out_bf16[t, f] = bf16(rs * acc)
//   EPI_GELU   out_bf16[t, f] = bf16(gelu(rs * acc))            (exact erf)
//   EPI_RESID  x[t, f] += acc; out_bf16[t, f] = bf16(x[t, f]) (if given);
//              ssq_out[tile, t] = sum over the tile's 128 f of x[t, f]^2 (if given)
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and one
// lane issues the MMAs, warps 2..5 move the accumulator TMEM -> shared
// memory; all six warps run the reduction/epilogue.
#pragma once

#include "dg_common.cuh"

namespace dg {
namespace gemm {

constexpr int BM = 128;  // output features per tile (UMMA M)
constexpr int BK = 64;   // K per stage: one 128-byte swizzle row of bf16
constexpr int A_BYTES = BM * BK * 2;
constexpr int THREADS = 192;
constexpr int WARPS = THREADS / 32;
constexpr int TILE_ROW_FLOATS = BM;                       // staged tile: [BN][BM] fp32
constexpr int MAX_SPLITS = 8;

// Shared memory of one CTA with a TMA stage ring of RING_KB kilobytes (the
// ring also holds the fp32 tile after the mainloop), the row scales and the
// barriers.  With a 96 KB ring two CTAs share an SM: each CTA's producer ->
// MMA pipeline has a fixed round trip per stage, so two pipelines per SM move
// more bytes than one pipeline with twice the stages.
constexpr int smem_bytes(int ring_kb) { return 1024 + ring_kb * 1024 + 256 * 4 + 256; }

// BN: tokens per tile (UMMA N), 64, 128 or 256.  A stage holds KPS k-blocks
// (the k-blocks' A tiles, then their B tiles): each stage costs a fixed share
// of the pipeline's round trip whatever its size, so with a 192 KB ring at
// BN = 128 two k-blocks per stage (3 stages of 64 KB) stream faster than one
// (6 stages of 32 KB).
template <int BN, int RING_KB>
struct TileCfg {
  static constexpr int RING_BYTES = RING_KB * 1024;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int KPS = (BN <= 128 && RING_KB >= 192) ? 2 : 1;
  static constexpr int STAGE_BYTES = KPS * (A_BYTES + B_BYTES);
  static constexpr int STAGES = RING_BYTES / STAGE_BYTES;
  static constexpr int TMEM_COLS = BN;
  static constexpr int MIN_CTAS = RING_KB <= 96 ? 2 : 1;  // CTAs per SM
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, false, false);
  static_assert(BN == 64 || BN == 128 || BN == 256, "token tile");
  static_assert(STAGES >= 2, "at least two stages");
  static_assert(BN * BM * 4 <= RING_BYTES, "staged tile must fit in the stage ring");
};

enum Epi : int { EPI_F32 = 0, EPI_BF16 = 1, EPI_GELU = 2, EPI_RESID = 3 };

struct Params {
  int M, N, K;
  int kb_per_split;        // k-blocks (128-byte rows: 64 bf16 or 128 e4m3) per split
  int splits;              // cluster size along z (1 = no cluster)
  int epi;
  float* out_f32;          // EPI_F32
  __nv_bfloat16* out_bf16; // EPI_BF16 / EPI_GELU / EPI_RESID (optional there)
  float* x;                // EPI_RESID residual stream [M, N] fp32, updated in place
  const float* ssq_in;     // [n_ssq_in, M] sums of squares of the input rows, or null
  int n_ssq_in;
  float inv_k;             // 1 / (input width) for the mean
  float eps;
  float* ssq_out;          // [N / 128, M] (EPI_RESID), or null
  const float* tok_scale;  // F8: [M] per-token scale of x
  const float* w_scale;    // F8: per-tensor scale of w (device scalar)
  unsigned long long* trace;  // optional [grid, 8] %globaltimer stamps of the phases
};

__device__ __forceinline__ void trace_stamp(const Params& p, int slot) {
  if (p.trace) {
    const size_t cta = (static_cast<size_t>(blockIdx.z) * gridDim.y + blockIdx.y) * gridDim.x +
                       blockIdx.x;
    p.trace[cta * 8 + slot] = globaltimer_ns();
  }
}

// erfc(a), a >= 0, by Abramowitz & Stegun, Handbook of Mathematical
// Functions, 7.1.26:
//   erfc(a) = t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-a^2),  t = 1 / (1 + p a),
// absolute error <= 1.5e-7.  One reciprocal and one exp2 on the special
// function unit plus a handful of FMAs.
__device__ __forceinline__ float erfc_pos_as7126(float a) {
  float t;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(0.3275911f, a, 1.0f)));
  float poly = fmaf(t, 1.061405429f, -1.453152027f);
  poly = fmaf(t, poly, 1.421413741f);
  poly = fmaf(t, poly, -0.284496736f);
  poly = fmaf(t, poly, 0.254829592f);
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-a * a * 1.4426950408889634f));
  return t * poly * e;
}

// GELU with the exact-erf definition, x * (1 + erf(x / sqrt 2)) / 2, where
// 1 + erf(z) = 2 - erfc(z) for z >= 0 and erfc(-z) for z < 0 (no cancellation).
// The absolute error (< 2e-7 |x|) is far below the bf16 step of the output.
__device__ __forceinline__ float gelu_erf(float x) {
  const float z = x * 0.70710678118654752f;
  const float q = erfc_pos_as7126(fabsf(z));
  return 0.5f * x * (z >= 0.f ? 2.0f - q : q);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// Remote shared-memory load.  Ordering against the peers' writes comes from
// the cluster barrier, so no compiler memory clobber is needed here and
// several loads can be in flight at once.
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

template <int S, int BN, bool F8 = false, int RING_KB = 192>
__global__ void __launch_bounds__(THREADS, TileCfg<BN, RING_KB>::MIN_CTAS)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                Params p) {
  static_assert(S == 1 || S == 2 || S == 4 || S == 8, "split count");
  using TC = TileCfg<BN, RING_KB>;
  constexpr int RING_BYTES = TC::RING_BYTES;
  constexpr int STAGES = TC::STAGES;
  constexpr int STAGE_BYTES = TC::STAGE_BYTES;
  constexpr int TMEM_COLS = TC::TMEM_COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* tile = reinterpret_cast<float*>(smem);  // [BN][BM] after the mainloop
  float* rowscale = reinterpret_cast<float*>(smem + RING_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + RING_BYTES + 256 * 4);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  // token tile fastest: the CTAs that share a weight tile start together, so
  // the second reader finds it in L2
  const int t0 = blockIdx.x * BN;
  const int f0 = blockIdx.y * BM;
  const int split = blockIdx.z;
  const int kb_begin = split * p.kb_per_split;
  constexpr int KB_ELEMS = F8 ? 128 : BK;  // elements per 128-byte k-block row
  const int nkb = min(p.kb_per_split, p.K / KB_ELEMS - kb_begin);

  if (threadIdx.x == 0) {
    trace_stamp(p, 0);
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
  if (threadIdx.x == 0) trace_stamp(p, 1);

  griddep_launch();
  constexpr int KPS = TC::KPS;
  const int nst = (nkb + KPS - 1) / KPS;  // stages of this split
  // k-blocks in stage q (the last one may be short)
  auto stage_kbs = [&](int q) { return min(KPS, nkb - q * KPS); };
  if (warp == 0) {
    if (lane == 0 && nkb > 0) {
      // weights are streamed once: evict them first unless another token tile
      // of this launch reads the same weight tile
      const uint64_t pol_w = gridDim.x > 1 ? l2_policy_evict_normal() : l2_policy_evict_first();
      auto load_w = [&](int q) {
        uint8_t* a = smem + (q % STAGES) * STAGE_BYTES;
        for (int j = 0; j < stage_kbs(q); ++j)
          tma_load_2d_hint(a + j * A_BYTES, &tm_w, &full[q % STAGES],
                           (kb_begin + q * KPS + j) * KB_ELEMS, f0, pol_w);
      };
      auto load_x = [&](int q) {
        uint8_t* b = smem + (q % STAGES) * STAGE_BYTES + KPS * A_BYTES;
        for (int j = 0; j < stage_kbs(q); ++j)
          tma_load_2d(b + j * TC::B_BYTES, &tm_x, &full[q % STAGES],
                      (kb_begin + q * KPS + j) * KB_ELEMS,
                      t0);
      };
      // the weights are never written by another kernel: the first stages'
      // weight tiles are requested before waiting on the predecessor
      const int pre = min(STAGES, nst);
      for (int q = 0; q < pre; ++q) {
        mbar_expect_tx(&full[q], stage_kbs(q) * (A_BYTES + TC::B_BYTES));
        load_w(q);
      }
      griddep_wait();
      for (int q = 0; q < pre; ++q) load_x(q);
      int issued = pre;
      for (int q = pre; q < nst; ++q) {
        const int st = q % STAGES;
        if (!mbar_wait(&empty[st], ((q / STAGES) - 1) & 1, abort_flag, 0x101)) break;
        mbar_expect_tx(&full[st], stage_kbs(q) * (A_BYTES + TC::B_BYTES));
        load_w(q);
        load_x(q);
        issued = q + 1;
      }
      if (*abort_flag) {
        for (int q = max(0, issued - STAGES); q < issued; ++q)
          mbar_wait(&full[q % STAGES], (q / STAGES) & 1, nullptr, 0x102);
      }
    } else {
      griddep_wait();
    }
  } else if (warp == 1) {
    griddep_wait();
    if (lane == 0 && nkb > 0) {
      for (int q = 0; q < nst; ++q) {
        const int st = q % STAGES;
        if (!mbar_wait(&full[st], (q / STAGES) & 1, abort_flag, 0x103)) break;
        if (q == 0) trace_stamp(p, 2);
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + st * STAGE_BYTES);
        const uint32_t b_base = a_base + KPS * A_BYTES;
        for (int j = 0; j < stage_kbs(q); ++j) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // four 32-byte K steps per 128-byte row
            const uint64_t ad = sdesc_sw128(a_base + j * A_BYTES + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b_base + j * TC::B_BYTES + kk * 32, 16, 1024);
            if constexpr (F8)
              umma_ss_f8(tmem_acc, ad, bd, idesc_e4m3_f32(BM, BN), (q | j | kk) != 0 ? 1u : 0u);
            else
              umma_ss(tmem_acc, ad, bd, TC::IDESC, (q | j | kk) != 0 ? 1u : 0u);
          }
        }
        umma_commit(&empty[st]);
      }
      trace_stamp(p, 3);
      umma_commit(acc_full);
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, 0x104);
    }
  } else {
    griddep_wait();
    // warps 2..5: row scales for this tile's tokens while the mainloop runs
    for (int t = threadIdx.x - 64; t < BN; t += THREADS - 64) {
      float rs = 1.f;
      const int tg = t0 + t;
      if (p.ssq_in != nullptr && tg < p.M) {
        // index order, sixteen loads in flight (as the pair pipelines)
        float acc = 0.f;
        for (int j0 = 0; j0 < p.n_ssq_in; j0 += 16) {
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            v[j] = j0 + j < p.n_ssq_in ? p.ssq_in[static_cast<size_t>(j0 + j) * p.M + tg] : 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j) acc += v[j];
        }
        rs = rsqrtf(acc * p.inv_k + p.eps);
      }
      if constexpr (F8) {
        if (tg < p.M) rs *= p.tok_scale[tg] * *p.w_scale;
      }
      rowscale[t] = rs;
    }
    // TMEM -> registers -> shared tile [token][feature]
    const bool have_acc =
        nkb > 0 && __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, 0x105));
    if (have_acc) {
      if (threadIdx.x == 64) trace_stamp(p, 4);
      tc_fence_after();
      const int quarter = warp & 3;
      const int fl = quarter * 32 + lane;
      const uint32_t taddr = tmem_acc + (static_cast<uint32_t>(quarter * 32) << 16);
      for (int c = 0; c < BN / 32; c += 2) {
        if (t0 + c * 32 >= p.M) break;  // warp-uniform
        uint32_t r0[32], r1[32];
        tmem_ld32(taddr + c * 32, r0);
        tmem_ld32(taddr + c * 32 + 32, r1);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          tile[(c * 32 + j) * TILE_ROW_FLOATS + fl] = __uint_as_float(r0[j]);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          tile[(c * 32 + 32 + j) * TILE_ROW_FLOATS + fl] = __uint_as_float(r1[j]);
      }
    } else {
      // no accumulator (empty split or an abandoned wait): contribute zeros
      for (int i = threadIdx.x - 64; i < BN * TILE_ROW_FLOATS; i += THREADS - 64) tile[i] = 0.f;
    }
  }
  // every CTA of the cluster has its partial tile in shared memory
  tc_fence_before();
  if constexpr (S > 1)
    cluster_sync();
  else
    __syncthreads();
  if (threadIdx.x == 0) trace_stamp(p, 5);

  // ---------------------------------------------------------------- reduce + epilogue
  // CTA r owns token rows [r*BN/S, (r+1)*BN/S) of the tile.  A warp gathers
  // MAX_SPLITS float4 per lane per round (S sources x MAX_SPLITS/S rows) so
  // that the remote loads overlap instead of queueing one by one.
  constexpr int rows_per = BN / S;
  constexpr int rows_round = MAX_SPLITS / S;
  const int r0 = (S > 1 ? static_cast<int>(cluster_rank()) : 0) * rows_per;
  const uint32_t tile_saddr = smem_u32(tile);
  for (int rb = warp * rows_round; rb < rows_per; rb += WARPS * rows_round) {
    float4 v[MAX_SPLITS];
#pragma unroll
    for (int i = 0; i < MAX_SPLITS; ++i) {
      const int t = r0 + rb + i / S;
      const uint32_t off = static_cast<uint32_t>((t * TILE_ROW_FLOATS + lane * 4) * 4);
      if (rb + i / S < rows_per && t0 + t < p.M) {
        if constexpr (S > 1)
          v[i] = ld_dsmem_f4(map_to_rank(tile_saddr + off, i % S));
        else
          v[i] = *reinterpret_cast<const float4*>(reinterpret_cast<const uint8_t*>(tile) + off);
      } else {
        v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int j = 0; j < rows_round; ++j) {
      const int t = r0 + rb + j;
      const int tg = t0 + t;
      if (rb + j >= rows_per || tg >= p.M) break;  // warp-uniform
      float4 a = v[j * S];
#pragma unroll
      for (int q = 1; q < S; ++q) {
        const float4 w = v[j * S + q];
        a.x += w.x; a.y += w.y; a.z += w.z; a.w += w.w;
      }
      const int f = f0 + lane * 4;
      const size_t o = static_cast<size_t>(tg) * p.N + f;
      if (p.epi == EPI_RESID) {
        if constexpr (F8) {
          const float sc = rowscale[t];
          a.x *= sc; a.y *= sc; a.z *= sc; a.w *= sc;
        }
        float4* xp = reinterpret_cast<float4*>(p.x + o);
        float4 xv = *xp;
        xv.x += a.x; xv.y += a.y; xv.z += a.z; xv.w += a.w;
        *xp = xv;
        if (p.out_bf16) {
          uint2 w;
          w.x = pack_bf16x2(xv.x, xv.y);
          w.y = pack_bf16x2(xv.z, xv.w);
          *reinterpret_cast<uint2*>(p.out_bf16 + o) = w;
        }
        if (p.ssq_out) {
          const float sq = warp_sum(xv.x * xv.x + xv.y * xv.y + xv.z * xv.z + xv.w * xv.w);
          if (lane == 0) p.ssq_out[static_cast<size_t>(blockIdx.y) * p.M + tg] = sq;
        }
      } else {
        const float rs = rowscale[t];
        a.x *= rs; a.y *= rs; a.z *= rs; a.w *= rs;
        if (p.epi == EPI_F32) {
          *reinterpret_cast<float4*>(p.out_f32 + o) = a;
        } else {
          if (p.epi == EPI_GELU) {
            a.x = gelu_erf(a.x); a.y = gelu_erf(a.y); a.z = gelu_erf(a.z); a.w = gelu_erf(a.w);
          }
          uint2 w;
          w.x = pack_bf16x2(a.x, a.y);
          w.y = pack_bf16x2(a.z, a.w);
          *reinterpret_cast<uint2*>(p.out_bf16 + o) = w;
        }
      }
    }
  }
  if (threadIdx.x == 0) trace_stamp(p, 6);
  // no CTA leaves while a peer may still read its shared memory
  if constexpr (S > 1) cluster_sync();
  __syncthreads();
  if (threadIdx.x == 0) trace_stamp(p, 7);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, TMEM_COLS);
  }
}

}  // namespace gemm
}  // namespace dg
