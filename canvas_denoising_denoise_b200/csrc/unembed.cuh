// unembed.cuh - the unembedding on CTA pairs:
//
//   logits[t, v] = rs[t] * sum_k h[t, k] W_U[v, k]     h bf16 [M, K], W_U bf16 [V, K]
//
// with rs[t] = 1/sqrt(mean_k x[t,k]^2 + eps) the final RMSNorm (unit gain)
// folded in as a per-token scale, from per-(128-column tile, token) sums of
// squares of the residual stream.
//
// The vocabulary is far larger than the 148 SMs, so one persistent grid of
// CTA pairs walks 256 (vocabulary) x 256 (token) output tiles.  A pair tile is
// one cta_group::2 MMA chain: each CTA stages 128 vocabulary rows of W_U and
// 128 tokens of h per k-block, and the pair's MMA (M = 256, N = 256, issued by
// the even CTA) reads both CTAs' halves.  Compared with one CTA per 128 x 256
// tile this halves the activation bytes every SM pulls in per weight byte:
// with 256 tokens the activation tile is as large as the weight tile, so the
// single-CTA form moves three bytes through each SM per weight byte and the
// pair form two.
//
// The accumulator is double-buffered in TMEM (2 x 256 columns), so the store
// of tile i (fp32 logits straight from registers, 128 contiguous bytes per
// warp store) overlaps the MMAs of tile i + 1.
//
// Roles, 192 threads per CTA: warp 0 issues the TMA loads (both CTAs, each
// into its own ring, completion counted on the even CTA's barrier); warp 1
// owns TMEM and, in the even CTA, one lane issues the MMAs; warps 2..5 read
// this CTA's 128 accumulator rows (vocabulary entries) and store the logits.
#pragma once

#include "dg_common.cuh"

namespace dg {
namespace unembed {

constexpr int TILE_V = 256;               // vocabulary rows per pair tile (MMA M)
constexpr int HALF_V = TILE_V / 2;        // ... per CTA
constexpr int TILE_T = 256;               // tokens per pair tile (MMA N)
constexpr int HALF_T = TILE_T / 2;        // ... per CTA
constexpr int BK = 64;                    // one 128-byte swizzle row of bf16
constexpr int A_BYTES = HALF_V * BK * 2;  // 16 KB
constexpr int B_BYTES = HALF_T * BK * 2;  // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int STAGES = 6;
constexpr int RING_BYTES = STAGES * STAGE_BYTES;  // 192 KB
constexpr int ACC_COLS = TILE_T;                  // fp32 columns per accumulator buffer
constexpr int TMEM_COLS = 2 * ACC_COLS;           // two buffers: all 512 columns
constexpr int THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr int SMEM_BYTES = 1024 + RING_BYTES + 256;
constexpr uint32_t IDESC = idesc_bf16_f32(TILE_V, TILE_T, false, false);

struct Params {
  int M, N, K;
  int n_ttiles;          // token tiles: ceil(M / 256)
  int n_tiles;           // (N / 256) * n_ttiles pair tiles, token tile fastest
  int n_pairs;           // CTA pairs in the grid
  float* logits;         // [M, N] fp32
  const float* ssq_in;   // [n_ssq_in, M] or null (rs = 1)
  int n_ssq_in;
  float inv_k, eps;
};

__global__ void __launch_bounds__(THREADS, 1)
    unembed_pair_kernel(const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_x, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + RING_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2], used in the even CTA
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs
  const uint32_t peer = rank ^ 1u;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int nkb = p.K / BK;
  const int my_tiles = pair < p.n_tiles ? (p.n_tiles - 1 - pair) / p.n_pairs + 1 : 0;
  const int total_kb = my_tiles * nkb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * (EPI_THREADS / 32));
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  // both CTAs' barriers exist before either CTA signals the other's
  cluster_arrive_wait();

  const uint32_t abort_peer = cluster_addr(const_cast<int*>(abort_flag), peer);
  const uint32_t full_even = cluster_addr(full, 0);
  const uint64_t pol_w = l2_policy_evict_first();  // streamed once
  const uint64_t pol_x = l2_policy_evict_last();   // re-read by every pair

  // k-block g of this pair's walk: tile index and coordinates
  auto tile_of = [&](int li) { return pair + li * p.n_pairs; };
  auto issue_w = [&](int g) {
    const int st = g % STAGES;
    const int j = tile_of(g / nkb);
    const int v0 = (j / p.n_ttiles) * TILE_V + static_cast<int>(rank) * HALF_V;
    tma_load_2d_pair(smem + st * STAGE_BYTES, &tm_w, full_even + st * 8, (g % nkb) * BK, v0,
                     pol_w);
  };
  auto issue_x = [&](int g) {
    const int st = g % STAGES;
    const int j = tile_of(g / nkb);
    const int t0 = (j % p.n_ttiles) * TILE_T + static_cast<int>(rank) * HALF_T;
    tma_load_2d_pair(smem + st * STAGE_BYTES + A_BYTES, &tm_x, full_even + st * 8,
                     (g % nkb) * BK, t0, pol_x);
  };

  // The weights are never written by another kernel: the first stages' weight
  // tiles are requested before waiting on the predecessor.
  const int pre = min(STAGES, total_kb);
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < pre; ++g) {
      if (rank == 0) mbar_expect_tx(&full[g], 2 * STAGE_BYTES);
      issue_w(g);
    }
  }
  griddep_wait();
  if (warp == 0 && lane == 0)
    for (int g = 0; g < pre; ++g) issue_x(g);
  // TMEM is taken only once every earlier kernel has finished, so a CTA that
  // holds it never waits on a predecessor
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_arrive_wait();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  griddep_launch();

  if (warp == 0) {
    if (lane == 0) {
      int g = pre;
      for (; g < total_kb; ++g) {
        const int st = g % STAGES;
        if (!mbar_wait_pair(&empty[st], ((g / STAGES) - 1) & 1, abort_flag, abort_peer, 0x301))
          break;
        if (rank == 0) mbar_expect_tx(&full[st], 2 * STAGE_BYTES);
        issue_w(g);
        issue_x(g);
      }
      if (*abort_flag && rank == 0) {
        // let the loads in flight land before the CTA can exit
        for (int q = max(0, g - STAGES); q < g; ++q)
          mbar_wait(&full[q % STAGES], (q / STAGES) & 1, nullptr, 0x302);
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0 && total_kb > 0) {
      int g = 0;
      bool ok = true;
      for (int li = 0; li < my_tiles && ok; ++li) {
        const int b = li & 1;
        if (li >= 2 &&
            !mbar_wait_pair(&acc_empty[b], ((li >> 1) - 1) & 1, abort_flag, abort_peer, 0x303))
          break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(b * ACC_COLS);
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int st = g % STAGES;
          if (!mbar_wait_pair(&full[st], (g / STAGES) & 1, abort_flag, abort_peer, 0x304)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + st * STAGE_BYTES);
          const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_ss_pair(d, sdesc_sw128(a_base + kk * 32, 16, 1024),
                         sdesc_sw128(b_base + kk * 32, 16, 1024), IDESC, (kb | kk) != 0 ? 1u : 0u);
          umma_commit_pair(&empty[st], 0x3);
        }
        if (ok) umma_commit_pair(&acc_full[b], 0x3);
      }
      // nothing may still write TMEM when it is released
      umma_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, nullptr, 0x306);
    }
  } else {
    // warps 2..5: TMEM lane quarter (warp % 4) = this CTA's vocabulary rows.
    // The warps work independently (no barrier among them), so one that gives
    // up after an expired wait cannot strand the others.
    const int quarter = warp & 3;
    const uint32_t acc_empty_even = cluster_addr(acc_empty, 0);
    for (int li = 0; li < my_tiles; ++li) {
      const int b = li & 1;
      const int j = tile_of(li);
      const int tb = (j % p.n_ttiles) * TILE_T;
      const int v = (j / p.n_ttiles) * TILE_V + static_cast<int>(rank) * HALF_V + quarter * 32 +
                    lane;
      // row scale of token tb + 32 c + lane, for every chunk c, while the MMAs run
      float rs[TILE_T / 32];
#pragma unroll
      for (int c = 0; c < TILE_T / 32; ++c) {
        rs[c] = 1.f;
        const int tg = tb + c * 32 + lane;
        if (p.ssq_in != nullptr && tg < p.M) {
          float acc = 0.f;
          for (int q = 0; q < p.n_ssq_in; ++q) acc += p.ssq_in[static_cast<size_t>(q) * p.M + tg];
          rs[c] = rsqrtf(acc * p.inv_k + p.eps);
        }
      }
      if (!__all_sync(0xffffffffu,
                      mbar_wait_pair(&acc_full[b], (li >> 1) & 1, abort_flag, abort_peer, 0x305)))
        break;
      tc_fence_after();
      const uint32_t taddr =
          tmem + static_cast<uint32_t>(b * ACC_COLS) + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll
      for (int c = 0; c < TILE_T / 32; ++c) {
        if (tb + c * 32 >= p.M) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_ld_wait();
        float* out = p.logits + static_cast<size_t>(tb + c * 32) * p.N + v;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float sc = __shfl_sync(0xffffffffu, rs[c], i);
          if (tb + c * 32 + i < p.M) out[static_cast<size_t>(i) * p.N] = __uint_as_float(r[i]) * sc;
        }
      }
      // this warp's reads of buffer b are complete: the MMAs may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_even + b * 8);
    }
  }

  // every MMA has completed (each CTA saw its last acc_full) and every remote
  // arrival has landed before either CTA releases TMEM or exits
  tc_fence_before();
  cluster_arrive_wait();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace unembed
}  // namespace dg
