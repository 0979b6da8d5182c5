// unembed.cuh - the unembedding on CTA pairs, alone or fused with the sampler's
// row pass.
//
//   logits[t, v] = rs[t] * sum_k h[t, k] W_U[v, k]     h bf16 [M, K], W_U bf16 [V, K]
//
// with rs[t] = 1/sqrt(mean_k x[t,k]^2 + eps) the final RMSNorm (unit gain)
// folded in as a per-token scale, from per-(128-column tile, token) sums of
// squares of the residual stream.
//
// The vocabulary is far larger than the 148 SMs, so one persistent grid of
// CTA pairs walks 256 (vocabulary) x 256 (token) output tiles.  A pair tile is
// one cta_group::2 MMA chain: each CTA stages 128 rows of each operand per
// k-block and the pair's MMA (M = 256, N = 256, issued by the even CTA) reads
// both CTAs' halves.  Compared with one CTA per 128 x 256 tile this halves the
// activation bytes every SM pulls in per weight byte: with 256 tokens the
// activation tile is as large as the weight tile, so the single-CTA form moves
// three bytes through each SM per weight byte and the pair form two.
//
// The accumulator is double-buffered in TMEM (2 x 256 columns), so the
// epilogue of tile i overlaps the MMAs of tile i + 1.
//
// Two epilogues share the pipeline:
//   unembed_pair_kernel    A = W_U, B = h: TMEM lanes are vocabulary entries;
//                          fp32 logits stored straight from registers (a warp
//                          store covers 128 contiguous bytes of one token row).
//   unembed_sample_kernel  A = h, B = W_U: TMEM lanes are tokens, so a thread
//                          sees one token's vocabulary values and runs the
//                          sampler's row pass on them in registers - online
//                          softmax sums, raw-logit argmax, Gumbel race - across
//                          all the tiles of its pair.  The logits never reach
//                          memory; each (token, pair segment) leaves one
//                          partial for the merge.
//
// The projections of the stack use the same pipeline when there are enough
// 256 x 256 tiles (many tokens: prefill, wide batches): proj_pair_kernel,
// A = weights, B = activations, with the projection epilogues of gemm.cuh.
//
// Roles: warp 0 issues the TMA loads (both CTAs, each into its own ring,
// completion counted on the even CTA's barrier); warp 1 owns TMEM and, in the
// even CTA, one lane issues the MMAs; the epilogue warps (2 ..) read this
// CTA's 128 accumulator lanes.
#pragma once

#include "dg_common.cuh"
#include "gemm.cuh"
#include "sampler.cuh"

namespace dg {
namespace unembed {

constexpr int TILE = 256;                 // rows of each operand per pair tile (MMA M and N)
constexpr int HALF = TILE / 2;            // ... per CTA
constexpr int BK = 64;                    // one 128-byte swizzle row of bf16
constexpr int A_BYTES = HALF * BK * 2;    // 16 KB
constexpr int B_BYTES = HALF * BK * 2;    // 16 KB
constexpr int RING_BYTES = 6 * (A_BYTES + B_BYTES);  // 192 KB of TMA stages
constexpr int ACC_COLS = TILE;                    // fp32 columns per accumulator buffer
constexpr int TMEM_COLS = 2 * ACC_COLS;           // two buffers: all 512 columns
constexpr int SMEM_BYTES = 1024 + RING_BYTES + 256;
constexpr uint32_t IDESC = idesc_bf16_f32(TILE, TILE, false, false);

// Epilogue warps: 4 for the logits store, 12 for the fused sampler (three
// warps per TMEM lane quarter, each taking a third of a tile's columns: the
// row pass is a long dependent chain per element, and more warps hide it).
constexpr int STORE_EPI_WARPS = 4;
// The projections' epilogues: two warps per lane quarter, each taking half of
// a tile's token columns, so that twice the residual loads are in flight and a
// launch's last tile (whose epilogue nothing hides) drains in half the time.
constexpr int PROJ_EPI_WARPS = 8;
constexpr int SAMPLE_EPI_WARPS = 12;
constexpr int SAMPLE_SLOTS = SAMPLE_EPI_WARPS / 4;  // partials per (token, segment)
__host__ __device__ constexpr int threads_for(int epi_warps) { return 64 + 32 * epi_warps; }

// ---------------------------------------------------------------------------
// Shared pipeline.  Sched: count (tiles of this pair), nkb, a_row(li),
// b_row(li) (pair-level row origins; CTA r takes rows origin + 128 r).
// Epi (epilogue warps): start() once the predecessor kernels have finished,
// prepare(li) before the tile's accumulator is ready, consume(li, taddr, col0,
// ncols) once it is, finish() after the last tile.
// ---------------------------------------------------------------------------
template <int EPI_WARPS, int KPS, bool F8, class Sched, class Epi>
__device__ __forceinline__ void pair_pipeline(const CUtensorMap* tm_a, const CUtensorMap* tm_b,
                                              uint64_t pol_a, uint64_t pol_b, const Sched& sc,
                                              Epi& epi) {
  // A stage holds KPS consecutive k-blocks (their A tiles, then their B
  // tiles), so each row of a weight tile is requested KPS * 128 contiguous
  // bytes at a time.  sc.nkb is a multiple of KPS.  A k-block is one 128-byte
  // swizzle row per operand row: 64 bf16 or, with F8, 128 e4m3 elements
  // (kind::f8f6f4, 32 K per MMA instead of 16: the same 32-byte step).
  constexpr int STAGE_BYTES = KPS * (A_BYTES + B_BYTES);
  constexpr int STAGES = RING_BYTES / STAGE_BYTES;
  constexpr int KB_ELEMS = F8 ? 128 : BK;
  constexpr uint32_t MMA_IDESC = F8 ? idesc_e4m3_f32(TILE, TILE) : IDESC;
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
  const int nkb = sc.nkb;
  const int nstg = nkb / KPS;              // stages per tile
  const int total_stg = sc.count * nstg;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(tm_a);
    tma_prefetch_desc(tm_b);
  }
  // both CTAs' barriers exist before either CTA signals the other's
  cluster_arrive_wait();

  const uint32_t abort_peer = cluster_addr(const_cast<int*>(abort_flag), rank ^ 1u);
  const uint32_t full_even = cluster_addr(full, 0);
  const int roff = static_cast<int>(rank) * HALF;

  // stage g of this pair's walk: tile g / nstg, k-blocks KPS * (g % nstg) + j
  auto issue_a = [&](int g) {
    const int st = g % STAGES;
    for (int j = 0; j < KPS; ++j)
      tma_load_2d_pair(smem + st * STAGE_BYTES + j * A_BYTES, tm_a, full_even + st * 8,
                       (KPS * (g % nstg) + j) * KB_ELEMS, sc.a_row(g / nstg) + roff, pol_a);
  };
  auto issue_b = [&](int g) {
    const int st = g % STAGES;
    for (int j = 0; j < KPS; ++j)
      tma_load_2d_pair(smem + st * STAGE_BYTES + KPS * A_BYTES + j * B_BYTES, tm_b,
                       full_even + st * 8, (KPS * (g % nstg) + j) * KB_ELEMS,
                       sc.b_row(g / nstg) + roff, pol_b);
  };

  // The weights are never written by another kernel: the first stages' weight
  // tiles are requested before waiting on the predecessor.
  const int pre = min(STAGES, total_stg);
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < pre; ++g) {
      if (rank == 0) mbar_expect_tx(&full[g], 2 * STAGE_BYTES);
      if (Sched::kAIsWeight) issue_a(g); else issue_b(g);
    }
  }
  griddep_wait();
  if (warp >= 2) epi.start();
  if (warp == 0 && lane == 0)
    for (int g = 0; g < pre; ++g) {
      if (Sched::kAIsWeight) issue_b(g); else issue_a(g);
    }
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
      for (; g < total_stg; ++g) {
        const int st = g % STAGES;
        if (!mbar_wait_pair(&empty[st], ((g / STAGES) - 1) & 1, abort_flag, abort_peer, 0x301))
          break;
        if (rank == 0) mbar_expect_tx(&full[st], 2 * STAGE_BYTES);
        issue_a(g);
        issue_b(g);
      }
      if (*abort_flag && rank == 0) {
        // let the loads in flight land before the CTA can exit
        for (int q = max(0, g - STAGES); q < g; ++q)
          mbar_wait(&full[q % STAGES], (q / STAGES) & 1, nullptr, 0x302);
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0 && total_stg > 0) {
      int g = 0;
      bool ok = true;
      for (int li = 0; li < sc.count && ok; ++li) {
        const int b = li & 1;
        if (li >= 2 &&
            !mbar_wait_pair(&acc_empty[b], ((li >> 1) - 1) & 1, abort_flag, abort_peer, 0x303))
          break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(b * ACC_COLS);
        for (int q = 0; q < nstg; ++q, ++g) {
          const int st = g % STAGES;
          if (!mbar_wait_pair(&full[st], (g / STAGES) & 1, abort_flag, abort_peer, 0x304)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + st * STAGE_BYTES);
          const uint32_t b_base = a_base + KPS * A_BYTES;
#pragma unroll
          for (int j = 0; j < KPS; ++j)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // four 32-byte K steps per 128-byte row
              const uint64_t ad = sdesc_sw128(a_base + j * A_BYTES + kk * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(b_base + j * B_BYTES + kk * 32, 16, 1024);
              if constexpr (F8)
                umma_ss_pair_f8(d, ad, bd, MMA_IDESC, (q | j | kk) != 0 ? 1u : 0u);
              else
                umma_ss_pair(d, ad, bd, MMA_IDESC, (q | j | kk) != 0 ? 1u : 0u);
            }
          umma_commit_pair(&empty[st], 0x3);
        }
        if (ok) umma_commit_pair(&acc_full[b], 0x3);
      }
      // nothing may still write TMEM when it is released
      umma_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, nullptr, 0x306);
    }
  } else {
    // Epilogue warps, TMEM lane quarter warp % 4; with more than four, the
    // warps of a quarter split each tile's columns.  The warps work
    // independently (no barrier among them), so one that gives up after an
    // expired wait cannot strand the others.
    const int e = warp - 2;
    const int quarter = warp & 3;
    // warps per lane quarter split the tile's 32-column chunks as evenly as
    // possible: warp set k takes chunks [k C / W, (k + 1) C / W)
    constexpr int WPQ = EPI_WARPS / 4;
    constexpr int CHUNKS = ACC_COLS / 32;
    const int col0 = ((e / 4) * CHUNKS / WPQ) * 32;
    const int ncols = (((e / 4) + 1) * CHUNKS / WPQ) * 32 - col0;
    const uint32_t acc_empty_even = cluster_addr(acc_empty, 0);
    for (int li = 0; li < sc.count; ++li) {
      const int b = li & 1;
      epi.prepare(li);
      if (!__all_sync(0xffffffffu,
                      mbar_wait_pair(&acc_full[b], (li >> 1) & 1, abort_flag, abort_peer, 0x305)))
        break;
      tc_fence_after();
      epi.consume(li, tmem + static_cast<uint32_t>(b * ACC_COLS + col0) +
                          (static_cast<uint32_t>(quarter * 32) << 16),
                  col0, ncols);
      // this warp's reads of buffer b are complete: the MMAs may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_even + b * 8);
    }
    epi.finish();
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

// Row scale of token t (1 without sums of squares).  The partials are summed
// in index order; they are loaded sixteen at a time so that one round trip to
// L2 serves sixteen of them (adding the zeros past the end changes nothing:
// the sum is non-negative).
__device__ __forceinline__ float row_scale(const float* ssq_in, int n_ssq_in, int M, int t,
                                           float inv_k, float eps) {
  if (ssq_in == nullptr || t >= M) return 1.f;
  float acc = 0.f;
  for (int q0 = 0; q0 < n_ssq_in; q0 += 16) {
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      v[j] = q0 + j < n_ssq_in ? ssq_in[static_cast<size_t>(q0 + j) * M + t] : 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) acc += v[j];
  }
  return rsqrtf(acc * inv_k + eps);
}

// The dequantisation scales of an e4m3 launch folded into the row scale:
// per-token scale of the activations (or null) times the weights' tensor scale
// (device scalar, or null).
__device__ __forceinline__ float fp8_scale(const float* tok_scale, const float* w_scale, int M,
                                           int t) {
  float s = 1.f;
  if (tok_scale != nullptr && t < M) s = tok_scale[t];
  if (w_scale != nullptr) s *= *w_scale;
  return s;
}

// ---------------------------------------------------------------------------
// Logits to memory.
// ---------------------------------------------------------------------------
struct Params {
  int M, N, K;
  int n_ttiles;          // token tiles: ceil(M / 256)
  int n_tiles;           // (N / 256) * n_ttiles pair tiles, token tile fastest
  int n_pairs;           // CTA pairs in the grid
  float* logits;         // [M, N] fp32
  const float* ssq_in;   // [n_ssq_in, M] or null (rs = 1)
  int n_ssq_in;
  float inv_k, eps;
  const float* tok_scale;  // e4m3 operands: per-token scale [M], else null
  const float* w_scale;    // e4m3 operands: the weights' scale (device scalar), else null
};

struct StoreSched {
  static constexpr bool kAIsWeight = true;
  int count, nkb, pair, n_pairs, n_ttiles;
  __device__ int tile(int li) const { return pair + li * n_pairs; }
  __device__ int a_row(int li) const { return (tile(li) / n_ttiles) * TILE; }  // vocabulary
  __device__ int b_row(int li) const { return (tile(li) % n_ttiles) * TILE; }  // tokens
};

struct StoreEpi {
  const Params* p;
  const StoreSched* sc;
  uint32_t rank;
  int quarter, lane;
  float rs[TILE / 32];  // scale of token (tile base + 32 c + lane)

  __device__ void start() {}
  __device__ void prepare(int li) {
    const int tb = sc->b_row(li);
#pragma unroll
    for (int c = 0; c < TILE / 32; ++c)
      rs[c] = row_scale(p->ssq_in, p->n_ssq_in, p->M, tb + c * 32 + lane, p->inv_k, p->eps) *
              fp8_scale(p->tok_scale, p->w_scale, p->M, tb + c * 32 + lane);
  }
  __device__ void consume(int li, uint32_t taddr, int col0, int ncols) {
    (void)col0;
    (void)ncols;
    const int tb = sc->b_row(li);
    const int v = sc->a_row(li) + static_cast<int>(rank) * HALF + quarter * 32 + lane;
#pragma unroll
    for (int c = 0; c < TILE / 32; ++c) {
      if (tb + c * 32 >= p->M) break;  // warp-uniform
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
      float* out = p->logits + static_cast<size_t>(tb + c * 32) * p->N + v;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float sc_i = __shfl_sync(0xffffffffu, rs[c], i);
        if (tb + c * 32 + i < p->M) out[static_cast<size_t>(i) * p->N] = __uint_as_float(r[i]) * sc_i;
      }
    }
  }
  __device__ void finish() {}
};

template <int KPS, bool F8>
__global__ void __launch_bounds__(threads_for(STORE_EPI_WARPS), 1)
    unembed_pair_kernel(const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_x, Params p) {
  const int pair = static_cast<int>(blockIdx.x >> 1);
  StoreSched sc;
  sc.nkb = p.K / (F8 ? 128 : BK);
  sc.pair = pair;
  sc.n_pairs = p.n_pairs;
  sc.n_ttiles = p.n_ttiles;
  sc.count = pair < p.n_tiles ? (p.n_tiles - 1 - pair) / p.n_pairs + 1 : 0;
  StoreEpi epi;
  epi.p = &p;
  epi.sc = &sc;
  epi.rank = cluster_ctarank();
  epi.quarter = warp_id() & 3;
  epi.lane = lane_id();
  pair_pipeline<STORE_EPI_WARPS, KPS, F8>(&tm_w, &tm_x, l2_policy_evict_first(), l2_policy_evict_last(),
                                 sc, epi);
}

// ---------------------------------------------------------------------------
// Projections of the stack on CTA pairs (many tokens).  The epilogues of
// gemm.cuh: EPI_F32 / EPI_BF16 / EPI_GELU take rs[t] * acc; EPI_RESID adds
// acc (times the e4m3 scales) to the fp32 residual stream, writes its bf16
// copy and the sums of squares of each 32-feature group (one warp's lanes),
// ssq_out [N / 32, M], so that no warp waits on another.
// ---------------------------------------------------------------------------
struct ProjParams {
  int M, N, K;
  int n_ttiles, n_tiles, n_pairs;
  int epi;                   // dg::gemm::Epi
  float* out_f32;            // EPI_F32
  __nv_bfloat16* out_bf16;   // EPI_BF16 / EPI_GELU / EPI_RESID (optional there)
  float* x;                  // EPI_RESID residual stream [M, N]
  const float* ssq_in;       // [n_ssq_in, M] or null (rs = 1)
  int n_ssq_in;
  float inv_k, eps;
  float* ssq_out;            // EPI_RESID: [N / 32, M], or null
  const float* tok_scale;    // e4m3 operands: per-token scale [M], else null
  const float* w_scale;      // e4m3 operands: the weights' scale (device scalar), else null
};

template <int EPI>
struct ProjEpi {
  ProjParams p;  // a copy: read in a rolled loop, a pointer to the launch's
                 // parameters would put them on the stack
  const StoreSched* sc;
  uint32_t rank;
  int quarter, lane;
  float rs[TILE / 32];  // scale of token (tile base + 32 c + lane)

  __device__ void start() {}
  // the scales of this warp's own token chunks only (the pipeline gives warp
  // set (warp - 2) / 4 the chunks [4 k, 4 k + 4) of a tile)
  __device__ void prepare(int li) {
    static_assert(PROJ_EPI_WARPS == 8, "two warps per lane quarter, four chunks each");
    const int tb = sc->b_row(li);
    const int mine = (warp_id() - 2) >> 2;
#pragma unroll
    for (int c = 0; c < TILE / 32; ++c) {
      if (c / (TILE / 64) != mine) {
        rs[c] = 1.f;  // another warp's chunk
        continue;
      }
      rs[c] = row_scale(p.ssq_in, p.n_ssq_in, p.M, tb + c * 32 + lane, p.inv_k, p.eps) *
              fp8_scale(p.tok_scale, p.w_scale, p.M, tb + c * 32 + lane);
    }
  }
  // A rolled loop over 32-token chunks with a small unrolled body (the whole
  // tile unrolled is thousands of instructions per warp and measured slower
  // than the mainloop it should hide behind).  Per 16 tokens: the residual
  // rows are all loaded before the first store; bf16 outputs go out two rows
  // per store with every lane active (even lanes row k, odd lanes row k + 1,
  // after one exchange of neighbours); the sums of squares of the 16 rows are
  // one transposed reduction (16 shuffles instead of 5 per row).
  __device__ void consume(int li, uint32_t taddr, int col0, int ncols) {
    constexpr bool kBf16 = EPI != gemm::EPI_F32;
    const unsigned full = 0xffffffffu;
    const int M = p.M;
    const size_t N = static_cast<size_t>(p.N);
    const int tb = sc->b_row(li);
    const int fq = sc->a_row(li) + static_cast<int>(rank) * HALF + quarter * 32;  // this warp's features
    const bool odd = (lane & 1) != 0;
    const int fpair = fq + (lane & ~1);  // first feature of this lane's bf16 pair
    // this warp's token columns [col0, col0 + ncols) of the tile (taddr
    // already points at col0)
    const int tc0 = tb + col0;
    const int nch = M - tc0 <= 0 ? 0 : min(ncols, M - tc0 + 31) / 32;
    // rs is rotated so that rs[0] is the current chunk's (static indices only)
    float rsr[TILE / 32];
#pragma unroll
    for (int c = 0; c < TILE / 32; ++c) rsr[c] = rs[c];
#pragma unroll 1
    for (int c = 0; c < col0 / 32; ++c) {
#pragma unroll
      for (int c2 = 0; c2 + 1 < TILE / 32; ++c2) rsr[c2] = rsr[c2 + 1];
    }
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
      const float rsc = rsr[0];
#pragma unroll
      for (int c2 = 0; c2 + 1 < TILE / 32; ++c2) rsr[c2] = rsr[c2 + 1];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t0 = tc0 + c * 32 + h * 16;
        const size_t o0 = static_cast<size_t>(t0) * N + fq + lane;
        uint32_t r[16];
        tmem_ld16(taddr + c * 32 + h * 16, r);
        float y[16];
        if constexpr (EPI == gemm::EPI_RESID) {
#pragma unroll
          for (int k = 0; k < 16; ++k) y[k] = t0 + k < M ? p.x[o0 + k * N] : 0.f;
        }
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float v = __uint_as_float(r[k]) * __shfl_sync(full, rsc, h * 16 + k);
          if constexpr (EPI == gemm::EPI_RESID)
            y[k] += v;
          else if constexpr (EPI == gemm::EPI_GELU)
            y[k] = gemm::gelu_erf(v);
          else
            y[k] = v;
        }
        if constexpr (EPI == gemm::EPI_RESID || EPI == gemm::EPI_F32) {
          float* const dst = EPI == gemm::EPI_RESID ? p.x : p.out_f32;
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (t0 + k < M) dst[o0 + k * N] = y[k];
        }
        if (kBf16 && p.out_bf16 != nullptr) {
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            const float got = __shfl_xor_sync(full, odd ? y[k] : y[k + 1], 1);
            const uint32_t w = odd ? pack_bf16x2(got, y[k + 1]) : pack_bf16x2(y[k], got);
            const int row = t0 + k + (odd ? 1 : 0);
            if (row < M)
              *reinterpret_cast<uint32_t*>(p.out_bf16 + static_cast<size_t>(row) * N + fpair) = w;
          }
        }
        if constexpr (EPI == gemm::EPI_RESID) {
          if (p.ssq_out != nullptr) {
            // halving exchange: after the step on lane bit b a lane keeps the
            // upper half of its rows if that bit is set; 16 rows end as one
            // per lane, row = bit-reverse of lane % 16
            float a[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) a[k] = y[k] * y[k];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              const int n = 16 >> b;
              const bool up = ((lane >> b) & 1) != 0;
#pragma unroll
              for (int i = 0; i < n / 2; ++i) {
                const float send = up ? a[i] : a[i + n / 2];
                const float keep = up ? a[i + n / 2] : a[i];
                a[i] = keep + __shfl_xor_sync(full, send, 1 << b);
              }
            }
            const float sq = a[0] + __shfl_xor_sync(full, a[0], 16);
            const int row = ((lane & 1) << 3) | ((lane & 2) << 1) | ((lane & 4) >> 1) |
                            ((lane & 8) >> 3);
            if (lane < 16 && t0 + row < M)
              p.ssq_out[static_cast<size_t>(fq / 32) * M + t0 + row] = sq;
          }
        }
      }
    }
  }
  __device__ void finish() {}
};

// One kernel per epilogue: each carries a single unrolled store path.
template <int KPS, bool F8, int EPI>
__global__ void __launch_bounds__(threads_for(PROJ_EPI_WARPS), 1)
    proj_pair_kernel(const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_x, ProjParams p) {
  const int pair = static_cast<int>(blockIdx.x >> 1);
  StoreSched sc;
  sc.nkb = p.K / (F8 ? 128 : BK);
  sc.pair = pair;
  sc.n_pairs = p.n_pairs;
  sc.n_ttiles = p.n_ttiles;
  sc.count = pair < p.n_tiles ? (p.n_tiles - 1 - pair) / p.n_pairs + 1 : 0;
  ProjEpi<EPI> epi;
  epi.p = p;
  epi.sc = &sc;
  epi.rank = cluster_ctarank();
  epi.quarter = warp_id() & 3;
  epi.lane = lane_id();
  // the pairs that share a weight tile run at the same time (token tile
  // fastest), so the weights can go first from L2 while the activations,
  // read by every weight tile, stay (evict-normal weights measured the same)
  pair_pipeline<PROJ_EPI_WARPS, KPS, F8>(&tm_w, &tm_x, l2_policy_evict_first(),
                                         l2_policy_evict_last(), sc, epi);
}

// ---------------------------------------------------------------------------
// Unembedding fused with the sampler's row pass.
//
// Pair p works on token tile p / segs and on the contiguous vocabulary range
// [seg * V / segs, (seg + 1) * V / segs) (in 256-entry tiles), seg = p % segs.
// A thread of an epilogue warp owns one token and one third of each tile's
// columns; it keeps the row pass state of sampler.cuh across the range and
// writes one FusedPartial at the end, slot (token, 3 seg + third).
// ---------------------------------------------------------------------------
struct SampleFusedParams {
  int M, N, K;            // tokens, vocabulary, width
  int n_vtiles;           // N / 256
  int segs;               // pairs per token tile
  int n_pairs;            // segs * ceil(M / 256)
  const float* ssq_in;
  int n_ssq_in;
  float inv_k, eps;
  const float* tok_scale; // e4m3 operands: per-token scale [M], else null
  const float* w_scale;   // e4m3 operands: the weights' scale (device scalar), else null
  SampleParams sp;        // sampler settings (B, C, V = N, seed, block, step, temperature)
  const int32_t* tok;     // [M] current canvas tokens
  FusedPartial* part;     // [M, SAMPLE_SLOTS * segs]
};

struct SampleSched {
  static constexpr bool kAIsWeight = false;
  int count, nkb, tt, vt0;
  __device__ int a_row(int li) const { (void)li; return tt * TILE; }   // tokens
  __device__ int b_row(int li) const { return (vt0 + li) * TILE; }     // vocabulary
};

struct SampleEpi {
  const SampleFusedParams* p;
  const SampleSched* sc;
  int t;            // token row (global), may be >= M in a ragged tile
  int slot;
  int cur;          // current canvas token (its logit is recorded)
  float k2, rs;
  uint32_t c1, step, block;
  uint2 key;
  RowState st;

  int seg;

  __device__ void start() {
    const uint32_t rank = cluster_ctarank();
    const int warp = warp_id(), lane = lane_id();
    const int e = warp - 2;
    t = sc->tt * TILE + static_cast<int>(rank) * HALF + (warp & 3) * 32 + lane;
    slot = SAMPLE_SLOTS * seg + e / 4;
    const bool valid = t < p->M;
    const int b = valid ? t / p->sp.C : 0;
    const int pos = valid ? t - b * p->sp.C : 0;
    cur = valid ? p->tok[t] : -1;
    const int s = read_step(p->sp);
    step = static_cast<uint32_t>(s);
    block = static_cast<uint32_t>(p->sp.block);
    k2 = 1.4426950408889634f / step_temperature(s, p->sp.max_steps, p->sp.t_start, p->sp.t_end);
    rs = row_scale(p->ssq_in, p->n_ssq_in, p->M, t, p->inv_k, p->eps) *
         fp8_scale(p->tok_scale, p->w_scale, p->M, t);
    c1 = (static_cast<uint32_t>(pos) & 0xFFFFFFu) | (kTagGumbel << 24);
    key = make_uint2(p->sp.seed, static_cast<uint32_t>(b));
    st.reset();
  }
  __device__ void prepare(int li) { (void)li; }
  __device__ void consume(int li, uint32_t taddr, int col0, int ncols) {
    const int vbase = sc->b_row(li) + col0;
    for (int c = 0; c < ncols; c += 32) {
      uint32_t r[32];
      tmem_ld32(taddr + c, r);
      tmem_ld_wait();
      float l[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) l[i] = __uint_as_float(r[i]) * rs;
      st.update32(l, vbase + c, cur, k2, c1, step, block, key);
    }
  }
  __device__ void finish() {
    if (t < p->M) p->part[static_cast<size_t>(t) * (SAMPLE_SLOTS * p->segs) + slot] = st.partial(k2);
  }
};

template <int KPS, bool F8>
__global__ void __launch_bounds__(threads_for(SAMPLE_EPI_WARPS), 1)
    unembed_sample_kernel(const __grid_constant__ CUtensorMap tm_x,
                          const __grid_constant__ CUtensorMap tm_w, SampleFusedParams p) {
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int seg = pair % p.segs;
  SampleSched sc;
  sc.nkb = p.K / (F8 ? 128 : BK);
  sc.tt = pair / p.segs;
  sc.vt0 = static_cast<int>((static_cast<long long>(seg) * p.n_vtiles) / p.segs);
  sc.count = static_cast<int>((static_cast<long long>(seg + 1) * p.n_vtiles) / p.segs) - sc.vt0;
  SampleEpi epi;
  epi.p = &p;
  epi.sc = &sc;
  epi.seg = seg;
  pair_pipeline<SAMPLE_EPI_WARPS, KPS, F8>(&tm_x, &tm_w, l2_policy_evict_last(), l2_policy_evict_first(),
                                  sc, epi);
}

}  // namespace unembed
}  // namespace dg
