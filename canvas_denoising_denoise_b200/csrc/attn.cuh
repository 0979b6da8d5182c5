// attn.cuh - canvas attention on tcgen05 (flash-style, one pass over the keys).
//
// Lq new rows of query head h attend to [cached prefix of kv head g ; new
// rows], g = h / (Hq / Hkv), scale 1/sqrt(hd), no positional encoding; the
// mask is full over the canvas (denoising) or lower-triangular over the new
// rows (prefill, block re-encode).  Sources: aiexpert.news "Google's
// DiffusionGemma Atinge 1.000 Tokens por Segundo", architecture paragraph
// (bidirectional attention on the 256-token canvas; causal prefill into the
// KV cache); "DiffusionGemma Guia do Desenvolvedor ...", bullet "Propagacao
// de Contexto Bidirecional".
//
// One CTA = two 128-row query tiles that share a kv head, over a contiguous
// range of 128-key tiles (the key range is split across CTAs when there are
// too few query tiles to fill the SMs; a combine kernel merges the splits by
// their log-sum-exp).  Per key tile j and query tile X in {A, B}:
//     S_X = Q_X K_j^T          tcgen05.mma, A = Q_X (smem), B = K_j (smem), D in TMEM
//     P_X = 2^(S_X*c - m_X)    softmax warpgroup X: TMEM -> registers -> bf16 -> TMEM
//     O_X += P_X V_j           tcgen05.mma, A = P_X (TMEM), B = V_j (smem, MN-major)
// Each K/V tile is loaded once for both query tiles.  The two softmax
// warpgroups ping-pong: while one works, the tensor core runs the other
// tile's MMAs.  P_X overwrites S_X in place.  The running max is only raised
// (and O rescaled) when it grows by more than 2^8, so most tiles need no O
// round trip; the final 1/l normalisation makes this exact.
//
// Warps: 0 = TMA producer, 1 = TMEM owner + MMA issuer, 2..5 = softmax of
// tile A, 6..9 = softmax of tile B (one query row per thread; warp w owns
// TMEM lanes 32*(w%4)..+31).
//
// The e4m3 variant (F8, hd = 128) runs both products as kind::f8f6f4 MMAs:
// Q, K and V^T tiles are 8-bit codes, the scores are dequantised by the row's
// query scale and the K scale inside the softmax's exponent, P is written to
// TMEM as e4m3 (four per column), and the V scale joins 1/l.  The FP8 serving
// figure this follows: aiexpert.news, "Google's DiffusionGemma Atinge 1.000
// Tokens por Segundo", throughput paragraph (FP8 on one H200).
#pragma once

#include <cuda_fp8.h>

#include <type_traits>

#include "dg_common.cuh"

namespace dg {
namespace attn {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int THREADS = 320;  // warp 0 TMA, warp 1 MMA, warps 2-5 softmax A, warps 6-9 softmax B
constexpr int TMEM_COLS = 512;  // S_A [0,128) S_B [128,256) O_A [256,384) O_B [384,512)
constexpr float kRescaleThreshold = 8.0f;

// 2^x on the special-function unit (flushes denormal results to zero, which
// only affects probabilities below 2^-126).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// F8: e4m3 operands (hd = 128).  Q, K and the probabilities are K-major as in
// the bf16 kernel; V is stored transposed (keys contiguous), so that V^T tiles
// are K-major B operands too.  Every MMA consumes 32 bytes of K either way.
template <int HD, bool F8 = false>
struct Cfg {
  static constexpr int EB = F8 ? 1 : 2;              // bytes per element
  static constexpr int ATOM = 128 / EB;              // elements per 128-byte swizzle row
  static constexpr int HALVES = HD / ATOM;           // swizzle atoms across a row of hd
  static constexpr int Q_BYTES = BQ * HD * EB;
  static constexpr int T_BYTES = BKV * HD * EB;      // one K or V tile
  static constexpr int STAGES = F8 ? 4 : (HD == 128 ? 2 : 3);
  static constexpr int SMEM_BYTES = 1024 + 2 * Q_BYTES + STAGES * 2 * T_BYTES + 256;
  static constexpr int QK_MMAS = HD * EB / 32;
  static constexpr int PV_MMAS = BKV * EB / 32;
  static constexpr uint32_t IDESC_QK =
      F8 ? idesc_e4m3_f32(BQ, BKV) : idesc_bf16_f32(BQ, BKV, false, false);
  static constexpr uint32_t IDESC_PV =
      F8 ? idesc_e4m3_f32(BQ, HD) : idesc_bf16_f32(BQ, HD, false, true);
  // the epilogue stages both tiles' fp32 O in the K/V ring
  static_assert(STAGES * 2 * T_BYTES >= 2 * BQ * HD * 4, "O staging does not fit the ring");
  static_assert(!F8 || HD == 128, "e4m3 attention needs hd = 128");
};

// Four probabilities as e4m3 codes, the first in the lowest byte (the K order
// of a TMEM A operand of an 8-bit MMA).
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

struct Params {
  int B, Hq, Hkv, Lq, lmax, group;
  int n_rt;        // 128-row tiles per head
  int n_pairs;     // CTAs (per kv head and split) = ceil(group * n_rt / 2)
  int n_splits, causal;
  float scale_log2;          // scale * log2(e)
  const int32_t* cache_len;  // [B]
  __nv_bfloat16* out;        // [B, Lq, ldo]
  int ldo;
  float* lse;                // [B, Hq, Lq] natural log, or null
  __nv_bfloat16* part_o;     // [S, B, Hq, Lq, hd] bf16 (n_splits > 1)
  float* part_lse;           // [S, B, Hq, Lq]
  // e4m3 operands: per-token query scales [B * Lq], K and V scales (scalars)
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
};


// One CTA = two 128-row query tiles that read the same kv head (the query
// tiles of a kv head are ordered row tile first, so a pair shares its row
// tile whenever the group size is even), over one contiguous range of
// 128-key tiles.  The tensor core alternates [PV_A(j), S_A(j+1)] and
// [PV_B(j), S_B(j+1)] so that one softmax warpgroup works while the other
// tile's MMAs run.  S_X(j+1) is issued after PV_X(j), so once S_X(j+1) is
// complete, O_X is stable and may be rescaled in TMEM.
template <int HD, bool F8 = false>
__global__ void __launch_bounds__(THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kn,
                const __grid_constant__ CUtensorMap tm_vn,
                const __grid_constant__ CUtensorMap tm_kc,
                const __grid_constant__ CUtensorMap tm_vc, Params p) {
  using CF = Cfg<HD, F8>;
  constexpr int ST = CF::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                          // [2][Q_BYTES]
  uint8_t* sK = sQ + 2 * CF::Q_BYTES;          // ST tiles
  uint8_t* sV = sK + ST * CF::T_BYTES;         // ST tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + ST * CF::T_BYTES);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;       // [ST]
  uint64_t* v_full = k_full + ST;      // [ST]
  uint64_t* kv_empty = v_full + ST;    // [ST]
  uint64_t* s_full = kv_empty + ST;    // [2] per tile
  uint64_t* p_full = s_full + 2;       // [2] per tile
  uint64_t* o_final = p_full + 2;      // after the last PV of both tiles
  uint64_t* drain = o_final + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  // Causal launches take their heaviest query tiles (the last rows, which see
  // the most keys) first, so that the light ones fill the tail of the grid;
  // the canvas mask gives every pair the same work.
  const int nbg = p.Hkv * p.B;
  const int pi = p.causal ? p.n_pairs - 1 - static_cast<int>(blockIdx.x) / nbg
                          : static_cast<int>(blockIdx.x) % p.n_pairs;
  const int gb = p.causal ? static_cast<int>(blockIdx.x) % nbg
                          : static_cast<int>(blockIdx.x) / p.n_pairs;
  const int g = gb % p.Hkv;
  const int b = gb / p.Hkv;
  const int split = blockIdx.y;
  const int nq = p.group * p.n_rt;  // query tiles of this kv head
  int hX[2], i0X[2];
  bool vX[2];
#pragma unroll
  for (int X = 0; X < 2; ++X) {
    const int qi = 2 * pi + X;
    vX[X] = qi < nq;
    const int qq = vX[X] ? qi : 2 * pi;
    hX[X] = g * p.group + qq % p.group;
    i0X[X] = (qq / p.group) * BQ;
  }

  // The cache length and the cached prefix are written only by launches that
  // are fully ordered before this one (prefill's length set, the block commit
  // and its length bump), so they are read before griddepcontrol.wait; the
  // query tiles and the new rows' keys come from the preceding projection and
  // are read after it, as is every write.
  griddep_launch();
  int L = p.cache_len[b];
  if (L < 0 || L > p.lmax) {
    if (threadIdx.x == 0 && split == 0 && pi == 0 && g == 0) raise_error(ERR_CHECK | 0x301, b);
    L = L < 0 ? 0 : p.lmax;
  }
  const int i0max = max(i0X[0], vX[1] ? i0X[1] : 0);
  const int lq_vis = p.causal ? min(p.Lq, i0max + BQ) : p.Lq;
  const int nP = (L + BKV - 1) / BKV;
  const int nC = (lq_vis + BKV - 1) / BKV;
  const int T = nP + nC;
  const int t_beg = static_cast<int>((static_cast<long long>(T) * split) / p.n_splits);
  const int t_end = static_cast<int>((static_cast<long long>(T) * (split + 1)) / p.n_splits);
  const int n = t_end - t_beg;

  if (n <= 0) {
    // empty key range: this split contributes nothing to the merge
    griddep_wait();
    for (int X = 0; X < 2; ++X) {
      if (!vX[X] || threadIdx.x >= BQ) continue;
      const int qrow = i0X[X] + threadIdx.x;
      if (qrow < p.Lq) {
        const size_t r = ((static_cast<size_t>(split) * p.B + b) * p.Hq + hX[X]) * p.Lq + qrow;
        p.part_lse[r] = -INFINITY;
        uint4* o = reinterpret_cast<uint4*>(p.part_o + r * HD);
        for (int c = 0; c < HD / 8; ++c) o[c] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], BQ);
    }
    mbar_init(o_final, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kn);
    tma_prefetch_desc(&tm_vn);
    tma_prefetch_desc(&tm_kc);
    tma_prefetch_desc(&tm_vc);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const bool vB = vX[1];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      auto load_kv = [&](int i) {
        const int st = i % ST;
        const int t = t_beg + i;
        const CUtensorMap* mk;
        const CUtensorMap* mv;
        int x0, y0, key0;
        if (t < nP) {
          mk = &tm_kc;
          mv = &tm_vc;
          x0 = 0;
          y0 = (b * p.Hkv + g) * p.lmax + t * BKV;
          key0 = t * BKV;
        } else {
          mk = &tm_kn;
          mv = &tm_vn;
          x0 = g * HD;
          y0 = b * p.Lq + (t - nP) * BKV;
          key0 = (t - nP) * BKV;
        }
        uint8_t* kd = sK + st * CF::T_BYTES;
        uint8_t* vd = sV + st * CF::T_BYTES;
        mbar_expect_tx(&k_full[st], CF::T_BYTES);
        for (int hf = 0; hf < CF::HALVES; ++hf)
          tma_load_2d(kd + hf * (BKV * 128), mk, &k_full[st], x0 + hf * CF::ATOM, y0);
        mbar_expect_tx(&v_full[st], CF::T_BYTES);
        if constexpr (F8) {
          // V^T tile: rows d of kv head (b, g), 128 keys from key0
          tma_load_2d(vd, mv, &v_full[st], key0, (b * p.Hkv + g) * HD);
        } else {
          for (int hf = 0; hf < CF::HALVES; ++hf)
            tma_load_2d(vd + hf * (BKV * 128), mv, &v_full[st], x0 + hf * CF::ATOM, y0);
        }
      };
      // the first stages' cached-prefix tiles need no wait on the predecessor
      int issued = 0;
      while (issued < min(ST, n) && t_beg + issued < nP) load_kv(issued++);
      griddep_wait();
      mbar_expect_tx(q_full, CF::Q_BYTES * (vB ? 2 : 1));
      for (int X = 0; X < (vB ? 2 : 1); ++X)
        for (int hf = 0; hf < CF::HALVES; ++hf)
          tma_load_2d(sQ + X * CF::Q_BYTES + hf * (BQ * 128), &tm_q, q_full,
                      hX[X] * HD + hf * CF::ATOM, b * p.Lq + i0X[X]);
      for (int i = issued; i < n; ++i) {
        const int st = i % ST;
        if (i >= ST && !mbar_wait(&kv_empty[st], ((i / ST) - 1) & 1, abort_flag, 0x311)) break;
        load_kv(i);
        issued = i + 1;
      }
      if (*abort_flag) {
        mbar_wait(q_full, 0, nullptr, 0x312);
        for (int i = max(0, issued - ST); i < issued; ++i) {
          mbar_wait(&k_full[i % ST], (i / ST) & 1, nullptr, 0x313);
          mbar_wait(&v_full[i % ST], (i / ST) & 1, nullptr, 0x314);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, abort_flag, 0x321);
      const uint32_t q_base = smem_u32(sQ);
      auto issue_s = [&](int X, int i) {
        const uint32_t k_base = smem_u32(sK + (i % ST) * CF::T_BYTES);
        const uint32_t qb = q_base + X * CF::Q_BYTES;
#pragma unroll
        for (int kk = 0; kk < CF::QK_MMAS; ++kk) {
          const uint32_t off = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;
          if constexpr (F8)
            umma_ss_f8(tmem + X * 128, sdesc_sw128(qb + off, 16, 1024),
                       sdesc_sw128(k_base + off, 16, 1024), CF::IDESC_QK, kk > 0 ? 1u : 0u);
          else
            umma_ss(tmem + X * 128, sdesc_sw128(qb + off, 16, 1024),
                    sdesc_sw128(k_base + off, 16, 1024), CF::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[X]);
      };
      auto issue_pv = [&](int X, int j) -> bool {
        if (!mbar_wait(&p_full[X], j & 1, abort_flag, 0x323)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(sV + (j % ST) * CF::T_BYTES);
#pragma unroll
        for (int kk = 0; kk < CF::PV_MMAS; ++kk) {
          // A = P (TMEM, 8 columns per MMA); B = V (MN-major bf16) or V^T (K-major e4m3)
          if constexpr (F8)
            umma_ts_f8(tmem + 256 + X * 128, tmem + X * 128 + kk * 8,
                       sdesc_sw128(v_base + kk * 32, 16, 1024), CF::IDESC_PV,
                       (j > 0 || kk > 0) ? 1u : 0u);
          else
            umma_ts(tmem + 256 + X * 128, tmem + X * 128 + kk * 8,
                    sdesc_sw128(v_base + kk * 16 * 128, BKV * 128, 1024), CF::IDESC_PV,
                    (j > 0 || kk > 0) ? 1u : 0u);
        }
        return true;
      };
      if (ok) ok = mbar_wait(&k_full[0], 0, abort_flag, 0x322);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        if (vB) issue_s(1, 0);
      }
      for (int j = 0; ok && j < n; ++j) {
        ok = mbar_wait(&v_full[j % ST], (j / ST) & 1, abort_flag, 0x324);
        if (ok) ok = issue_pv(0, j);
        const bool more = j + 1 < n;
        if (ok && more) {
          ok = mbar_wait(&k_full[(j + 1) % ST], ((j + 1) / ST) & 1, abort_flag, 0x322);
          if (ok) {
            tc_fence_after();
            issue_s(0, j + 1);
          }
        }
        if (ok && vB) ok = issue_pv(1, j);
        if (ok) umma_commit(&kv_empty[j % ST]);
        if (ok && vB && more) issue_s(1, j + 1);
      }
      if (ok) umma_commit(o_final);
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, 0x325);
    }
  } else {
    // ------------------------------------------------------------ softmax (tile X)
    griddep_wait();  // before this warpgroup's writes
    const int X = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int qrow = i0X[X] + r;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + X * 128 + lane_off;
    const uint32_t tO = tmem + 256 + X * 128 + lane_off;
    float m = -INFINITY;  // running max in scaled log2 units
    float l = 0.f;
    bool ok = vX[X];
    // score -> log2 units: scale log2(e), times the dequantisation scales of
    // the row's query and of K on e4m3 operands (all positive)
    float sc = p.scale_log2;
    if constexpr (F8)
      sc *= (qrow < p.Lq ? p.q_scale[static_cast<size_t>(b) * p.Lq + qrow] : 1.f) * *p.k_scale;
    for (int j = 0; j < n && ok; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[X], j & 1, abort_flag, 0x331))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // key validity of this tile for this row: keys [0, lim] may be valid
      const int t = t_beg + j;
      int lim;
      if (t < nP) {
        lim = min(BKV, L - t * BKV) - 1;
      } else {
        const int ck0 = (t - nP) * BKV;
        lim = min(BKV, p.Lq - ck0) - 1;
        if (p.causal) lim = min(lim, qrow - ck0);
      }
      const bool masked = __any_sync(0xffffffffu, lim < BKV - 1);
      // pass 1: row max of the raw scores (the scale is positive)
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t sa[32], sb[32];
        tmem_ld32(tS + h2 * 64, sa);
        tmem_ld32(tS + h2 * 64 + 32, sb);
        tmem_ld_wait();
        if (masked) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (h2 * 64 + c > lim) sa[c] = __float_as_uint(-INFINITY);
            if (h2 * 64 + 32 + c > lim) sb[c] = __float_as_uint(-INFINITY);
          }
        }
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          mx0 = fmaxf(mx0, __uint_as_float(sa[c]));
          mx1 = fmaxf(mx1, __uint_as_float(sa[c + 1]));
          mx2 = fmaxf(mx2, __uint_as_float(sb[c]));
          mx3 = fmaxf(mx3, __uint_as_float(sb[c + 1]));
        }
      }
      const float tmax = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sc;
      // Raise the running max only when it grows by more than 2^8 (the final
      // 1/l keeps this exact).  Decided per warp: TMEM accesses are
      // warp-collective.  PV_X(j-1) is complete because S_X(j) is.
      const bool want = tmax > m + kRescaleThreshold || m == -INFINITY;
      if (__any_sync(0xffffffffu, want)) {
        const float m_new = fmaxf(tmax, m);
        if (j > 0) {
          const float f = (m == -INFINITY) ? 0.f : fast_exp2(m - m_new);
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(tO + c * 32, o);
          }
          l *= f;
        }
        m = m_new;
      }
      const float neg_m = (m == -INFINITY) ? 0.f : -m;
      float rs0 = 0.f, rs1 = 0.f, rs2 = 0.f, rs3 = 0.f;
      // pass 2: re-read S in halves, exponentiate, pack P (bf16 pairs, or
      // e4m3 quadruples) over the consumed columns
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t sa[64];
        {
          uint32_t(&c0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sa[0]);
          uint32_t(&c1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sa[32]);
          tmem_ld32(tS + h2 * 64, c0);
          tmem_ld32(tS + h2 * 64 + 32, c1);
          tmem_ld_wait();
        }
        if (masked) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (h2 * 64 + c > lim) sa[c] = __float_as_uint(-INFINITY);
        }
        if constexpr (F8) {
          // 64 keys -> 16 columns; the normaliser sums the unrounded values
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int k0 = 4 * c;
            const float p0 = fast_exp2(fmaf(__uint_as_float(sa[k0]), sc, neg_m));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sa[k0 + 1]), sc, neg_m));
            const float p2 = fast_exp2(fmaf(__uint_as_float(sa[k0 + 2]), sc, neg_m));
            const float p3 = fast_exp2(fmaf(__uint_as_float(sa[k0 + 3]), sc, neg_m));
            rs0 += p0;
            rs1 += p1;
            rs2 += p2;
            rs3 += p3;
            pk[c] = pack_e4m3x4(p0, p1, p2, p3);
          }
          tmem_st16(tS + h2 * 16, pk);
        } else {
#pragma unroll
          for (int q2 = 0; q2 < 2; ++q2) {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              const int k0 = q2 * 32 + 2 * c;
              const float p0 = fast_exp2(fmaf(__uint_as_float(sa[k0]), sc, neg_m));
              const float p1 = fast_exp2(fmaf(__uint_as_float(sa[k0 + 1]), sc, neg_m));
              const float p2 = fast_exp2(fmaf(__uint_as_float(sa[k0 + 2]), sc, neg_m));
              const float p3 = fast_exp2(fmaf(__uint_as_float(sa[k0 + 3]), sc, neg_m));
              rs0 += p0;
              rs1 += p1;
              rs2 += p2;
              rs3 += p3;
              pk[c] = pack_bf16x2(p0, p1);
              pk[c + 1] = pack_bf16x2(p2, p3);
            }
            tmem_st16(tS + h2 * 32 + q2 * 16, pk);
          }
        }
      }
      l += (rs0 + rs1) + (rs2 + rs3);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[X]);
    }
    const bool fin = __all_sync(0xffffffffu, ok && mbar_wait(o_final, 0, abort_flag, 0x333));
    // Stage O_X (fp32, 1/l applied) in the K/V ring, which is idle once the
    // last PV has completed: row r at [X][r][HD] with its 16-byte chunks
    // XOR-swizzled by (r & 7) so that both the row-per-thread writes and the
    // row-per-warp reads are bank-conflict free.  Then each warp writes whole
    // rows: coalesced stores instead of one 16-byte piece per row per lane.
    float* stage = reinterpret_cast<float*>(sK) + X * (BQ * HD);
    const int h = hX[X];
    float vs = 1.f;
    if constexpr (F8) vs = *p.v_scale;
    const float inv_l = (l > 0.f) ? vs / l : 0.f;
    const float lse_nat = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
    if (fin) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const int chunk = (c * 8 + v) ^ (r & 7);
          reinterpret_cast<float4*>(stage + r * HD)[chunk] =
              make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                          __uint_as_float(o[4 * v + 2]) * inv_l,
                          __uint_as_float(o[4 * v + 3]) * inv_l);
        }
      }
      if (qrow < p.Lq) {
        if (p.n_splits == 1) {
          if (p.lse) p.lse[(static_cast<size_t>(b) * p.Hq + h) * p.Lq + qrow] = lse_nat;
        } else {
          p.part_lse[((static_cast<size_t>(split) * p.B + b) * p.Hq + h) * p.Lq + qrow] = lse_nat;
        }
      }
    }
    // the four warps of this tile's warpgroup meet here (named barrier 1 + X)
    asm volatile("bar.sync %0, %1;" ::"r"(1 + X), "r"(BQ) : "memory");
    if (fin) {
      constexpr int CPR = HD / 4;  // 16-byte chunks per row
      for (int rr = quarter; rr < BQ; rr += 4) {
        const int qr = i0X[X] + rr;
        if (qr >= p.Lq) break;
        for (int cc = lane; cc < CPR; cc += 32) {
          const float4 v = reinterpret_cast<const float4*>(stage + rr * HD)[cc ^ (rr & 7)];
          uint2 w;
          w.x = pack_bf16x2(v.x, v.y);
          w.y = pack_bf16x2(v.z, v.w);
          if (p.n_splits == 1) {
            *reinterpret_cast<uint2*>(p.out + (static_cast<size_t>(b) * p.Lq + qr) * p.ldo +
                                      static_cast<size_t>(h) * HD + cc * 4) = w;
          } else {
            const size_t row =
                ((static_cast<size_t>(split) * p.B + b) * p.Hq + h) * p.Lq + qr;
            *reinterpret_cast<uint2*>(p.part_o + row * HD + cc * 4) = w;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Merge key-range splits: O = sum_s w_s O_s / sum_s w_s, w_s = exp(lse_s - max).
// One warp per (b, h, row), each lane owning HD / 32 consecutive values.
// Every split's log-sum-exp and partial row are requested before any
// arithmetic (a batch of COMBINE_BATCH splits in flight per lane), so a warp
// waits for memory once per batch; the sums run in split order (the bits do
// not depend on scheduling).  The register cap keeps three CTAs on an SM: the
// kernel is bound by how many loads are in flight, not by arithmetic.
constexpr int MAX_SPLITS = 32;
constexpr int COMBINE_THREADS = 256;

// acc[0..] += w * (the bf16 values of a lane's slice of a row)
__device__ __forceinline__ void add_weighted(float (&acc)[4], float w, uint2 v) {
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
  acc[0] = fmaf(w, __low2float(a), acc[0]);
  acc[1] = fmaf(w, __high2float(a), acc[1]);
  acc[2] = fmaf(w, __low2float(b), acc[2]);
  acc[3] = fmaf(w, __high2float(b), acc[3]);
}
__device__ __forceinline__ void add_weighted(float (&acc)[2], float w, uint32_t v) {
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v);
  acc[0] = fmaf(w, __low2float(a), acc[0]);
  acc[1] = fmaf(w, __high2float(a), acc[1]);
}
__device__ __forceinline__ uint2 pack_row(const float (&a)[4], float inv) {
  return make_uint2(pack_bf16x2(a[0] * inv, a[1] * inv), pack_bf16x2(a[2] * inv, a[3] * inv));
}
__device__ __forceinline__ uint32_t pack_row(const float (&a)[2], float inv) {
  return pack_bf16x2(a[0] * inv, a[1] * inv);
}
constexpr int COMBINE_BATCH = 12;

template <int HD>
__global__ void __launch_bounds__(COMBINE_THREADS, 3)
    attn_combine_kernel(const __nv_bfloat16* __restrict__ part_o,
                        const float* __restrict__ part_lse, int S, int B, int Hq, int Lq,
                        __nv_bfloat16* __restrict__ out, int ldo, float* __restrict__ lse) {
  constexpr int PER = HD / 32;  // values per lane: 4 (8 bytes) or 2 (4 bytes)
  using Vec = typename std::conditional<PER == 4, uint2, uint32_t>::type;
  griddep_launch();
  griddep_wait();
  const int row = (static_cast<int>(blockIdx.x) * COMBINE_THREADS +
                   static_cast<int>(threadIdx.x)) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = B * Hq * Lq;
  if (row >= rows) return;  // warp-uniform
  const size_t stride = static_cast<size_t>(rows);
  float mx = -INFINITY, wsum = 0.f;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  for (int s0 = 0; s0 < S; s0 += COMBINE_BATCH) {
    float ls[COMBINE_BATCH];
    Vec v[COMBINE_BATCH];
#pragma unroll
    for (int k = 0; k < COMBINE_BATCH; ++k) {
      const int sp = s0 + k;
      ls[k] = sp < S ? part_lse[sp * stride + row] : -INFINITY;
      v[k] = sp < S ? reinterpret_cast<const Vec*>(part_o + (sp * stride + row) * HD)[lane]
                    : Vec{};
    }
    float bmx = -INFINITY;
#pragma unroll
    for (int k = 0; k < COMBINE_BATCH; ++k) bmx = fmaxf(bmx, ls[k]);
    if (bmx > mx) {
      // rescale what earlier batches accumulated (exact for any reference)
      const float f = mx == -INFINITY ? 0.f : expf(mx - bmx);
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] *= f;
      wsum *= f;
      mx = bmx;
    }
#pragma unroll
    for (int k = 0; k < COMBINE_BATCH; ++k) {
      if (ls[k] == -INFINITY) continue;  // an empty split
      const float w = expf(ls[k] - mx);
      wsum += w;
      add_weighted(acc, w, v[k]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  const int qrow = row % Lq;
  const int bh = row / Lq;
  const int h = bh % Hq;
  const int b = bh / Hq;
  const Vec o = pack_row(acc, inv);
  reinterpret_cast<Vec*>(out + (static_cast<size_t>(b) * Lq + qrow) * ldo +
                         static_cast<size_t>(h) * HD)[lane] = o;
  if (lse && lane == 0) lse[row] = (wsum > 0.f) ? mx + logf(wsum) : -INFINITY;
}

}  // namespace attn
}  // namespace dg
