// sampler.cuh - the denoising sampler on the GPU.
//
// Per step (Google docs page "DiffusionGemma", table "Configuracao de exibicao
// recomendada": 48-step cap, linear 0.8 -> 0.4 temperature, adaptive stop on
// mean entropy + two identical predictions; aiexpert.news "Google's
// DiffusionGemma Atinge 1.000 Tokens por Segundo", architecture paragraph:
// confident tokens locked each pass, low-confidence ones re-noised):
//
//   rowpass   streams the fp32 logits once.  Each CTA reduces one chunk of one
//             position's vocabulary row to a partial: running max and the
//             two sums of the online softmax (for logsumexp and entropy), the
//             raw-logit argmax, and the best Gumbel-perturbed score.
//   commit    one CTA per sequence, one thread per canvas position: merges the
//             partials, ranks log confidences for the top-k commit, applies
//             re-noise / unselected policy / stop rule, updates the canvas.
//
// Arithmetic is done in the log2 domain: zl = l * log2(e) / T.  The Gumbel
// score in that domain is zl - log2(E), E = -ln(u), which orders exactly like
// z - ln(E).  Ties resolve to the lowest vocabulary index / position.
#pragma once

#include <type_traits>

#include "dg_common.cuh"

namespace dg {

constexpr uint32_t kTagGumbel = 0;
constexpr uint32_t kTagRenoise = 1;
constexpr uint32_t kTagInit = 2;

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): per round two 32x32->64
// multiplies by the Philox constants; the high halves are XORed with the other
// two counter words and the round key; the key is bumped by the Weyl constants.
__host__ __device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c.x;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c.z;
    const uint32_t hi0 = static_cast<uint32_t>(p0 >> 32), lo0 = static_cast<uint32_t>(p0);
    const uint32_t hi1 = static_cast<uint32_t>(p1 >> 32), lo1 = static_cast<uint32_t>(p1);
    c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
    k.x += 0x9E3779B9u;
    k.y += 0xBB67AE85u;
  }
  return c;
}

// The same generator with its ten round keys computed once by the caller
// (ks[2r], ks[2r+1] = the key after r Weyl bumps).
struct PhiloxKeys {
  uint32_t k[20];
  __device__ __forceinline__ explicit PhiloxKeys(uint2 key) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
      k[2 * r] = key.x;
      k[2 * r + 1] = key.y;
      key.x += 0x9E3779B9u;
      key.y += 0xBB67AE85u;
    }
  }
};
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, const PhiloxKeys& ks) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c.x;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c.z;
    const uint32_t hi0 = static_cast<uint32_t>(p0 >> 32), lo0 = static_cast<uint32_t>(p0);
    const uint32_t hi1 = static_cast<uint32_t>(p1 >> 32), lo1 = static_cast<uint32_t>(p1);
    c = make_uint4(hi1 ^ c.y ^ ks.k[2 * r], lo1, hi0 ^ c.w ^ ks.k[2 * r + 1], lo0);
  }
  return c;
}

__device__ __forceinline__ uint32_t position_word(uint32_t seed, uint32_t b, uint32_t block,
                                                  uint32_t step, uint32_t pos, uint32_t tag) {
  return philox4x32_10(make_uint4(0u, (pos & 0xFFFFFFu) | (tag << 24), step, block),
                       make_uint2(seed, b))
      .x;
}

__device__ __forceinline__ int32_t token_from_word(uint32_t r, int vocab) {
  return static_cast<int32_t>((static_cast<uint64_t>(r) * static_cast<uint32_t>(vocab)) >> 32);
}

__device__ __forceinline__ float sfu_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float sfu_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Exponential variate E = -ln(u) of the draw word r, u = (2 (r >> 9) + 1) 2^-24.
// u is built exactly from the bits: 1 + (r >> 9) 2^-23 is an fp32 in [1, 2), and
// subtracting 1 - 2^-24 (representable) is exact; w = 1 - u is exact too.
// Away from u = 1 the special-function log2 is accurate to ~2^-22 absolute, i.e.
// ~3e-6 relative in E for u <= 15/16.  For w = 1 - u <= 1/16 the series
// -ln(1 - w) = w + w^2/2 + ... + w^6/6 (truncation < 1e-8 relative) is used.
__device__ __forceinline__ float exp_variate(uint32_t r) {
  const float f = __uint_as_float(0x3F800000u | (r >> 9));
  const float u = f - 0.999999940395355224609375f;  // f - (1 - 2^-24)
  const float w = 1.0f - u;
  const float e_log = sfu_log2(u) * -0.693147180559945309f;
  const float e_ser =
      w * fmaf(w, fmaf(w, fmaf(w, fmaf(w, fmaf(w, 0.16666667f, 0.2f), 0.25f), 0.33333334f), 0.5f),
               1.0f);
  return w <= 0.0625f ? e_ser : e_log;
}

// u of the draw word r as in exp_variate (exact); E >= 1 - u.  The bits
// 0x3F800000 | (r >> 9) are formed as hi32(r * 2^23) + 0x3F800000 (the two
// fields do not overlap), one multiply-add instead of a shift and an OR.
__device__ __forceinline__ float draw_uniform(uint32_t r) {
  return __uint_as_float(__umulhi(r, 1u << 23) + 0x3F800000u) - 0.999999940395355224609375f;
}

__device__ __forceinline__ float step_temperature(int step, int max_steps, float t0, float t1) {
  if (max_steps <= 1) return t0;
  return t0 + (t1 - t0) * (static_cast<float>(step) / static_cast<float>(max_steps - 1));
}

struct RowPartial {
  float m;      // running max of zl
  float s;      // sum 2^(zl - m)
  float q;      // sum 2^(zl - m) (zl - m)
  float amax;   // max raw logit
  int aidx;     // its index (lowest on ties)
  float best;   // best Gumbel score, log2 domain
  int bidx;     // its index (lowest on ties)
  int pad;
};

// Row pass partial of the fused unembedding: as RowPartial, plus the raw
// logit of the Gumbel winner and of the current canvas token (NaN when that
// token lies outside the partial's vocabulary range).
struct FusedPartial {
  float m, s, q, amax;
  int aidx;
  float best;
  int bidx;
  float lx;
  float lcur;
  int pad;
};

// Merged per-position statistics that the commit step consumes.
struct RowStats {
  float lam;   // natural log confidence of the token at stake
  float ent;   // tempered entropy, nats
  int amax;    // raw-logit argmax
  int xhat;    // Gumbel-max sample
};

// Row pass state of one thread over an ascending run of vocabulary entries.
// Per element, in the log2 domain with m the running maximum:
//   pe = 2^(l k2 - m)         one FFMA + one ex2 (shared by the softmax sums)
//   E  = -ln(u)               Philox word -> exponential variate
// The Gumbel-max sample argmax_v (z_v - ln E_v) equals argmax_v pe_v / E_v (the
// exponential race), so the best is kept as (pb, Eb) and compared by
// cross-multiplication; pb rescales with the running maximum.  It becomes the
// score l k2 - log2(E) only for the merges.
struct RowState {
  float m, s, q;        // running max of zl, sum 2^(zl - m), sum 2^(zl - m) (zl - m)
  float amax;           // max raw logit
  int aidx;             // its index (lowest on ties)
  float pb, eb, lb;     // race leader: pe, E, raw logit
  int bidx;             // its index (lowest on ties)
  float lcur;           // raw logit of the current token, NaN until seen

  __device__ __forceinline__ void reset() {
    m = -INFINITY; s = 0.f; q = 0.f;
    amax = -INFINITY; aidx = 0x7FFFFFFF;
    pb = 0.f; eb = 1.f; lb = -INFINITY; bidx = 0x7FFFFFFF;
    lcur = __int_as_float(0x7FC00000);
  }

  // G groups of 4 consecutive entries, group g starting at vg[g] (a multiple
  // of 4, ascending in g); only groups [0, n_valid) are counted (the others
  // hold -inf).  The Philox words of group g are counter (vg[g] / 4, c1, step,
  // block), key `key`.
  template <int G, bool TRACK_CUR>
  __device__ __forceinline__ void update(const float (&l)[4 * G], const int (&vg)[G],
                                         int n_valid, int cur, float k2, uint32_t c1,
                                         uint32_t step, uint32_t block, uint2 key) {
    float bm = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4 * G; ++i) bm = fmaxf(bm, l[i]);
    if (bm > amax) {
      // new raw maximum in this batch: first index holding it (ascending order)
      amax = bm;
#pragma unroll
      for (int g = G - 1; g >= 0; --g)
#pragma unroll
        for (int e = 3; e >= 0; --e)
          if (l[4 * g + e] == bm) aidx = vg[g] + e;
    }
    const float bmz = bm * k2;
    if (bmz > m) {
      if (m != -INFINITY) {
        const float d = m - bmz, f = sfu_exp2(d);
        q = f * (q + d * s);
        s *= f;
        pb *= f;
      }
      m = bmz;
    }
    const float neg_m = -m;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (g >= n_valid) break;
      const uint4 r = philox4x32_10(
          make_uint4(static_cast<uint32_t>(vg[g] >> 2), c1, step, block), key);
      const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lv = l[4 * g + e];
        const float t = fmaf(lv, k2, neg_m);
        const float pe = sfu_exp2(t);
        s += pe;
        q = fmaf(pe, t, q);
        // E >= 1 - u: when pe eb <= pb (1 - u) the race step below cannot take
        // the lead, so the variate is only computed for entries that might
        // (the outcome is bit for bit that of the plain race)
        const float lhs = pe * eb;
        if (lhs > fmaf(-pb, draw_uniform(rw[e]), pb)) {
          const float ev = exp_variate(rw[e]);
          if (lhs > pb * ev) {
            pb = pe;
            eb = ev;
            lb = lv;
            bidx = vg[g] + e;
          }
        }
        if (TRACK_CUR && vg[g] + e == cur) lcur = lv;
      }
    }
  }

  // 32 consecutive entries starting at v0 (a multiple of 4)
  __device__ __forceinline__ void update32(const float (&l)[32], int v0, int cur, float k2,
                                           uint32_t c1, uint32_t step, uint32_t block,
                                           uint2 key) {
    int vg[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) vg[g] = v0 + 4 * g;
    update<8, true>(l, vg, 8, cur, k2, c1, step, block, key);
  }

  __device__ __forceinline__ float best_score(float k2) const {
    return (bidx == 0x7FFFFFFF) ? -INFINITY : lb * k2 - sfu_log2(eb);
  }

  __device__ __forceinline__ FusedPartial partial(float k2) const {
    return FusedPartial{m, s, q, amax, aidx, best_score(k2), bidx, lb, lcur, 0};
  }
};

struct SampleParams {
  int B, C, V;
  int chunk, nchunk;         // vocabulary chunk per rowpass CTA
  uint32_t seed;
  int block;
  const int32_t* step_ptr;   // device step index, or null: use step_val
  int step_val;
  int max_steps;
  float t_start, t_end;
  int commit_k;
  float log_tau;             // ln(renoise_conf), -inf disables re-noise
  float stop_entropy;
  int policy;
  int selection;             // 0: top commit_k by confidence, 1: entropy-bounded
  float entropy_bound;
  int32_t* near_ties;        // optional [B, 3] decision counters (sample_commit_kernel)
};

// A decision whose deciding quantity lies within this distance (log space,
// nats) of flipping is counted as a near-tie.
constexpr float kNearTieMargin = 1e-4f;

__device__ __forceinline__ int read_step(const SampleParams& p) {
  return p.step_ptr ? *p.step_ptr : p.step_val;
}

__device__ __forceinline__ void merge_softmax(float& m, float& s, float& q, float m2, float s2,
                                              float q2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2; s = s2; q = q2;
    return;
  }
  if (m2 > m) {
    const float d = m - m2, f = exp2f(d);
    q = f * (q + d * s) + q2;
    s = f * s + s2;
    m = m2;
  } else {
    const float d = m2 - m, f = exp2f(d);
    q = q + f * (q2 + d * s2);
    s = s + f * s2;
  }
}

__device__ __forceinline__ void merge_best(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) {
    v = v2;
    i = i2;
  }
}

// Grid: B * C * nchunk CTAs of RP_THREADS threads.  Chunk length is a multiple
// of 4.  The chunk streams through a ring of RP_STAGES shared-memory batches of
// RP_THREADS * 16 entries, filled by bulk async copies (thread 0 keeps the
// next RP_STAGES - 1 batches in flight while the CTA works on one); thread t takes the
// float4 groups at t*4 + u*RP_THREADS*4, u < 4, so each thread meets its
// entries in ascending order.
//
// Every entry enters the softmax sums (one FFMA and one ex2 against the
// thread's running maximum m).  Few can win the Gumbel race, and two exact
// bounds on the exponential variate E = -ln(u) of an entry's draw word keep
// the rest out of it:
//   * E >= w = 1 - u (exact from the word's bits): with S the best race score
//     known to the warp (log2 units, a real entry's), an entry whose
//     2^(zl - m) < 2^(S - m - kTieSlack) w cannot beat that entry, so its
//     variate and race step are skipped;
//   * E >= E_min ~ 2^-24 for every word: a group of four whose largest zl lies
//     more than kRaceSlack below S cannot win whatever its draws; when no lane
//     of the warp holds such a group, its Philox block is skipped too.
// S is shared across the CTA through an order-preserving integer max, read
// without a barrier (a stale value is only a weaker bound), after batches
// 0, 1, 3, 7, ... .  When every group of a batch needs its Philox block, the
// four blocks run as one straight-line piece (four independent round chains).
// The race keeps (pe, E) of the leader; its score is log2(pe) + m - log2(E).
constexpr int RP_THREADS = 256;
constexpr int RP_CTAS_PER_SM = 4;   // resident CTAs per SM, guaranteed by the launch bounds
constexpr int RP_STAGES = 3;
constexpr int RP_BATCH = RP_THREADS * 16;              // entries per batch (16 KB)
constexpr int RP_SMEM = RP_STAGES * RP_BATCH * 4;       // dynamic shared memory
constexpr float kRaceSlack = 24.5f;   // > -log2(E_min) = 24
constexpr float kTieSlack = 1e-3f;    // far above the rounding of a score

__device__ __forceinline__ int ordered_bits(float f) {
  const int b = __float_as_int(f);
  return b ^ ((b >> 31) & 0x7FFFFFFF);
}
__device__ __forceinline__ float ordered_float(int k) {
  return __int_as_float(k ^ ((k >> 31) & 0x7FFFFFFF));
}


// any = any || (a >= b), one comparison with a predicate operand.
__device__ __forceinline__ bool ge_or(float a, float b, bool any) {
  uint32_t r;
  asm("{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %3, 0;\n\t"
      "setp.ge.or.f32 po, %1, %2, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "r"(static_cast<uint32_t>(any)));
  return r != 0;
}

__global__ void __launch_bounds__(RP_THREADS, RP_CTAS_PER_SM) sample_rowpass_kernel(
    const float* __restrict__ logits, const int32_t* __restrict__ seq_status, SampleParams p,
    RowPartial* __restrict__ part) {
  griddep_wait();
  griddep_launch();
  extern __shared__ __align__(128) uint8_t rp_smem[];
  float* ring = reinterpret_cast<float*>(rp_smem);  // [RP_STAGES][RP_BATCH]
  __shared__ uint64_t full_bar[RP_STAGES], empty_bar[RP_STAGES];
  __shared__ int s_best;  // the CTA's best race score so far, ordered bits
  __shared__ int s_abort;
  const int row = blockIdx.x / p.nchunk;
  const int ck = blockIdx.x - row * p.nchunk;
  const int b = row / p.C;
  const int pos = row - b * p.C;
  if (seq_status[b] != 0) return;
  const int step = read_step(p);
  const float T = step_temperature(step, p.max_steps, p.t_start, p.t_end);
  const float k2 = 1.4426950408889634f / T;  // log2(e) / T
  const float* x = logits + static_cast<size_t>(row) * p.V;
  const int v0 = ck * p.chunk;
  const int v1 = min(p.V, v0 + p.chunk);
  const uint32_t c1 = (static_cast<uint32_t>(pos) & 0xFFFFFFu) | (kTagGumbel << 24);
  const PhiloxKeys keys(make_uint2(p.seed, static_cast<uint32_t>(b)));
  const int lane = threadIdx.x & 31;
  const int nb = (v1 - v0 + RP_BATCH - 1) / RP_BATCH;
  if (threadIdx.x == 0) {
    s_best = ordered_bits(-INFINITY);
    s_abort = 0;
    for (int st = 0; st < RP_STAGES; ++st) {
      mbar_init(&full_bar[st], 1);
      mbar_init(&empty_bar[st], RP_THREADS / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();
  int issued = 0;  // batches requested (thread 0)
  auto issue = [&](int bt) {
    const int st = bt % RP_STAGES;
    const int bs = v0 + bt * RP_BATCH;
    const uint32_t bytes = static_cast<uint32_t>(min(RP_BATCH, v1 - bs)) * 4u;
    mbar_expect_tx(&full_bar[st], bytes);
    bulk_load(ring + st * RP_BATCH, x + bs, bytes, &full_bar[st]);
    issued = bt + 1;
  };
  if (threadIdx.x == 0)
    for (int bt = 0; bt < min(RP_STAGES, nb); ++bt) issue(bt);

  float m = -INFINITY, s = 0.f, q = 0.f;     // this thread's running max of zl and sums
  float amax = -INFINITY;
  int aidx = 0x7FFFFFFF;
  float pb = 0.f, eb = 1.f;                  // race leader of this thread: pe, E
  int bidx = 0x7FFFFFFF;
  auto leader_score = [&]() {
    return (bidx == 0x7FFFFFFF || pb == 0.f) ? -INFINITY : sfu_log2(pb) + m - sfu_log2(eb);
  };
  float S = -INFINITY;                       // best score known to the warp (log2 units)
  float theta = 0.f;                         // 2^(S - m - kTieSlack), this thread's m

  // One batch; PAD: the batch runs past v1 (only the last one can), whose
  // missing entries read as -inf.  There the exponent is clamped at -256
  // (where ex2 is 0 already) so that a missing entry adds 0 to both sums.
  auto batch = [&](int bt, int bstart, auto pad_tag) {
    constexpr bool PAD = decltype(pad_tag)::value;
    const int st = bt % RP_STAGES;
    // thread 0 refills the stage read one batch ago, once every warp has read it
    if (threadIdx.x == 0 && bt >= 1 && bt - 1 + RP_STAGES < nb) {
      const int sp = (bt - 1) % RP_STAGES;
      mbar_wait(&empty_bar[sp], ((bt - 1) / RP_STAGES) & 1, &s_abort, 0x611);
      issue(bt - 1 + RP_STAGES);
    }
    mbar_wait(&full_bar[st], (bt / RP_STAGES) & 1, &s_abort, 0x612);
    const float4* src = reinterpret_cast<const float4*>(ring + st * RP_BATCH);
    float l[16];
    int vg[4];
    float gmax[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = bstart + u * RP_THREADS * 4 + threadIdx.x * 4;
      vg[u] = v;
      const float4 l4 = (!PAD || v < v1)
                            ? src[u * RP_THREADS + threadIdx.x]
                            : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      l[4 * u] = l4.x;
      l[4 * u + 1] = l4.y;
      l[4 * u + 2] = l4.z;
      l[4 * u + 3] = l4.w;
      gmax[u] = fmaxf(fmaxf(l4.x, l4.y), fmaxf(l4.z, l4.w));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[st]);
    const float bm = fmaxf(fmaxf(gmax[0], gmax[1]), fmaxf(gmax[2], gmax[3]));
    if (bm > amax) {
      // new raw maximum in this batch: first index holding it (ascending
      // order): the first group holding it, then the first entry of that group
      amax = bm;
      float4 g4 = make_float4(l[12], l[13], l[14], l[15]);
      int gv = vg[3];
#pragma unroll
      for (int u = 2; u >= 0; --u) {
        if (gmax[u] == bm) {
          g4 = make_float4(l[4 * u], l[4 * u + 1], l[4 * u + 2], l[4 * u + 3]);
          gv = vg[u];
        }
      }
      aidx = gv + (g4.x == bm ? 0 : g4.y == bm ? 1 : g4.z == bm ? 2 : 3);
    }
    const float bmz = bm * k2;
    if (bmz > m) {
      if (m != -INFINITY) {
        const float d = m - bmz, f = sfu_exp2(d);
        q = f * (q + d * s);
        s *= f;
        pb *= f;
        theta *= f;
      }
      m = bmz;
    }
    const float neg_m = (PAD && m == -INFINITY) ? 0.f : -m;
    float pe[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float t = fmaf(l[i], k2, neg_m);
      if (PAD) t = fmaxf(t, -256.f);
      pe[i] = sfu_exp2(t);
      s += pe[i];
      q = fmaf(pe[i], t, q);
    }
    const float thr = S - kRaceSlack;
    bool cand[4];
    unsigned need = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      cand[u] = (!PAD || vg[u] < v1) && gmax[u] * k2 >= thr;
      if (__any_sync(0xffffffffu, cand[u])) need |= 1u << u;
    }
    if (need != 0) {
      uint32_t rw[16];
      auto draw = [&](int u) {
        const uint4 r = philox4x32_10(
            make_uint4(static_cast<uint32_t>(vg[u] >> 2), c1, static_cast<uint32_t>(step),
                       static_cast<uint32_t>(p.block)), keys);
        rw[4 * u] = r.x;
        rw[4 * u + 1] = r.y;
        rw[4 * u + 2] = r.z;
        rw[4 * u + 3] = r.w;
      };
      if (need == 0xFu) {
#pragma unroll
        for (int u = 0; u < 4; ++u) draw(u);
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (need & (1u << u)) {
            draw(u);
          } else {
            rw[4 * u] = rw[4 * u + 1] = rw[4 * u + 2] = rw[4 * u + 3] = 0u;
          }
        }
      }
      // pe < theta (1 - u) <= theta E: the entry cannot beat the best known one.
      // The test is exact on its own, so it runs on every entry of the batch: a
      // group whose block was skipped has words 0 (u = 2^-24, bound ~ theta),
      // and its entries, more than 24.5 below S, lie far under that bound.
      float bound[16];
      bool any = false;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        bound[i] = fmaf(-theta, draw_uniform(rw[i]), theta);
        any = ge_or(pe[i], bound[i], any);
      }
      if (__any_sync(0xffffffffu, any)) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (!(pe[i] >= bound[i])) continue;
          const float ev = exp_variate(rw[i]);
          if (pe[i] * eb > pb * ev) {
            pb = pe[i];
            eb = ev;
            bidx = vg[i >> 2] + (i & 3);
          }
        }
      }
    }
    if ((bt & (bt + 1)) == 0) {
      // share the best score: this warp's, then the CTA's
      float sc = leader_score();
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, o));
      if (lane == 0 && sc > S) atomicMax(&s_best, ordered_bits(sc));
      const float cta = ordered_float(*reinterpret_cast<volatile int*>(&s_best));
      const float s_new = fmaxf(fmaxf(S, sc), __shfl_sync(0xffffffffu, cta, 0));
      if (s_new > S) {
        S = s_new;
        theta = sfu_exp2(S - m - kTieSlack);
      }
    }
  };
  const int nfull = (v1 - v0) / (RP_THREADS * 16);
  for (int bt = 0; bt < nfull; ++bt) batch(bt, v0 + bt * RP_THREADS * 16, std::false_type{});
  if (v0 + nfull * RP_THREADS * 16 < v1)
    batch(nfull, v0 + nfull * RP_THREADS * 16, std::true_type{});
  if (threadIdx.x == 0 && s_abort) {
    // a wait gave up: let every requested copy land before the CTA exits
    for (int bt = max(0, issued - RP_STAGES); bt < issued; ++bt)
      mbar_wait(&full_bar[bt % RP_STAGES], (bt / RP_STAGES) & 1, nullptr, 0x613);
  }
  float best = leader_score();

  // CTA reduction: warp shuffles, then across warps through shared memory.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const float q2 = __shfl_xor_sync(0xffffffffu, q, o);
    merge_softmax(m, s, q, m2, s2, q2);
    const float a2 = __shfl_xor_sync(0xffffffffu, amax, o);
    const int ai2 = __shfl_xor_sync(0xffffffffu, aidx, o);
    merge_best(amax, aidx, a2, ai2);
    const float b2 = __shfl_xor_sync(0xffffffffu, best, o);
    const int bi2 = __shfl_xor_sync(0xffffffffu, bidx, o);
    merge_best(best, bidx, b2, bi2);
  }
  __shared__ RowPartial red[RP_THREADS / 32];
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = RowPartial{m, s, q, amax, aidx, best, bidx, 0};
  __syncthreads();
  if (threadIdx.x == 0) {
    RowPartial r = red[0];
    for (int i = 1; i < RP_THREADS / 32; ++i) {
      merge_softmax(r.m, r.s, r.q, red[i].m, red[i].s, red[i].q);
      merge_best(r.amax, r.aidx, red[i].amax, red[i].aidx);
      merge_best(r.best, r.bidx, red[i].best, red[i].bidx);
    }
    part[blockIdx.x] = r;
  }
}

// Merge of the fused unembedding's partials: one warp per position.  Lane j
// merges partials j, j + 32, ... in order, then lanes merge pairwise (xor
// pattern) and lane 0's result is used, so the order is fixed.
constexpr int MERGE_WARPS = 8;

__global__ void __launch_bounds__(MERGE_WARPS * 32) sample_merge_kernel(
    const FusedPartial* __restrict__ part, int nparts, const uint8_t* __restrict__ committed,
    SampleParams p, RowStats* __restrict__ stats) {
  griddep_wait();
  griddep_launch();
  const int row = blockIdx.x * MERGE_WARPS + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.B * p.C) return;  // warp-uniform
  const int step = read_step(p);
  const float k2 = 1.4426950408889634f / step_temperature(step, p.max_steps, p.t_start, p.t_end);
  const FusedPartial* pr = part + static_cast<size_t>(row) * nparts;
  float m = -INFINITY, s = 0.f, q = 0.f, av = -INFINITY, bv = -INFINITY;
  float lx = 0.f, lcur = __int_as_float(0x7FC00000);
  int ai = 0x7FFFFFFF, bi = 0x7FFFFFFF;
  for (int j = lane; j < nparts; j += 32) {
    const FusedPartial f = pr[j];
    merge_softmax(m, s, q, f.m, f.s, f.q);
    merge_best(av, ai, f.amax, f.aidx);
    const int b_before = bi;
    merge_best(bv, bi, f.best, f.bidx);
    if (bi != b_before) lx = f.lx;
    if (!isnan(f.lcur)) lcur = f.lcur;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const float q2 = __shfl_xor_sync(0xffffffffu, q, o);
    merge_softmax(m, s, q, m2, s2, q2);
    const float a2 = __shfl_xor_sync(0xffffffffu, av, o);
    const int ai2 = __shfl_xor_sync(0xffffffffu, ai, o);
    merge_best(av, ai, a2, ai2);
    const float b2 = __shfl_xor_sync(0xffffffffu, bv, o);
    const int bi2 = __shfl_xor_sync(0xffffffffu, bi, o);
    const float lx2 = __shfl_xor_sync(0xffffffffu, lx, o);
    const int b_before = bi;
    merge_best(bv, bi, b2, bi2);
    if (bi != b_before) lx = lx2;
    const float lc2 = __shfl_xor_sync(0xffffffffu, lcur, o);
    if (isnan(lcur)) lcur = lc2;
  }
  if (lane == 0) {
    const float l2s = log2f(s);
    const float lse2 = m + l2s;  // log2-domain logsumexp
    float lat = lx;
    if (committed[row] != 0) {
      lat = lcur;
      if (isnan(lcur)) {  // the current token is not a vocabulary entry
        raise_error(ERR_CHECK | 0x502, static_cast<uint32_t>(row));
        lat = lse2 / k2;
      }
    }
    stats[row] = RowStats{(lat * k2 - lse2) * 0.69314718055994531f,
                          0.69314718055994531f * (l2s - q / s), ai, bi};
  }
}

// Grid: B CTAs; blockDim = C rounded up to a multiple of 32 (C <= 1024).
// Per-position statistics come either from the row pass partials (`part`,
// nchunk per position, and the logit at stake read from `logits`) or, when
// `stats` is given, from the fused unembedding's merged statistics.
__global__ void __launch_bounds__(1024) sample_commit_kernel(
    const float* __restrict__ logits, const RowPartial* __restrict__ part,
    const RowStats* __restrict__ stats, SampleParams p,
    int32_t* __restrict__ tok, uint8_t* __restrict__ committed, int32_t* __restrict__ prev_argmax,
    int32_t* __restrict__ seq_status, int32_t* __restrict__ o_xhat,
    int32_t* __restrict__ o_argmax, float* __restrict__ o_logconf,
    float* __restrict__ o_entropy, uint8_t* __restrict__ o_flags) {
  __shared__ float s_lam[1024];
  __shared__ float s_ent[1024];
  __shared__ uint8_t s_unc[1024];
  __shared__ float s_red[32];
  __shared__ int s_flag;
  __shared__ float s_mean_h;
  __shared__ float s_cut[2];    // selection key (confidence, or entropy) at ranks k - 1 and k
  __shared__ double s_csum[2];  // entropy-bounded: entropies summed through those ranks

  griddep_wait();
  griddep_launch();
  const int b = blockIdx.x;
  if (seq_status[b] != 0) return;
  const int i = threadIdx.x;
  const bool live = i < p.C;
  const int step = read_step(p);
  const float T = step_temperature(step, p.max_steps, p.t_start, p.t_end);
  const float k2 = 1.4426950408889634f / T;
  const size_t row = static_cast<size_t>(b) * p.C + i;

  float lam = 0.f, ent = 0.f;
  int amax_i = -1, xhat = 0, cur = 0;
  bool was_committed = true;
  if (live && stats != nullptr) {
    const RowStats rs = stats[row];
    lam = rs.lam;
    ent = rs.ent;
    amax_i = rs.amax;
    xhat = rs.xhat;
    cur = tok[row];
    was_committed = committed[row] != 0;
  } else if (live) {
    const RowPartial* pr = part + row * p.nchunk;
    float m = pr[0].m, s = pr[0].s, q = pr[0].q, av = pr[0].amax, bv = pr[0].best;
    int ai = pr[0].aidx, bi = pr[0].bidx;
    for (int c = 1; c < p.nchunk; ++c) {
      merge_softmax(m, s, q, pr[c].m, pr[c].s, pr[c].q);
      merge_best(av, ai, pr[c].amax, pr[c].aidx);
      merge_best(bv, bi, pr[c].best, pr[c].bidx);
    }
    const float l2s = log2f(s);
    const float lse2 = m + l2s;                          // log2-domain logsumexp
    ent = 0.69314718055994531f * (l2s - q / s);           // nats
    amax_i = ai;
    xhat = bi;
    cur = tok[row];
    was_committed = committed[row] != 0;
    int x = was_committed ? cur : xhat;
    if (x < 0 || x >= p.V) {
      raise_error(ERR_CHECK | 0x501, static_cast<uint32_t>(row));
      x = 0;
    }
    const float zl = logits[row * p.V + x] * k2;
    lam = (zl - lse2) * 0.69314718055994531f;             // natural log confidence
  }

  // mean entropy (fixed-order reduction), same-prediction test, uncommitted count
  float hs = live ? ent : 0.f;
  hs = warp_sum(hs);
  if ((i & 31) == 0) s_red[i >> 5] = hs;
  const bool same = !live || (amax_i == prev_argmax[live ? row : 0]);
  const int all_same = __syncthreads_and(same);
  const int n_unc = __syncthreads_count(live && !was_committed);
  if (i == 0) {
    float tot = 0.f;
    for (int w = 0; w < (blockDim.x + 31) / 32; ++w) tot += s_red[w];
    const float mean_h = tot / static_cast<float>(p.C);
    const bool crit = (mean_h < p.stop_entropy) && step >= 1 && all_same;
    const bool cap = step >= p.max_steps - 1;
    s_flag = (crit || cap) ? 1 : 0;
    s_mean_h = mean_h;
    s_cut[0] = s_cut[1] = 0.f;
    s_csum[0] = s_csum[1] = 0.0;
  }
  if (live) {
    s_lam[i] = lam;
    s_ent[i] = ent;
    s_unc[i] = was_committed ? 0 : 1;
  }
  __syncthreads();
  const bool final_step = s_flag != 0;

  bool selected = false;
  int rank = -1;       // rank among the uncommitted positions, in selection order
  double csum = 0.0;   // entropy-bounded: the entropies summed through this rank
  if (live && !was_committed && p.selection == 1) {
    // entropy-bounded: rank by (entropy, position) among the uncommitted; the
    // selection is the ranked prefix whose entropies sum to <= the bound, and
    // at least rank 0 (the sum is taken in fp64: order-independent)
    rank = 0;
    csum = static_cast<double>(ent);
    for (int j = 0; j < p.C; ++j) {
      if (s_unc[j] && j != i) {
        const float ej = s_ent[j];
        if (ej < ent || (ej == ent && j < i)) {
          ++rank;
          csum += static_cast<double>(ej);
        }
      }
    }
    selected = rank == 0 || csum <= static_cast<double>(p.entropy_bound);
  } else if (live && !was_committed) {
    // top-k among uncommitted: rank = number of uncommitted positions that beat this one
    const int k = min(p.commit_k, n_unc);
    rank = 0;
    for (int j = 0; j < p.C; ++j) {
      if (s_unc[j]) {
        const float lj = s_lam[j];
        rank += (lj > lam || (lj == lam && j < i)) ? 1 : 0;
      }
    }
    selected = rank < k;
  }

  if (p.near_ties != nullptr) {
    // Decisions within kNearTieMargin of flipping, per sequence:
    // [0] positions at the commit cut: the keys on either side of the cut
    //     nearly tie (then the uncommitted positions near the cut count), or,
    //     entropy-bounded, a sum through the cut nearly meets the bound;
    // [1] committed positions whose confidence is near the re-noise threshold;
    // [2] 1 when the mean entropy is near the stop threshold.
    const float m = kNearTieMargin;
    const int n_sel = __syncthreads_count(selected);
    const float key = p.selection == 1 ? ent : lam;
    if (rank >= 0 && rank == n_sel - 1) { s_cut[0] = key; s_csum[0] = csum; }
    if (rank >= 0 && rank == n_sel) { s_cut[1] = key; s_csum[1] = csum; }
    __syncthreads();
    const double bound = static_cast<double>(p.entropy_bound);
    bool cut = false;
    float edge = 0.f;
    if (n_sel > 0 && n_sel < n_unc) {
      if (p.selection == 1) {
        cut = fabs(s_csum[1] - bound) < m || fabs(s_csum[0] - bound) < m ||
              (s_cut[1] - s_cut[0]) < m;
      } else {
        cut = (s_cut[0] - s_cut[1]) < m;
        edge = 0.5f * (s_cut[0] + s_cut[1]);
      }
    } else if (p.selection == 1 && n_sel > 1 && n_sel == n_unc) {
      cut = fabs(s_csum[0] - bound) < m;  // all selected, the sum just under the bound
    }
    bool at_cut = false;
    if (cut && rank >= 0) {
      at_cut = p.selection == 1 ? (rank == n_sel - 1 || (n_sel < n_unc && rank == n_sel))
                                : fabsf(lam - edge) < m;
    }
    const int n_cut = __syncthreads_count(at_cut);
    const int n_ren = __syncthreads_count(live && was_committed && fabsf(lam - p.log_tau) < m);
    if (i == 0) {
      p.near_ties[b * 3 + 0] = n_cut;
      p.near_ties[b * 3 + 1] = n_ren;
      p.near_ties[b * 3 + 2] = fabsf(s_mean_h - p.stop_entropy) < m ? 1 : 0;
    }
  }

  int new_tok = cur;
  bool new_comm = was_committed;
  uint8_t flags = 0;
  if (live) {
    if (final_step) {
      if (!was_committed) {
        new_tok = xhat;
        flags |= 1;
      }
      new_comm = true;
    } else if (selected) {
      new_tok = xhat;
      new_comm = true;
      flags |= 1;
    } else if (was_committed) {
      if (lam < p.log_tau) {
        new_tok = token_from_word(
            position_word(p.seed, b, p.block, step, i, kTagRenoise), p.V);
        new_comm = false;
        flags |= 2;
      }
    } else {
      new_tok = (p.policy == 0) ? xhat
                                : token_from_word(position_word(p.seed, b, p.block, step, i,
                                                                kTagRenoise),
                                                  p.V);
    }
    tok[row] = new_tok;
    committed[row] = new_comm ? 1 : 0;
    prev_argmax[row] = amax_i;
    if (o_xhat) o_xhat[row] = xhat;
    if (o_argmax) o_argmax[row] = amax_i;
    if (o_logconf) o_logconf[row] = lam;
    if (o_entropy) o_entropy[row] = ent;
    if (o_flags) o_flags[row] = flags;
  }
  const int all_comm = __syncthreads_and(!live || new_comm);
  if (i == 0 && (final_step || all_comm)) seq_status[b] = step + 1;
}

// Fresh canvas: uniform tokens (tag INIT), nothing committed, no prediction yet.
__global__ void init_canvas_kernel(int B, int C, int V, uint32_t seed, int block,
                                   int32_t* __restrict__ tok, uint8_t* __restrict__ committed,
                                   int32_t* __restrict__ prev_argmax,
                                   int32_t* __restrict__ seq_status, int32_t* __restrict__ step) {
  const int b = blockIdx.x;
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    const size_t row = static_cast<size_t>(b) * C + i;
    tok[row] = token_from_word(position_word(seed, b, block, 0, i, kTagInit), V);
    committed[row] = 0;
    prev_argmax[row] = -1;
  }
  if (threadIdx.x == 0) seq_status[b] = 0;
  if (b == 0 && threadIdx.x == 0 && step) *step = 0;
}

// After a step: advance the step counter and publish whether any sequence runs on.
__global__ void step_advance_kernel(int B, int max_steps, const int32_t* __restrict__ seq_status,
                                    int32_t* __restrict__ step, int32_t* __restrict__ running) {
  int n = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) n += (seq_status[b] == 0) ? 1 : 0;
  n = __syncthreads_count(n > 0);
  if (threadIdx.x == 0) {
    const int s = *step + 1;
    *step = s;
    *running = (n > 0 && s < max_steps) ? 1 : 0;
  }
}

__global__ void philox_kernel(const uint32_t* __restrict__ in, uint32_t* __restrict__ out,
                              int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t* a = in + static_cast<size_t>(i) * 6;
  const uint4 r = philox4x32_10(make_uint4(a[0], a[1], a[2], a[3]), make_uint2(a[4], a[5]));
  uint32_t* o = out + static_cast<size_t>(i) * 4;
  o[0] = r.x;
  o[1] = r.y;
  o[2] = r.z;
  o[3] = r.w;
}

}  // namespace dg
