// kvcommit.cuh - append a finished block's K/V to the per-layer caches.
//
// "DiffusionGemma Guia do Desenvolvedor ...", Denoising bullet: when the
// 256-token block is finished it is committed to the KV cache and the next
// block starts (aiexpert.news architecture paragraph: each fully denoised
// block is committed and a new canvas is conditioned on the history).
//
// Pure data movement: 16-byte vectors (8 bf16) from the token-major block K/V
// [B, C, ld] into the head-major cache [B, Hkv, lmax, hd] at rows
// cache_len[b] + t.  A second one-CTA kernel then bumps cache_len, so every
// copy reads the same base row.
#pragma once

#include "dg_common.cuh"

namespace dg {

constexpr int KV_MAX_LAYERS = 64;

struct KVTables {
  const __nv_bfloat16* k_blk[KV_MAX_LAYERS];
  const __nv_bfloat16* v_blk[KV_MAX_LAYERS];
  __nv_bfloat16* k_cache[KV_MAX_LAYERS];
  __nv_bfloat16* v_cache[KV_MAX_LAYERS];
};

struct KVParams {
  int n_layers, B, Hkv, C, hd, lmax, ld_blk;
  const int32_t* cache_len;
};

constexpr int KV_THREADS = 256;
constexpr int KV_UNROLL = 4;

// Grid: y = one row group (layer, K or V, sequence, kv head), x strides over
// its C * hd / 8 vectors.  Within a row group the destination rows
// [cache_len, cache_len + C) are one contiguous run of the head-major cache
// and each source token row is hd contiguous elements, so consecutive threads
// move consecutive 16-byte vectors; the index arithmetic is one shift and one
// mask per vector (hd is 64 or 128).
__global__ void __launch_bounds__(KV_THREADS) kv_commit_kernel(const __grid_constant__ KVTables tab,
                                                               KVParams p) {
  int y = blockIdx.y;
  const int g = y % p.Hkv;
  y /= p.Hkv;
  const int b = y % p.B;
  y /= p.B;
  const int which = y & 1;
  const int l = y >> 1;
  const int base = p.cache_len[b];
  if (base < 0 || base + p.C > p.lmax) {
    if (blockIdx.x == 0 && threadIdx.x == 0 && g == 0 && which == 0 && l == 0)
      raise_error(ERR_CHECK | 0x401, static_cast<uint32_t>(b));
    return;
  }
  const int shift = p.hd == 128 ? 4 : 3;  // log2(hd / 8)
  const int nvec = p.C << shift;
  const __nv_bfloat16* src = (which == 0 ? tab.k_blk[l] : tab.v_blk[l]) +
                             static_cast<size_t>(b) * p.C * p.ld_blk +
                             static_cast<size_t>(g) * p.hd;
  __nv_bfloat16* dst = (which == 0 ? tab.k_cache[l] : tab.v_cache[l]) +
                       ((static_cast<size_t>(b) * p.Hkv + g) * p.lmax + base) * p.hd;
  // KV_UNROLL loads in flight per thread before their stores
  const int stride = gridDim.x * KV_THREADS;
  for (int i0 = blockIdx.x * KV_THREADS + threadIdx.x; i0 < nvec; i0 += KV_UNROLL * stride) {
    uint4 val[KV_UNROLL];
#pragma unroll
    for (int u = 0; u < KV_UNROLL; ++u) {
      const int i = i0 + u * stride;
      if (i < nvec)
        val[u] = __ldg(reinterpret_cast<const uint4*>(
            src + static_cast<size_t>(i >> shift) * p.ld_blk + (i & ((1 << shift) - 1)) * 8));
    }
#pragma unroll
    for (int u = 0; u < KV_UNROLL; ++u) {
      const int i = i0 + u * stride;
      if (i < nvec) *reinterpret_cast<uint4*>(dst + static_cast<size_t>(i) * 8) = val[u];
    }
  }
}

__global__ void cache_len_bump_kernel(int32_t* __restrict__ cache_len, int B, int C, int lmax) {
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int base = cache_len[b];
    if (base >= 0 && base + C <= lmax) cache_len[b] = base + C;
  }
}

__global__ void cache_len_set_kernel(int32_t* __restrict__ cache_len, int B, int value) {
  for (int b = threadIdx.x; b < B; b += blockDim.x) cache_len[b] = value;
}

}  // namespace dg
