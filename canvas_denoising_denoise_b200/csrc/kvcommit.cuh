// kvcommit.cuh - append a finished block's K/V to the per-layer caches.
//
// "DiffusionGemma Guia do Desenvolvedor ...", Denoising bullet: when the
// 256-token block is finished it is committed to the KV cache and the next
// block starts (aiexpert.news architecture paragraph: each fully denoised
// block is committed and a new canvas is conditioned on the history).
//
// Pure data movement: each thread moves one 16-byte vector (8 bf16) from the
// token-major block K/V [B, C, ld] into the head-major cache [B, Hkv, lmax, hd]
// at row cache_len[b] + t.  A second one-CTA kernel then bumps cache_len, so
// every copy reads the same base row.
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

// Grid-stride over n_layers * 2 (K, V) * B * Hkv * C * (hd / 8) vectors.
__global__ void kv_commit_kernel(const __grid_constant__ KVTables tab, KVParams p) {
  const int vec_per_row = p.hd / 8;
  const size_t per_kv = static_cast<size_t>(p.B) * p.Hkv * p.C * vec_per_row;
  const size_t total = per_kv * 2 * p.n_layers;
  for (size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
    size_t r = idx;
    const int v8 = static_cast<int>(r % vec_per_row); r /= vec_per_row;
    const int t = static_cast<int>(r % p.C); r /= p.C;
    const int g = static_cast<int>(r % p.Hkv); r /= p.Hkv;
    const int b = static_cast<int>(r % p.B); r /= p.B;
    const int which = static_cast<int>(r % 2); r /= 2;
    const int l = static_cast<int>(r);
    const int base = p.cache_len[b];
    if (base < 0 || base + p.C > p.lmax) {
      if (v8 == 0 && t == 0 && g == 0 && which == 0 && l == 0)
        raise_error(ERR_CHECK | 0x401, static_cast<uint32_t>(b));
      continue;
    }
    const __nv_bfloat16* src = (which == 0 ? tab.k_blk[l] : tab.v_blk[l]) +
                               (static_cast<size_t>(b) * p.C + t) * p.ld_blk +
                               static_cast<size_t>(g) * p.hd + v8 * 8;
    __nv_bfloat16* dst = (which == 0 ? tab.k_cache[l] : tab.v_cache[l]) +
                         ((static_cast<size_t>(b) * p.Hkv + g) * p.lmax + base + t) * p.hd +
                         v8 * 8;
    *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
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
