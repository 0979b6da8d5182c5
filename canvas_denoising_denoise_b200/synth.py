"""Seeded synthetic inputs for the denoiser: weights, prompts, attention and logits tensors.

This module holds no step of the denoising method.  It only draws random
numbers with torch generators in a fixed order, so that the CUDA path and the
CPU oracle can be handed identical inputs.  Nothing here is trained: the
weights are random initialisations of the architecture's shapes.

Workload shapes:
  tiny        B=1, 64-token prompt, d=256, 2 layers, 4 q / 2 kv heads, hd=64,
              MLP 1024, vocab 512.
  attn_micro  B=1, Q [32 heads, 256, 128], prefix K/V [8, L, 128], canvas K/V
              [8, 256, 128], all N(0, 1), L in {1024, 4096, 16384, 32768}.
  full        B=1, 4096-token prompt, d=2048, 24 layers, 16 q / 8 kv heads,
              hd=128, MLP 8192, vocab 262144.
  sampler     logits [B, 256, 262144] fp32, N(0, 3) plus one planted token per
              position raised by U(2, 10); B in {1, 4, 16}.
  long        the full model, B in {1, 8}, 2048-token prompt, 8 canvases.
All matrices and embeddings are N(0, 0.02) in bf16; prompts are uniform token ids.
"""
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class ModelShape:
    d: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    eps: float = 1e-6


TINY = ModelShape(d=256, n_layers=2, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=1024, vocab=512)
FULL = ModelShape(d=2048, n_layers=24, n_q_heads=16, n_kv_heads=8, head_dim=128, ffn=8192,
                  vocab=262144)

CANVAS = 256

WORKLOADS = {
    "tiny": {"model": TINY, "batch": 1, "prompt": 64, "blocks": 1},
    "full": {"model": FULL, "batch": 1, "prompt": 4096, "blocks": 1},
    "long_b1": {"model": FULL, "batch": 1, "prompt": 2048, "blocks": 8},
    "long_b8": {"model": FULL, "batch": 8, "prompt": 2048, "blocks": 8},
}


def make_weights(shape, seed=0, device="cpu", std=0.02):
    """Random bf16 weights, drawn in a fixed order from one generator.

    Order: embed, then per layer (w_qkv, w_o, w_up, w_down), then unembed.
    Layout is [out_features, in_features].  Drawn in fp32 on the CPU and
    converted, so CPU and GPU callers get identical bits.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    hq, hkv, hd, d, f, v = (shape.n_q_heads, shape.n_kv_heads, shape.head_dim, shape.d,
                            shape.ffn, shape.vocab)

    def draw(*size):
        t = torch.empty(size, dtype=torch.float32)
        # chunked so that huge matrices do not need a second fp32 copy
        flat = t.view(-1)
        step = 1 << 24
        for i in range(0, flat.numel(), step):
            n = min(step, flat.numel() - i)
            flat[i:i + n] = torch.randn(n, generator=g) * std
        return t.to(torch.bfloat16).to(device)

    w = {"embed": draw(v, d), "layers": []}
    for _ in range(shape.n_layers):
        w["layers"].append({
            "w_qkv": draw((hq + 2 * hkv) * hd, d),
            "w_o": draw(d, hq * hd),
            "w_up": draw(f, d),
            "w_down": draw(d, f),
        })
    w["unembed"] = draw(v, d)
    return w


def make_weights_fast(shape, seed=0, device="cuda", std=0.02):
    """Random bf16 weights drawn directly on `device` (for large benchmark models).

    Same distribution and order as make_weights, but from a device generator,
    so the bits differ from make_weights.  Used where no oracle comparison of
    the whole model is made.
    """
    g = torch.Generator(device=device).manual_seed(seed)
    hq, hkv, hd, d, f, v = (shape.n_q_heads, shape.n_kv_heads, shape.head_dim, shape.d,
                            shape.ffn, shape.vocab)

    def draw(*size):
        return (torch.randn(size, generator=g, device=device, dtype=torch.float32) * std
                ).to(torch.bfloat16)

    w = {"embed": draw(v, d), "layers": []}
    for _ in range(shape.n_layers):
        w["layers"].append({
            "w_qkv": draw((hq + 2 * hkv) * hd, d),
            "w_o": draw(d, hq * hd),
            "w_up": draw(f, d),
            "w_down": draw(d, f),
        })
    w["unembed"] = draw(v, d)
    return w


def make_prompt(batch, length, vocab, seed=1):
    """Uniform random prompt token ids [batch, length] int32 (CPU)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randint(0, vocab, (batch, length), generator=g, dtype=torch.int64).to(torch.int32)


def make_attn_inputs(batch, n_q_heads, n_kv_heads, head_dim, q_len, prefix_len, seed=0,
                     device="cpu", lmax=None):
    """N(0, 1) bf16 attention inputs in the product's layouts.

    q        [B, q_len, Hq * hd]            (token-major, head h at columns h*hd)
    k_new,v_new [B, q_len, Hkv * hd]        (token-major)
    k_cache,v_cache [B, Hkv, lmax, hd]      (head-major; rows >= prefix_len are
                                             filled with noise that must be ignored)
    """
    lmax = lmax if lmax is not None else prefix_len
    g = torch.Generator(device="cpu").manual_seed(seed)

    def draw(*size):
        return torch.randn(size, generator=g, dtype=torch.float32).to(torch.bfloat16).to(device)

    q = draw(batch, q_len, n_q_heads * head_dim)
    k_new = draw(batch, q_len, n_kv_heads * head_dim)
    v_new = draw(batch, q_len, n_kv_heads * head_dim)
    k_cache = draw(batch, n_kv_heads, max(lmax, 1), head_dim)
    v_cache = draw(batch, n_kv_heads, max(lmax, 1), head_dim)
    return q, k_new, v_new, k_cache, v_cache


def make_sampler_logits(batch, canvas, vocab, seed, step, device="cpu"):
    """Sampler workload logits [B, canvas, vocab] fp32: N(0, 3) plus one planted token.

    One token per position (uniform index) is raised by U(2, 10).  Keyed by
    (seed, step) so that every step of the sweep sees fresh logits.
    """
    g = torch.Generator(device=device).manual_seed(int(seed) * 1000003 + int(step))
    x = torch.randn((batch, canvas, vocab), generator=g, device=device, dtype=torch.float32) * 3.0
    idx = torch.randint(0, vocab, (batch, canvas, 1), generator=g, device=device)
    bump = torch.rand((batch, canvas, 1), generator=g, device=device) * 8.0 + 2.0
    x.scatter_add_(2, idx, bump)
    return x
