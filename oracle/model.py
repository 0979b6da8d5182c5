"""Plain fp64 CPU forward pass of the canvas denoiser (the oracle's model half).

TEST INFRASTRUCTURE ONLY: only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path.

What it computes, and where it comes from:

* Prefill is ordinary causal attention over the prompt whose keys and values
  are written to a KV cache ("DiffusionGemma Guia do Desenvolvedor ...",
  section "Block Autoregressive Diffusion para Sequencias Longas", the Prefill
  bullet; aiexpert.news "Google's DiffusionGemma Atinge 1.000 Tokens por
  Segundo", architecture paragraph).
* Denoising runs the same stack over a 256-token canvas whose tokens attend
  bidirectionally to each other and to the cached prefix (same pages; the
  Google docs page, bullet "Arquitetura de codificador-decodificador").
* The finished block is committed to the cache (Guia do Desenvolvedor, the
  Denoising bullet).  Reading taken here: the committed K/V are those of a
  causal pass over the final block tokens, so that a block-committed cache is
  identical to a one-shot causal prefill of the same token sequence.
* The backbone is a generic pre-norm transformer with random weights: RMSNorm
  (eps 1e-6, unit gain), fused QKV projection, grouped-query attention scaled
  by 1/sqrt(head_dim) with no positional encoding, output projection with a
  residual, a dense exact-erf GELU MLP with a residual (standing in for the
  mixture-of-experts FFN, whose routing the pages leave open), a final
  RMSNorm and an untied unembedding.

Weight layout (nn.Linear convention, [out_features, in_features]):
    embed   [V, d]          unembed [V, d]
    w_qkv   [(Hq + 2 Hkv) hd, d]   rows ordered [Q heads | K heads | V heads]
    w_o     [d, Hq hd]
    w_up    [F, d]          w_down  [d, F]

FP8 (a reading: the pages quote FP8 checkpoints but fix no recipe).  With
``e4m3_unembed=True`` the final normalised hidden state, stored as bfloat16,
is quantised to e4m3 per token and the unembedding per tensor (oracle.fp8),
and the logits are the scaled products of the codes.  With
``e4m3_layers=True`` every projection of the stack (QKV, output, MLP up and
down) does the same with its input as stored (bf16) and its weight.

Storage rounding: with ``bf16_storage=True`` (default) the oracle rounds to
bfloat16 at the points where the product stores bfloat16 tensors - the
normalised GEMM inputs, Q/K/V (hence the KV cache), the attention output and
the GELU output - and keeps everything else, the residual stream included, in
fp64.  All arithmetic between those points is fp64.
"""
from dataclasses import dataclass

import numpy as np
from scipy.special import erf

from . import fp8


@dataclass(frozen=True)
class ModelCfg:
    d: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    eps: float = 1e-6


def round_bf16(x):
    """Round to the nearest bfloat16 (ties to even), returned as fp64.

    Goes through fp32 first; a double rounding can only differ from a direct
    rounding on exact fp32 ties of the discarded half, which the tolerance-based
    comparisons never resolve.
    """
    x32 = np.asarray(x, dtype=np.float32)
    bits = x32.view(np.uint32).astype(np.uint64)
    bits = (bits + np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))) & np.uint64(0xFFFF0000)
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


def rmsnorm(x, eps):
    """x / sqrt(mean(x^2) + eps) over the last axis; the gain is 1."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def gelu(x):
    """Exact GELU: x * Phi(x) with the normal CDF written through erf."""
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def attention_head(q, k, v, mask, scale):
    """softmax(q k^T * scale, masked) v for one head.

    q [Lq, hd], k/v [Lk, hd], mask [Lq, Lk] boolean (True = may attend).
    Every query row must have at least one allowed key.
    """
    s = (q @ k.T) * scale
    s = np.where(mask, s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    p = np.exp(s - m)
    p = p / np.sum(p, axis=1, keepdims=True)
    return p @ v


def canvas_mask(prefix_len, lq, causal):
    """Key mask for Lq new rows attending to [prefix ; new rows].

    All prefix keys are visible.  Within the new rows the mask is full for a
    denoising canvas (bidirectional) and lower-triangular for a causal pass
    (prefill, block re-encode).
    """
    pre = np.ones((lq, prefix_len), dtype=bool)
    if causal:
        own = np.tril(np.ones((lq, lq), dtype=bool))
    else:
        own = np.ones((lq, lq), dtype=bool)
    return np.concatenate([pre, own], axis=1)


def gqa_attention(q, k_new, v_new, k_pre, v_pre, causal, scale):
    """Grouped-query attention of one sequence.

    q [Lq, Hq, hd]; k_new/v_new [Lq, Hkv, hd]; k_pre/v_pre [Hkv, L, hd].
    Query head h reads kv head h // (Hq // Hkv).  Returns [Lq, Hq, hd].
    """
    lq, hq, hd = q.shape
    hkv = k_new.shape[1]
    group = hq // hkv
    prefix_len = k_pre.shape[1]
    mask = canvas_mask(prefix_len, lq, causal)
    out = np.empty_like(q)
    for h in range(hq):
        g = h // group
        k = np.concatenate([k_pre[g], k_new[:, g, :]], axis=0)
        v = np.concatenate([v_pre[g], v_new[:, g, :]], axis=0)
        out[:, h, :] = attention_head(q[:, h, :], k, v, mask, scale)
    return out


def _r(x, on):
    return round_bf16(x) if on else x


def linear_e4m3(a, w):
    """a [R, K] @ w [N, K]^T on e4m3 operands: per-row codes and scales of a, one
    scale for w, products of the decoded codes summed in fp64 and scaled
    (the same arithmetic as the FP8 unembedding, whose pins cover it)."""
    aq, as_ = fp8.quantize_rows(a)
    wq, ws = fp8.quantize_tensor(w)
    acc = fp8.decode(aq) @ fp8.decode(wq).T
    return acc * (np.asarray(as_, dtype=np.float64) * np.float64(ws))[:, None]


def layer_forward(cfg, w, x, k_pre, v_pre, causal, bf16_storage=True, skip_tail=False,
                  e4m3=False):
    """One pre-norm transformer layer over one sequence's new rows.

    x [Lq, d] (residual stream, fp64); k_pre/v_pre [Hkv, L, hd] cached prefix.
    Returns (x_out, k_new, v_new) with k_new/v_new [Lq, Hkv, hd] as stored.
    With skip_tail the attention/MLP half is skipped (only K/V are wanted).
    With e4m3 the four projections run on e4m3 operands (linear_e4m3).
    """
    hq, hkv, hd = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    lq = x.shape[0]

    def lin(a, name):
        return linear_e4m3(a, w[name]) if e4m3 else a @ w[name].T

    xn = _r(rmsnorm(x, cfg.eps), bf16_storage)
    qkv = _r(lin(xn, "w_qkv"), bf16_storage)
    q = qkv[:, : hq * hd].reshape(lq, hq, hd)
    k_new = qkv[:, hq * hd: (hq + hkv) * hd].reshape(lq, hkv, hd)
    v_new = qkv[:, (hq + hkv) * hd:].reshape(lq, hkv, hd)
    if skip_tail:
        return x, k_new, v_new
    o = gqa_attention(q, k_new, v_new, k_pre, v_pre, causal, 1.0 / np.sqrt(hd))
    o = _r(o.reshape(lq, hq * hd), bf16_storage)
    h = x + lin(o, "w_o")
    hn = _r(rmsnorm(h, cfg.eps), bf16_storage)
    u = _r(gelu(lin(hn, "w_up")), bf16_storage)
    x_out = h + lin(u, "w_down")
    return x_out, k_new, v_new


def unembed_e4m3(hn, w_unembed):
    """FP8 logits of normalised hidden states hn [Lq, d]: per-token e4m3 codes and
    scales of hn, one e4m3 scale for the unembedding, products of the decoded
    codes summed in fp64 and scaled."""
    hq, hs = fp8.quantize_rows(hn)
    wq, ws = fp8.quantize_tensor(w_unembed)
    return fp8.unembed_logits(hq, hs, wq, ws).astype(np.float64)


def forward(cfg, weights, tokens, k_cache, v_cache, prefix_len, causal,
            bf16_storage=True, want_logits=True, e4m3_unembed=False, e4m3_layers=False,
            logit_rows=None):
    """Run the stack over new rows of one sequence.

    tokens [Lq] int; k_cache/v_cache: per layer [Hkv, >=prefix_len, hd] arrays.
    Returns (logits [Lq, V] or None, list of per-layer (k_new, v_new)).
    The embedding lookup has no scaling.  With logit_rows (indices into the
    Lq rows) only those rows are unembedded, in that order: every row of the
    stack is still computed, since attention mixes them.
    """
    x = weights["embed"][np.asarray(tokens)].astype(np.float64)
    kv = []
    for l in range(cfg.n_layers):
        k_pre = k_cache[l][:, :prefix_len, :]
        v_pre = v_cache[l][:, :prefix_len, :]
        last = (l == cfg.n_layers - 1)
        x, k_new, v_new = layer_forward(cfg, weights["layers"][l], x, k_pre, v_pre, causal,
                                        bf16_storage, skip_tail=(last and not want_logits),
                                        e4m3=e4m3_layers)
        kv.append((k_new, v_new))
    if not want_logits:
        return None, kv
    hn = _r(rmsnorm(x, cfg.eps), bf16_storage)
    if logit_rows is not None:
        hn = hn[np.asarray(logit_rows)]
    if e4m3_unembed:
        return unembed_e4m3(hn, weights["unembed"]), kv
    logits = hn @ weights["unembed"].T
    return logits, kv


def empty_cache(cfg, lmax):
    """Per-layer zero K/V caches [Hkv, lmax, hd] for one sequence."""
    shape = (cfg.n_kv_heads, lmax, cfg.head_dim)
    return ([np.zeros(shape) for _ in range(cfg.n_layers)],
            [np.zeros(shape) for _ in range(cfg.n_layers)])


def commit_kv(k_cache, v_cache, kv, at):
    """Append per-layer new K/V [Lq, Hkv, hd] into the caches at row `at`."""
    for l, (k_new, v_new) in enumerate(kv):
        lq = k_new.shape[0]
        k_cache[l][:, at: at + lq, :] = np.transpose(k_new, (1, 0, 2))
        v_cache[l][:, at: at + lq, :] = np.transpose(v_new, (1, 0, 2))
    return at + kv[0][0].shape[0]


def prefill(cfg, weights, prompt, k_cache, v_cache, bf16_storage=True, e4m3_layers=False):
    """Causal pass over the prompt; writes its K/V at rows [0, P).  Returns P."""
    _, kv = forward(cfg, weights, prompt, k_cache, v_cache, 0, causal=True,
                    bf16_storage=bf16_storage, want_logits=False, e4m3_layers=e4m3_layers)
    return commit_kv(k_cache, v_cache, kv, 0)


def denoise_logits(cfg, weights, canvas, k_cache, v_cache, prefix_len, bf16_storage=True,
                   e4m3_unembed=False, e4m3_layers=False, rows=None):
    """Bidirectional pass of the canvas over the cached prefix -> logits [C, V]
    (or [len(rows), V] for the canvas rows listed in `rows`)."""
    logits, _ = forward(cfg, weights, canvas, k_cache, v_cache, prefix_len, causal=False,
                        bf16_storage=bf16_storage, want_logits=True, e4m3_unembed=e4m3_unembed,
                        e4m3_layers=e4m3_layers, logit_rows=rows)
    return logits


def block_commit(cfg, weights, block_tokens, k_cache, v_cache, prefix_len, bf16_storage=True):
    """Causal re-encode of the finished block and append of its K/V.  Returns new length."""
    _, kv = forward(cfg, weights, block_tokens, k_cache, v_cache, prefix_len, causal=True,
                    bf16_storage=bf16_storage, want_logits=False)
    return commit_kv(k_cache, v_cache, kv, prefix_len)


def weights_to_f64(w_torch):
    """Convert a weight dict of bf16 torch tensors to fp64 NumPy arrays (exact)."""
    out = {"embed": w_torch["embed"].double().numpy(),
           "unembed": w_torch["unembed"].double().numpy(),
           "layers": []}
    for lw in w_torch["layers"]:
        out["layers"].append({k: v.double().numpy() for k, v in lw.items()})
    return out
