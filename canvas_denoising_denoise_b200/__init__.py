"""B200-native block-autoregressive canvas denoising (DiffusionGemma-style).

Thin Python binding over libdg.so (include/dg.h).  PyTorch provides device
memory and streams; every step of the path runs in the library's CUDA
kernels.  There is no CPU fallback: every call needs the built library and a
CUDA device, and raises otherwise.

Functions take torch tensors and pass their device pointers:
    canvas_attn, unembed, linear, sample_commit, unembed_sample_commit, kv_block_commit,
    canvas_attn_e4m3, quantize_e4m3, linear_e4m3, unembed_e4m3, unembed_sample_commit_e4m3,
    philox
Objects:
    DgModel   weights + configuration (dg_model)
    DgState   KV caches and canvas state of a batch (dg_state)
    prefill, denoise_logits, denoise_block
"""
import ctypes

import torch

from . import _lib
from ._lib import (EPI_BF16, EPI_F32, EPI_GELU_BF16, EPI_RESID_F32, MASK_BIDIR, MASK_CAUSAL,
                   UNSELECTED_KEEP, UNSELECTED_RENOISE, DgError)

__all__ = ["canvas_attn", "canvas_attn_e4m3", "unembed", "linear", "sample_commit", "unembed_sample_commit",
           "quantize_e4m3", "linear_e4m3", "unembed_e4m3", "unembed_sample_commit_e4m3",
           "kv_block_commit", "philox",
           "DgModel", "DgState", "SamplerSettings", "prefill", "denoise_logits", "denoise_block",
           "linear_plan_of", "model_residual_on_pairs", "set_wait_limit_ns", "self_test_wait",
           "check_device_errors", "Workspace", "DgError", "MASK_BIDIR", "MASK_CAUSAL",
           "EPI_F32", "EPI_BF16", "EPI_GELU_BF16", "EPI_RESID_F32", "UNSELECTED_KEEP",
           "UNSELECTED_RENOISE"]


# dg_step_out fields, in order: x_hat, argmax (int32 [B, C]), logconf,
# entropy (fp32 [B, C]), flags (uint8 [B, C]), near_ties (int32 [B, 3])
_OUT_KEYS = ("x_hat", "argmax", "logconf", "entropy", "flags", "near_ties")


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _need_contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


class Workspace:
    """A growable device scratch buffer handed to the library."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = None

    def get(self, nbytes):
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self.buf

    def args(self, nbytes):
        if nbytes == 0:
            return None, 0
        b = self.get(nbytes)
        return _ptr(b), b.numel()


_default_ws = {}


def _ws(ws):
    if ws is not None:
        return ws
    dev = torch.cuda.current_device()
    if dev not in _default_ws:
        _default_ws[dev] = Workspace(f"cuda:{dev}")
    return _default_ws[dev]


def check_device_errors(stream=None):
    """Synchronise and raise if a kernel recorded a device-side error."""
    code = ctypes.c_uint32(0)
    _lib.check(_lib.load().dg_check_device_errors(_stream(stream), ctypes.byref(code)))
    return code.value


def canvas_attn(q, k_new, v_new, k_cache, v_cache, cache_len, max_prefix, out, *, n_q_heads,
                n_kv_heads, head_dim, lse=None, scale=None, mask=MASK_BIDIR, ws=None,
                stream=None):
    """Grouped-query attention of new rows over [cache prefix ; new rows].

    q [B, Lq, >=Hq*hd] bf16, k_new/v_new [B, Lq, ld] bf16 (views allowed via
    their row stride), k_cache/v_cache [B, Hkv, lmax, hd] bf16, cache_len [B]
    int32 (device), out [B, Lq, >=Hq*hd] bf16.
    """
    lib = _lib.load()
    B, Lq = q.shape[0], q.shape[1]
    lmax = k_cache.shape[2]
    for t in (q, k_new, v_new, out):
        if t.stride(-1) != 1 or t.stride(0) != t.shape[1] * t.stride(1):
            raise ValueError("q/k_new/v_new/out must be [B, Lq, ld] with unit inner stride")
    if k_new.stride(1) != v_new.stride(1):
        raise ValueError("k_new and v_new must share a row stride")
    _need_contig(k_cache, v_cache, cache_len, lse)
    scale = head_dim ** -0.5 if scale is None else scale
    need = lib.dg_canvas_attn_workspace_bytes(B, n_q_heads, n_kv_heads, Lq, head_dim, max_prefix)
    wp, wn = _ws(ws).args(need)
    _lib.check(lib.dg_canvas_attn(_ptr(q), q.stride(1), _ptr(k_new), _ptr(v_new), k_new.stride(1),
                                  _ptr(k_cache), _ptr(v_cache), _ptr(cache_len), max_prefix,
                                  lmax, _ptr(out), out.stride(1), _ptr(lse), B, n_q_heads,
                                  n_kv_heads, Lq, head_dim, scale, mask, wp, wn, _stream(stream)))
    return out


def canvas_attn_e4m3(q, q_scale, k_new, vt_new, k_cache, vt_cache, k_scale, v_scale, cache_len,
                     max_prefix, out, *, n_q_heads, n_kv_heads, lse=None, scale=None,
                     mask=MASK_BIDIR, ws=None, stream=None):
    """canvas_attn on e4m3 codes (uint8 tensors), head_dim 128.

    q [B, Lq, >=Hq*128] with per-token scales q_scale [B*Lq] fp32; k_new [B, Lq, ld];
    vt_new [B, Hkv, 128, ldvt] (V transposed, keys contiguous); k_cache [B, Hkv, lmax, 128];
    vt_cache [B, Hkv, 128, lmax]; k_scale, v_scale one-element fp32 tensors; out bf16.
    """
    lib = _lib.load()
    B, Lq = q.shape[0], q.shape[1]
    lmax = k_cache.shape[2]
    for t in (q, k_new, out):
        if t.stride(-1) != 1 or t.stride(0) != t.shape[1] * t.stride(1):
            raise ValueError("q/k_new/out must be [B, Lq, ld] with unit inner stride")
    if vt_new.stride(-1) != 1 or vt_new.stride(2) * 128 != vt_new.stride(1) or \
            vt_new.stride(1) * vt_new.shape[1] != vt_new.stride(0):
        raise ValueError("vt_new must be [B, Hkv, 128, ldvt] with unit inner stride")
    _need_contig(q_scale, k_cache, vt_cache, k_scale, v_scale, cache_len, lse)
    scale = 128 ** -0.5 if scale is None else scale
    need = lib.dg_canvas_attn_workspace_bytes(B, n_q_heads, n_kv_heads, Lq, 128, max_prefix)
    wp, wn = _ws(ws).args(need)
    _lib.check(lib.dg_canvas_attn_e4m3(
        _ptr(q), q.stride(1), _ptr(q_scale), _ptr(k_new), k_new.stride(1), _ptr(vt_new),
        vt_new.stride(2), _ptr(k_cache), _ptr(vt_cache), _ptr(k_scale), _ptr(v_scale),
        _ptr(cache_len), max_prefix, lmax, _ptr(out), out.stride(1), _ptr(lse), B, n_q_heads,
        n_kv_heads, Lq, 128, scale, mask, wp, wn, _stream(stream)))
    return out


def unembed(h, w_u, logits, stream=None):
    """logits[M, V] (fp32) = h[M, d] (bf16) @ w_u[V, d]^T (bf16)."""
    _need_contig(h, w_u, logits)
    M, d = h.shape
    V = w_u.shape[0]
    _lib.check(_lib.load().dg_unembed(_ptr(h), _ptr(w_u), _ptr(logits), M, d, V, None, 0,
                                      _stream(stream)))
    return logits


def linear(x, w, out, epilogue=EPI_BF16, ws=None, stream=None):
    """out[M, N] = epilogue(x[M, K] @ w[N, K]^T); see enum dg_epilogue."""
    _need_contig(x, w, out)
    lib = _lib.load()
    M, K = x.shape
    N = w.shape[0]
    wp, wn = _ws(ws).args(lib.dg_linear_workspace_bytes(M, N, K))
    _lib.check(lib.dg_linear(_ptr(x), _ptr(w), _ptr(out), M, N, K, epilogue, wp, wn,
                             _stream(stream)))
    return out


class SamplerSettings:
    """Mirror of dg_sampler_cfg; defaults are the published settings."""

    def __init__(self, **kw):
        c = _lib.SamplerCfg()
        _lib.load().dg_sampler_defaults(ctypes.byref(c))
        for k, v in kw.items():
            if not hasattr(c, k):
                raise AttributeError(k)
            setattr(c, k, v)
        self.c = c

    def __getattr__(self, k):
        return getattr(self.__dict__["c"], k)


def sample_commit(logits, tok, committed, prev_argmax, seq_status, settings, seed, block, step,
                  out=None, ws=None, stream=None):
    """One sampler step over logits [B, C, V] fp32; updates the canvas in place.

    out: optional dict of device tensors [B, C]: x_hat, argmax (int32),
    logconf, entropy (fp32), flags (uint8); and near_ties (int32 [B, 3]).
    """
    _need_contig(logits, tok, committed, prev_argmax, seq_status)
    lib = _lib.load()
    B, C, V = logits.shape
    so = None
    if out is not None:
        so = _lib.StepOut(*[(out[k].data_ptr() if out.get(k) is not None else None)
                            for k in _OUT_KEYS])
    wp, wn = _ws(ws).args(lib.dg_sample_commit_workspace_bytes(B, C, V))
    _lib.check(lib.dg_sample_commit(_ptr(logits), _ptr(tok), _ptr(committed), _ptr(prev_argmax),
                                    _ptr(seq_status), ctypes.byref(settings.c), seed, block, step,
                                    B, C, V, ctypes.byref(so) if so is not None else None,
                                    wp, wn, _stream(stream)))


def unembed_sample_commit(h, w_u, tok, committed, prev_argmax, seq_status, settings, seed,
                          block, step, out=None, ws=None, stream=None):
    """The unembedding h[B*C, d] @ w_u[V, d]^T fused with one sampler step.

    Same canvas updates and outputs as sample_commit on those logits; the
    logits are never written.  V % 256 == 0.
    """
    _need_contig(h, w_u, tok, committed, prev_argmax, seq_status)
    lib = _lib.load()
    B, C = tok.shape
    V, d = w_u.shape
    so = None
    if out is not None:
        so = _lib.StepOut(*[(out[k].data_ptr() if out.get(k) is not None else None)
                            for k in _OUT_KEYS])
    wp, wn = _ws(ws).args(lib.dg_unembed_sample_commit_workspace_bytes(B, C, V))
    _lib.check(lib.dg_unembed_sample_commit(
        _ptr(h), _ptr(w_u), d, _ptr(tok), _ptr(committed), _ptr(prev_argmax), _ptr(seq_status),
        ctypes.byref(settings.c), seed, block, step, B, C, V,
        ctypes.byref(so) if so is not None else None, wp, wn, _stream(stream)))


def quantize_e4m3(x, out, scales, per_row=True, stream=None):
    """bf16 x[R, C] -> e4m3 codes out[R, C] (uint8) and fp32 scales ([R] per row, else [1])."""
    _need_contig(x, out, scales)
    R, C = x.shape
    _lib.check(_lib.load().dg_quantize_e4m3(_ptr(x), R, C, 1 if per_row else 0, _ptr(out),
                                            _ptr(scales), _stream(stream)))


def linear_e4m3(x_q, x_scale, w_q, w_scale, out, epilogue=EPI_BF16, stream=None):
    """linear on e4m3 codes: acc = x_scale[m] w_scale (x_q[M, K] . w_q[N, K]), then the epilogue."""
    _need_contig(x_q, x_scale, w_q, w_scale, out)
    M, K = x_q.shape
    N = w_q.shape[0]
    _lib.check(_lib.load().dg_linear_e4m3(_ptr(x_q), _ptr(x_scale), _ptr(w_q), _ptr(w_scale),
                                          _ptr(out), M, N, K, epilogue, _stream(stream)))


def unembed_e4m3(h_q, h_scale, w_q, w_scale, logits, stream=None):
    """logits[M, V] = h_scale[m] w_scale (h_q[M, d] . w_q[V, d]) on e4m3 codes."""
    _need_contig(h_q, h_scale, w_q, w_scale, logits)
    M, d = h_q.shape
    V = w_q.shape[0]
    _lib.check(_lib.load().dg_unembed_e4m3(_ptr(h_q), _ptr(h_scale), _ptr(w_q), _ptr(w_scale),
                                           _ptr(logits), M, d, V, _stream(stream)))


def unembed_sample_commit_e4m3(h_q, h_scale, w_q, w_scale, tok, committed, prev_argmax,
                               seq_status, settings, seed, block, step, out=None, ws=None,
                               stream=None):
    """unembed_sample_commit with the logits of unembed_e4m3."""
    _need_contig(h_q, h_scale, w_q, w_scale, tok, committed, prev_argmax, seq_status)
    lib = _lib.load()
    B, C = tok.shape
    V, d = w_q.shape
    so = None
    if out is not None:
        so = _lib.StepOut(*[(out[k].data_ptr() if out.get(k) is not None else None)
                            for k in _OUT_KEYS])
    wp, wn = _ws(ws).args(lib.dg_unembed_sample_commit_workspace_bytes(B, C, V))
    _lib.check(lib.dg_unembed_sample_commit_e4m3(
        _ptr(h_q), _ptr(h_scale), _ptr(w_q), _ptr(w_scale), d, _ptr(tok), _ptr(committed),
        _ptr(prev_argmax), _ptr(seq_status), ctypes.byref(settings.c), seed, block, step, B, C,
        V, ctypes.byref(so) if so is not None else None, wp, wn, _stream(stream)))


def kv_block_commit(k_blk, v_blk, k_cache, v_cache, cache_len, *, n_kv_heads, head_dim,
                    stream=None):
    """Append per-layer block K/V ([B, C, ld] views) to the caches; cache_len += C."""
    n = len(k_blk)
    B, C = k_blk[0].shape[0], k_blk[0].shape[1]
    lmax = k_cache[0].shape[2]
    ld = k_blk[0].stride(1)
    arr = ctypes.c_void_p * n
    kb = arr(*[t.data_ptr() for t in k_blk])
    vb = arr(*[t.data_ptr() for t in v_blk])
    kc = arr(*[t.data_ptr() for t in k_cache])
    vc = arr(*[t.data_ptr() for t in v_cache])
    _lib.check(_lib.load().dg_kv_block_commit(kb, vb, ld, kc, vc, _ptr(cache_len), n, B,
                                              n_kv_heads, C, head_dim, lmax, _stream(stream)))


def philox(inp, out, stream=None):
    """Philox4x32-10 of n rows (counter c0..c3, key k0, k1) -> out [n, 4]; uint32 as int32."""
    _need_contig(inp, out)
    _lib.check(_lib.load().dg_philox4x32_10(_ptr(inp), _ptr(out), inp.shape[0], _stream(stream)))
    return out


def set_wait_limit_ns(ns, stream=None):
    """Wait limit of the kernels' bounded waits on the current device (0: the 2 s default)."""
    _lib.check(_lib.load().dg_set_wait_limit_ns(int(ns), _stream(stream)))


def self_test_wait(kind=0, stream=None):
    """Launch a kernel whose wait can never complete (0: one CTA, 1: a CTA pair);
    check_device_errors() then reports DG_ERR_TIMEOUT."""
    _lib.check(_lib.load().dg_self_test_wait(int(kind), _stream(stream)))


class DgModel:
    """Model weights (bf16 device tensors, [out, in]) and their dg_model view.

    fp8_unembed=True also keeps an e4m3 copy of the unembedding (one tensor
    scale), which the denoising loop's unembedding + sampler step then uses;
    fp8_layers=True keeps e4m3 copies of every projection weight (one scale
    each), and every forward pass then runs its projections in FP8.
    """

    def __init__(self, shape, weights, fp8_unembed=False, fp8_layers=False):
        self.shape = shape
        self.w = weights
        n = shape.n_layers
        self._layers = (_lib.LayerWeights * n)()
        for i, lw in enumerate(weights["layers"]):
            self._layers[i] = _lib.LayerWeights(lw["w_qkv"].data_ptr(), lw["w_o"].data_ptr(),
                                                lw["w_up"].data_ptr(), lw["w_down"].data_ptr())
        self.cfg = _lib.ModelCfg(shape.d, shape.n_layers, shape.n_q_heads, shape.n_kv_heads,
                                 shape.head_dim, shape.ffn, shape.vocab, shape.eps)
        self.unembed_q = self.unembed_scale = None
        if fp8_unembed:
            wu = weights["unembed"]
            self.unembed_q = torch.empty(wu.shape, dtype=torch.uint8, device=wu.device)
            self.unembed_scale = torch.empty(1, dtype=torch.float32, device=wu.device)
            quantize_e4m3(wu, self.unembed_q, self.unembed_scale, per_row=False)
        self.layers_q = None
        self._layers_q = None
        if fp8_layers:
            self.layers_q = []
            self._layers_q = (_lib.LayerWeightsE4M3 * n)()
            for i, lw in enumerate(weights["layers"]):
                q = {}
                sc = torch.empty(4, dtype=torch.float32, device=lw["w_qkv"].device)
                for j, name in enumerate(("w_qkv", "w_o", "w_up", "w_down")):
                    q[name] = torch.empty(lw[name].shape, dtype=torch.uint8,
                                          device=lw[name].device)
                    quantize_e4m3(lw[name], q[name], sc[j:j + 1], per_row=False)
                q["scales"] = sc
                self.layers_q.append(q)
                self._layers_q[i] = _lib.LayerWeightsE4M3(
                    q["w_qkv"].data_ptr(), q["w_o"].data_ptr(), q["w_up"].data_ptr(),
                    q["w_down"].data_ptr(), sc.data_ptr())
        self.c = _lib.Model(self.cfg, weights["embed"].data_ptr(), weights["unembed"].data_ptr(),
                            ctypes.cast(self._layers, ctypes.POINTER(_lib.LayerWeights)),
                            self.unembed_q.data_ptr() if fp8_unembed else None,
                            self.unembed_scale.data_ptr() if fp8_unembed else None,
                            ctypes.cast(self._layers_q, ctypes.POINTER(_lib.LayerWeightsE4M3))
                            if fp8_layers else None)


class DgState:
    """KV caches and canvas state of a batch, allocated with torch on `device`."""

    def __init__(self, shape, batch, lmax, canvas=256, device="cuda"):
        self.shape = shape
        self.batch, self.lmax, self.canvas = batch, lmax, canvas
        kvshape = (batch, shape.n_kv_heads, lmax, shape.head_dim)
        self.k_cache = [torch.zeros(kvshape, dtype=torch.bfloat16, device=device)
                        for _ in range(shape.n_layers)]
        self.v_cache = [torch.zeros(kvshape, dtype=torch.bfloat16, device=device)
                        for _ in range(shape.n_layers)]
        self.cache_len = torch.zeros(batch, dtype=torch.int32, device=device)
        self.tok = torch.zeros((batch, canvas), dtype=torch.int32, device=device)
        self.committed = torch.zeros((batch, canvas), dtype=torch.uint8, device=device)
        self.prev_argmax = torch.full((batch, canvas), -1, dtype=torch.int32, device=device)
        self.seq_status = torch.zeros(batch, dtype=torch.int32, device=device)
        self.step = torch.zeros(1, dtype=torch.int32, device=device)
        n = shape.n_layers
        self._kc = (ctypes.c_void_p * n)(*[t.data_ptr() for t in self.k_cache])
        self._vc = (ctypes.c_void_p * n)(*[t.data_ptr() for t in self.v_cache])
        self.c = _lib.State(batch, lmax, canvas, 0, self._kc, self._vc, self.cache_len.data_ptr(),
                            self.tok.data_ptr(), self.committed.data_ptr(),
                            self.prev_argmax.data_ptr(), self.seq_status.data_ptr(),
                            self.step.data_ptr())

    @property
    def cache_len_host(self):
        return self.c.cache_len_host

    @cache_len_host.setter
    def cache_len_host(self, v):
        self.c.cache_len_host = int(v)


def prefill(model, state, prompt, ws=None, stream=None):
    """Causal prefill of prompt [B, P] int32 (device) into the state's caches."""
    _need_contig(prompt)
    lib = _lib.load()
    P = prompt.shape[1]
    need = lib.dg_prefill_workspace_bytes(ctypes.byref(model.cfg), state.batch, P)
    wp, wn = _ws(ws).args(need)
    _lib.check(lib.dg_prefill(ctypes.byref(model.c), ctypes.byref(state.c), _ptr(prompt), P, wp, wn,
                              _stream(stream)))


def linear_plan_of(M, N, K, e4m3=False):
    """The plan dg_linear (or dg_linear_e4m3) uses for this shape: 0 split-K, 1 CTA pairs, -1 rejected."""
    return _lib.load().dg_linear_plan_of(M, N, K, 1 if e4m3 else 0)


def model_residual_on_pairs(model, M, e4m3=False):
    """1 when a forward pass of `model` over M tokens runs its residual projections on CTA pairs."""
    return _lib.load().dg_model_residual_on_pairs(ctypes.byref(model.cfg), M, 1 if e4m3 else 0)


def denoise_workspace_bytes(model, state):
    return _lib.load().dg_denoise_block_workspace_bytes(ctypes.byref(model.cfg), state.batch,
                                                        state.canvas, state.lmax)


def denoise_logits(model, state, logits, ws=None, stream=None):
    """One bidirectional forward of the canvas into logits [B, C, V] fp32."""
    lib = _lib.load()
    wp, wn = _ws(ws).args(denoise_workspace_bytes(model, state))
    _lib.check(lib.dg_denoise_logits(ctypes.byref(model.c), ctypes.byref(state.c), _ptr(logits),
                                     wp, wn, _stream(stream)))
    return logits


def denoise_block(model, state, settings, seed, block, ws=None, stream=None):
    """Denoise one canvas per sequence to its stop and commit its K/V; returns steps taken."""
    lib = _lib.load()
    wp, wn = _ws(ws).args(denoise_workspace_bytes(model, state))
    steps = ctypes.c_int(0)
    _lib.check(lib.dg_denoise_block(ctypes.byref(model.c), ctypes.byref(state.c),
                                    ctypes.byref(settings.c), seed, block, ctypes.byref(steps),
                                    wp, wn, _stream(stream)))
    return steps.value
