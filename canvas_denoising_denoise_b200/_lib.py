"""ctypes declarations of libdg.so (include/dg.h).  Argument marshalling only."""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# DG_LIB_PATH selects another build of the library (e.g. a tuning variant)
LIB_PATH = os.environ.get("DG_LIB_PATH") or os.path.join(HERE, "libdg.so")

c_int = ctypes.c_int
c_float = ctypes.c_float
c_size_t = ctypes.c_size_t
c_uint32 = ctypes.c_uint32
c_void_p = ctypes.c_void_p
c_char_p = ctypes.c_char_p
P = ctypes.POINTER

DG_OK = 0
STATUS = {0: "DG_OK", 1: "DG_ERR_INVALID_ARG", 2: "DG_ERR_UNSUPPORTED_SHAPE",
          3: "DG_ERR_ALIGNMENT", 4: "DG_ERR_WORKSPACE_TOO_SMALL", 5: "DG_ERR_CUDA",
          6: "DG_ERR_TIMEOUT", 7: "DG_ERR_DEVICE_CHECK"}

MASK_BIDIR = 0
MASK_CAUSAL = 1
UNSELECTED_KEEP = 0
UNSELECTED_RENOISE = 1
EPI_F32 = 0
EPI_BF16 = 1
EPI_GELU_BF16 = 2
EPI_RESID_F32 = 3


class ModelCfg(ctypes.Structure):
    _fields_ = [("d", c_int), ("n_layers", c_int), ("n_q_heads", c_int), ("n_kv_heads", c_int),
                ("head_dim", c_int), ("ffn", c_int), ("vocab", c_int), ("eps", c_float)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("w_qkv", c_void_p), ("w_o", c_void_p), ("w_up", c_void_p), ("w_down", c_void_p)]


class LayerWeightsE4M3(ctypes.Structure):
    _fields_ = [("w_qkv", c_void_p), ("w_o", c_void_p), ("w_up", c_void_p), ("w_down", c_void_p),
                ("scales", c_void_p)]


class Model(ctypes.Structure):
    _fields_ = [("cfg", ModelCfg), ("embed", c_void_p), ("unembed", c_void_p),
                ("layers", P(LayerWeights)), ("unembed_e4m3", c_void_p),
                ("unembed_scale", c_void_p), ("layers_e4m3", P(LayerWeightsE4M3))]


class SamplerCfg(ctypes.Structure):
    _fields_ = [("max_steps", c_int), ("t_start", c_float), ("t_end", c_float),
                ("commit_k", c_int), ("renoise_conf", c_float), ("stop_entropy", c_float),
                ("unselected_policy", c_int), ("selection", c_int), ("entropy_bound", c_float)]


class StepOut(ctypes.Structure):
    _fields_ = [("x_hat", c_void_p), ("argmax", c_void_p), ("logconf", c_void_p),
                ("entropy", c_void_p), ("flags", c_void_p), ("near_ties", c_void_p)]


class State(ctypes.Structure):
    _fields_ = [("batch", c_int), ("lmax", c_int), ("canvas", c_int), ("cache_len_host", c_int),
                ("k_cache", P(c_void_p)), ("v_cache", P(c_void_p)), ("cache_len", c_void_p),
                ("tok", c_void_p), ("committed", c_void_p), ("prev_argmax", c_void_p),
                ("seq_status", c_void_p), ("step", c_void_p)]


# name -> (restype, argtypes); every name here is declared in include/dg.h
SIGNATURES = {
    "dg_status_string": (c_char_p, [c_int]),
    "dg_last_error": (c_char_p, []),
    "dg_version": (c_int, []),
    "dg_launch_count": (ctypes.c_ulonglong, []),
    "dg_sampler_defaults": (None, [P(SamplerCfg)]),
    "dg_check_device_errors": (c_int, [c_void_p, P(c_uint32)]),
    "dg_canvas_attn": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p,
                               c_void_p, c_int, c_int, c_void_p, c_int, c_void_p, c_int, c_int,
                               c_int, c_int, c_int, c_float, c_int, c_void_p, c_size_t,
                               c_void_p]),
    "dg_canvas_attn_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int]),
    "dg_canvas_attn_e4m3": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int, c_void_p, c_int,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                    c_int, c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int,
                                    c_int, c_float, c_int, c_void_p, c_size_t, c_void_p]),
    "dg_unembed": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_size_t,
                           c_void_p]),
    "dg_linear": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p,
                          c_size_t, c_void_p]),
    "dg_linear_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
    "dg_linear_plan_of": (c_int, [c_int, c_int, c_int, c_int]),
    "dg_model_residual_on_pairs": (c_int, [P(ModelCfg), c_int, c_int]),
    "dg_sample_commit": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, P(SamplerCfg),
                                 c_uint32, c_int, c_int, c_int, c_int, c_int, P(StepOut),
                                 c_void_p, c_size_t, c_void_p]),
    "dg_sample_commit_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
    "dg_unembed_sample_commit": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                         c_void_p, P(SamplerCfg), c_uint32, c_int, c_int, c_int,
                                         c_int, c_int, P(StepOut), c_void_p, c_size_t,
                                         c_void_p]),
    "dg_unembed_sample_commit_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
    "dg_quantize_e4m3": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "dg_linear_e4m3": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
                               c_int, c_int, c_void_p]),
    "dg_unembed_e4m3": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
                                c_int, c_void_p]),
    "dg_unembed_sample_commit_e4m3": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                              c_void_p, c_void_p, c_void_p, c_void_p,
                                              P(SamplerCfg), c_uint32, c_int, c_int, c_int,
                                              c_int, c_int, P(StepOut), c_void_p, c_size_t,
                                              c_void_p]),
    "dg_sample_commit_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         P(SamplerCfg), c_uint32, c_int, c_int, c_int, c_int,
                                         c_int, P(StepOut), c_void_p]),
    "dg_kv_block_commit": (c_int, [P(c_void_p), P(c_void_p), c_int, P(c_void_p), P(c_void_p),
                                   c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p]),
    "dg_prefill": (c_int, [P(Model), P(State), c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "dg_prefill_workspace_bytes": (c_size_t, [P(ModelCfg), c_int, c_int]),
    "dg_denoise_logits": (c_int, [P(Model), P(State), c_void_p, c_void_p, c_size_t, c_void_p]),
    "dg_denoise_block": (c_int, [P(Model), P(State), P(SamplerCfg), c_uint32, c_int, P(c_int),
                                 c_void_p, c_size_t, c_void_p]),
    "dg_denoise_block_workspace_bytes": (c_size_t, [P(ModelCfg), c_int, c_int, c_int]),
    "dg_philox4x32_10": (c_int, [c_void_p, c_void_p, c_int, c_void_p]),
    "dg_set_wait_limit_ns": (c_int, [ctypes.c_uint64, c_void_p]),
    "dg_self_test_wait": (c_int, [c_int, c_void_p]),
}

_LIB = None


class DgError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


def load():
    """Load libdg.so; fails loudly if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m canvas_denoising_denoise_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def check(status):
    if status != DG_OK:
        msg = load().dg_last_error().decode(errors="replace")
        raise DgError(status, msg)
