"""ctypes binding of libdllm.so: the C ABI declared in include/dllm.h.

Argument marshalling only; every step of the decode path runs in the
library's CUDA kernels.  Loading fails loudly (``DllmError``) when the
library has not been built.  Functions keep the C names.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdllm.so")

DLLM_OK, DLLM_ERR_INVALID, DLLM_ERR_UNSUPPORTED = 0, -1, -2
DLLM_ERR_CUDA, DLLM_ERR_TIMEOUT, DLLM_ERR_WORKSPACE = -3, -4, -5
DLLM_CACHE_NONE, DLLM_CACHE_PREFIX, DLLM_CACHE_DUAL, DLLM_CACHE_DUAL_PRUNED = 0, 1, 2, 3
DLLM_W_BF16, DLLM_W_F32_SPLIT = 0, 1
DLLM_COMMIT_THRESHOLD, DLLM_COMMIT_TOPK = 0, 1
DLLM_DEVICE_TIMEOUT = 1  # status-word bit of a device wait that gave up
DLLM_DEVICE_BAD_TOKEN = 2  # a token id outside [0, V) reached the embedding gather
DLLM_DEVICE_INDEX = 4  # DLLM_DEBUG build: a row position from device memory was out of range


class DllmError(RuntimeError):
    pass


class dllm_config(C.Structure):
    _fields_ = [("batch", C.c_int32), ("n_layers", C.c_int32), ("hidden", C.c_int32),
                ("n_q_heads", C.c_int32), ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32),
                ("vocab", C.c_int32), ("prompt_len", C.c_int32), ("gen_len", C.c_int32),
                ("block", C.c_int32), ("window", C.c_int32), ("mask_id", C.c_int32),
                ("tau", C.c_float), ("rope_theta", C.c_float), ("mode", C.c_int32),
                ("weight_format", C.c_int32), ("commit_mode", C.c_int32),
                ("steps_per_block", C.c_int32), ("exit_tau", C.c_float)]


class dllm_weights(C.Structure):
    _fields_ = [("wqkv", C.c_void_p), ("wo", C.c_void_p), ("w_lm", C.c_void_p),
                ("embed", C.c_void_p)]


class dllm_state(C.Structure):
    _fields_ = [("tokens", C.c_void_p), ("masked", C.c_void_p), ("seq_start", C.c_void_p),
                ("k_cache", C.c_void_p), ("v_cache", C.c_void_p), ("plants", C.c_void_p),
                ("tau", C.c_void_p)]


_P = C.c_void_p
_I = C.c_int32
_CFG = C.POINTER(dllm_config)
_W = C.POINTER(dllm_weights)
_ST = C.POINTER(dllm_state)

# name -> (restype, argtypes)
SIGNATURES = {
    "dllm_workspace_size": (C.c_int, [_CFG, C.POINTER(C.c_size_t)]),
    "dllm_workspace_init": (C.c_int, [_CFG, _P, C.c_size_t, _P]),
    "dllm_split_f32_weights": (C.c_int, [_P, _P, C.c_int64, C.c_int64, _P]),
    "dllm_embed_rows": (C.c_int, [_CFG, _W, _ST, _I, _I, _P, _P, _P, _P]),
    "dllm_qkv_proj": (C.c_int, [_CFG, _W, _I, _P, _P, _I, _I, _P, _P, _P, _P, _P, C.c_size_t,
                                _P]),
    "dllm_block_attn": (C.c_int, [_CFG, _I, _I, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "dllm_o_proj": (C.c_int, [_CFG, _W, _I, _P, _I, _I, _P, _P, _P, _P, C.c_size_t, _P]),
    "dllm_final_norm": (C.c_int, [_CFG, _P, _I, _I, _I, _P, _P, _P, _P]),
    "dllm_lmhead_confidence": (C.c_int, [_CFG, _W, _P, _I, _P, _P, _P, _P, C.c_size_t, _P]),
    "dllm_lmhead_confidence_noalloc": (C.c_int, [_CFG, _W, _P, _I, _P, _P, _P, _P]),
    "dllm_threshold_commit": (C.c_int, [_CFG, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "dllm_prefill": (C.c_int, [_CFG, _W, _ST, _P, C.c_size_t, _P]),
    "dllm_decode_step": (C.c_int, [_CFG, _W, _ST, _I, _P, C.c_size_t, _P]),
    "dllm_kv_cache_refresh": (C.c_int, [_CFG, _W, _ST, _I, _P, C.c_size_t, _P]),
    "dllm_decode_block": (C.c_int, [_CFG, _W, _ST, _I, _I, C.POINTER(C.c_int32), _P,
                                    C.c_size_t, _P]),
    "dllm_decode_all": (C.c_int, [_CFG, _W, _ST, C.POINTER(C.c_int32), _P, C.c_size_t, _P]),
    "dllm_step_outputs": (C.c_int, [_CFG, _P, C.c_size_t, C.POINTER(C.c_void_p),
                                    C.POINTER(C.c_void_p), C.POINTER(C.c_void_p),
                                    C.POINTER(C.c_void_p), C.POINTER(C.c_void_p),
                                    C.POINTER(C.c_void_p)]),
    "dllm_device_status": (C.c_int, [_P, C.POINTER(C.c_int32), _P]),
    "dllm_launch_count": (C.c_uint64, []),
    "dllm_graph_cache_clear": (None, []),
    "dllm_set_l2_prefetch": (C.c_int, [C.c_int64, C.c_int64, C.c_int32]),
    "dllm_set_layer_stack": (C.c_int, [C.c_int32, C.c_int32]),
    "dllm_layer_stack_plan": (C.c_int, [_CFG, _I, C.POINTER(C.c_int32)]),
    "dllm_attention_plan": (C.c_int, [_CFG, _I, C.POINTER(C.c_int32)]),
    "dllm_selftest_wait_timeout": (C.c_int, [_P, C.c_int32, _P]),
    "dllm_status_string": (C.c_char_p, [C.c_int]),
}

_lib = None


def lib():
    """The loaded library (loaded on first use; raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise DllmError(f"CUDA library not built: {LIB_PATH} is missing "
                            "(run diffusion_decoding_step_b200/build.py)")
        handle = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(status: int, what: str = "") -> None:
    if status != DLLM_OK:
        msg = lib().dllm_status_string(status).decode()
        raise DllmError(f"{what}: {msg} ({status})")


def _call(name):
    def f(*args):
        return getattr(lib(), name)(*args)
    f.__name__ = name
    return f


for _name in SIGNATURES:
    globals()[_name] = _call(_name)
