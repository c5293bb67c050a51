"""ctypes mirror of include/xlpk.h (argument marshalling only)."""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "lib", "libxlpk.so")

XLPK_OK = 0
XLPK_ERR_INVALID_ARG = -1
XLPK_ERR_UNSUPPORTED = -2
XLPK_ERR_CUDA = -3
XLPK_ERR_OOM = -4
XLPK_ERR_KV_FULL = -5
XLPK_ERR_TIMEOUT = -6
XLPK_ERR_ABORTED = -7

XLPK_NOALLOC_SCRATCH_BYTES = 8 << 20

XLPK_DTYPE_BF16 = 0
XLPK_DTYPE_FP8_E4M3 = 1
XLPK_DTYPE_NVFP4 = 2

XLPK_FLAG_NO_FUSED_FFN = 1
XLPK_FLAG_NO_TENSOR_CORES = 2
XLPK_FLAG_FLOAT_FFN_REDUCE = 4


class xlpk_config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
        "n_experts", "top_k", "n_shared_experts", "expert_ffn", "weight_dtype", "batch",
        "max_seq")] + [("rope_theta", C.c_float), ("rms_eps", C.c_float),
                       ("n_ctas", C.c_int32), ("spin_limit_us", C.c_int32), ("flags", C.c_int32),
                       ("window", C.c_int32), ("kv_dtype", C.c_int32), ("k_scale", C.c_float),
                       ("v_scale", C.c_float)]


class xlpk_linear(C.Structure):
    _fields_ = [("w_dev", C.c_void_p), ("scale_dev", C.c_void_p), ("global_scale", C.c_float)]


class xlpk_layer_weights(C.Structure):
    _fields_ = [("attn_norm_dev", C.c_void_p), ("wq", xlpk_linear), ("wk", xlpk_linear),
                ("wv", xlpk_linear), ("wo", xlpk_linear), ("ffn_norm_dev", C.c_void_p),
                ("w_gate", xlpk_linear), ("w_up", xlpk_linear), ("w_down", xlpk_linear),
                ("router_dev", C.c_void_p), ("we_gate", xlpk_linear), ("we_up", xlpk_linear),
                ("we_down", xlpk_linear), ("ws_gate", xlpk_linear), ("ws_up", xlpk_linear),
                ("ws_down", xlpk_linear)]


class xlpk_weights(C.Structure):
    _fields_ = [("embed_dev", C.c_void_p), ("final_norm_dev", C.c_void_p),
                ("lm_head", xlpk_linear), ("layers", C.POINTER(xlpk_layer_weights))]


class xlpk_kv(C.Structure):
    _fields_ = [("k_dev", C.c_void_p), ("v_dev", C.c_void_p), ("page_table_dev", C.c_void_p),
                ("page_size", C.c_int32), ("n_pages", C.c_int32)]


class xlpk_decode_io(C.Structure):
    _fields_ = [("forced_tokens_dev", C.c_void_p), ("logits_dev", C.c_void_p),
                ("hidden_dev", C.c_void_p), ("experts_dev", C.c_void_p), ("trace_dev", C.c_void_p),
                ("withhold_release", C.c_int32)]


class xlpk_info(C.Structure):
    _fields_ = [("n_ctas", C.c_int32), ("threads_per_cta", C.c_int32), ("smem_bytes", C.c_int32),
                ("ring_slots", C.c_int32), ("slot_bytes", C.c_int32),
                ("kernels_per_step_unfused", C.c_int32), ("packed_weight_bytes", C.c_int64),
                ("workspace_bytes", C.c_int64), ("weight_bytes_per_step", C.c_int64)]


# name -> (restype, argtypes); every symbol the header declares
SIGNATURES = {
    "xlpk_create": (C.c_int32, [C.POINTER(xlpk_config), C.POINTER(xlpk_weights),
                                C.POINTER(xlpk_kv), C.POINTER(C.c_void_p)]),
    "xlpk_destroy": (C.c_int32, [C.c_void_p]),
    "xlpk_set_state": (C.c_int32, [C.c_void_p, C.POINTER(C.c_int32), C.POINTER(C.c_int32), C.c_void_p]),
    "xlpk_decode": (C.c_int32, [C.c_void_p, C.c_int32, C.c_void_p, C.POINTER(xlpk_decode_io), C.c_void_p]),
    "xlpk_decode_unfused": (C.c_int32, [C.c_void_p, C.c_int32, C.c_void_p,
                                        C.POINTER(xlpk_decode_io), C.c_void_p]),
    "xlpk_decode_noalloc": (C.c_int32, [C.c_void_p, C.c_int32, C.c_void_p,
                                        C.POINTER(xlpk_decode_io), C.c_void_p]),
    "xlpk_debug_logits": (C.c_int32, [C.c_void_p, C.c_void_p, C.c_void_p]),
    "xlpk_verify": (C.c_int32, [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.POINTER(C.c_int32),
                                C.POINTER(xlpk_decode_io), C.c_void_p]),
    "xlpk_serve_start": (C.c_int32, [C.c_void_p, C.c_int32, C.c_void_p]),
    "xlpk_serve_post": (C.c_int32, [C.c_void_p, C.c_int32, C.POINTER(C.c_int64)]),
    "xlpk_serve_wait": (C.c_int32, [C.c_void_p, C.c_int64, C.c_int32, C.POINTER(C.c_int32), C.c_int32]),
    "xlpk_serve_stop": (C.c_int32, [C.c_void_p]),
    "xlpk_generate": (C.c_int32, [C.c_void_p, C.POINTER(C.c_int32), C.POINTER(C.c_int32), C.c_int32,
                                  C.POINTER(C.c_int32), C.c_void_p]),
    "xlpk_get_status": (C.c_int32, [C.c_void_p]),
    "xlpk_get_info": (C.c_int32, [C.c_void_p, C.POINTER(xlpk_info)]),
    "xlpk_status_string": (C.c_char_p, [C.c_int32]),
    "xlpk_last_cuda_error": (C.c_char_p, []),
    "xlpk_tc_gemm_tile": (C.c_int32, [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]),
}


def load(path: str = LIB_PATH) -> C.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"libxlpk.so not found at {path}: build it with `python -m persistent_decode_b200.build` "
            "(there is no CPU fallback)")
    lib = C.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
