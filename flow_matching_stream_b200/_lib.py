"""ctypes declarations of include/krea2.h and the loader of the in-tree libkrea2.so."""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_longlong, c_size_t, c_uint8, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkrea2.so")

KREA2_OK, KREA2_ERR_ARG, KREA2_ERR_WORKSPACE, KREA2_ERR_CUDA, KREA2_ERR_TIMEOUT, KREA2_ERR_UNSUPPORTED = 0, -1, -2, -3, -4, -5
KREA2_BF16, KREA2_F32 = 0, 1
KREA2_EPI_STORE, KREA2_EPI_SWIGLU, KREA2_EPI_RESID = 0, 1, 2
KREA2_NOALLOC_SCRATCH_BYTES = 64 << 20


class Krea2Dims(ctypes.Structure):
    _fields_ = [("C", c_int), ("H", c_int), ("Hkv", c_int), ("D", c_int), ("F", c_int),
                ("axes", c_int * 3), ("theta", c_float), ("eps", c_float),
                ("n_layers", c_int), ("in_ch", c_int), ("t_dim", c_int)]


class Krea2BlockWeights(ctypes.Structure):
    _fields_ = [("w_qkvg", c_void_p), ("w_out", c_void_p), ("w_gu", c_void_p), ("w_down", c_void_p),
                ("norm1_w", c_void_p), ("norm2_w", c_void_p), ("q_norm_w", c_void_p), ("k_norm_w", c_void_p),
                ("scale_shift_table", c_void_p)]


class Krea2ModelWeights(ctypes.Structure):
    _fields_ = [("img_in_w", c_void_p), ("img_in_b", c_void_p), ("t1_w", c_void_p), ("t1_b", c_void_p),
                ("t2_w", c_void_p), ("t2_b", c_void_p), ("mod_w", c_void_p), ("mod_b", c_void_p),
                ("final_norm_w", c_void_p), ("final_table", c_void_p), ("final_w", c_void_p),
                ("final_b", c_void_p), ("blocks", POINTER(Krea2BlockWeights))]


class Krea2TextDims(ctypes.Structure):
    _fields_ = [("Dt", c_int), ("L", c_int), ("H", c_int), ("Hkv", c_int), ("D", c_int), ("F", c_int),
                ("n_layerwise", c_int), ("n_refiner", c_int), ("C", c_int), ("eps", c_float)]


class Krea2TextWeights(ctypes.Structure):
    _fields_ = [("layerwise", POINTER(Krea2BlockWeights)), ("refiner", POINTER(Krea2BlockWeights)),
                ("layer_w", c_void_p), ("txt_in_w", c_void_p), ("txt_in_b", c_void_p)]


_PD = POINTER(Krea2Dims)
_PTD = POINTER(Krea2TextDims)
_PTW = POINTER(Krea2TextWeights)
_PB = POINTER(Krea2BlockWeights)
_PM = POINTER(Krea2ModelWeights)
V = c_void_p

# name -> (restype, argtypes); the full set of entry points declared in include/krea2.h
SIGNATURES = {
    "krea2_last_error_string": (c_char_p, []),
    "krea2_check_device_error": (c_int, [V]),
    "krea2_workspace_size": (c_size_t, [_PD, c_int, c_int, c_int, c_int]),
    "krea2_selftest_wait_timeout": (c_int, [c_int, V, V]),
    "krea2_attention_workspace_size": (c_size_t, [_PD, c_int, c_int, c_int, c_int]),
    "krea2_rope_tables": (c_int, [_PD, V, c_int, V, V, V]),
    "krea2_gqa_attention": (c_int, [_PD, c_int, c_int, c_int, c_int, V, V, V, V, V, V, V, V, c_size_t, V]),
    "krea2_modulated_rmsnorm": (c_int, [_PD, c_int, c_int, c_int, V, V, V, V, c_int, V, V]),
    "krea2_linear": (c_int, [c_int, c_int, c_int, c_int, c_int, V, V, V, V, c_int, c_longlong, V]),
    "krea2_time_embed": (c_int, [_PD, c_int, c_int, V, _PM, V, V, V, V]),
    "krea2_final_layer_workspace_size": (c_size_t, [_PD, c_int, c_int, c_int]),
    "krea2_final_layer": (c_int, [_PD, c_int, c_int, c_int, c_int, V, V, _PM, V, V, c_size_t, V]),
    "krea2_block_forward": (c_int, [_PD, c_int, c_int, c_int, c_int, V, V, _PB, V, V, V, V, c_size_t, V]),
    "krea2_backbone_forward": (c_int, [_PD, c_int, c_int, c_int, c_int, V, V, V, V, V, _PM, V, V, c_size_t, V]),
    "krea2_block_forward_traced": (c_int, [_PD, c_int, c_int, c_int, c_int, V, V, _PB, V, V, V, V, c_size_t,
                                           POINTER(c_void_p), V]),
    "krea2_launch_count": (ctypes.c_ulonglong, []),
    "krea2_shift_mu": (ctypes.c_double, [c_int]),
    "krea2_sigma_schedule": (c_int, [c_int, ctypes.c_double, V]),
    "krea2_euler_cfg_step": (c_int, [c_int, c_longlong, V, V, V, c_float, c_float, c_float, V, c_int, V, V]),
    "krea2_sample_workspace_size": (c_size_t, [_PD, c_int, c_int, c_int, c_int]),
    "krea2_sample": (c_int, [_PD, c_int, c_int, c_int, V, V, V, V, V, V, V, c_int, c_float, _PM, V, c_size_t, V]),
    "krea2_text_fusion_workspace_size": (c_size_t, [_PTD, c_int, c_int, c_int]),
    "krea2_text_fusion": (c_int, [_PTD, c_int, c_int, c_int, V, V, _PTW, V, V, c_size_t, V]),
    "krea2_block_causal_key_end": (c_int, [V, c_int, V]),
    "krea2_kv_cache_append": (c_int, [_PD, c_int, c_int, c_int, c_int, c_int, V, V, V, V, V, V, V]),
    "krea2_kv_cache_attention_workspace_size": (c_size_t, [_PD, c_int, c_int, c_int]),
    "krea2_gqa_attention_kv_cache": (c_int, [_PD, c_int, c_int, c_int, c_int, c_int, V, V, V, V, V, V, V, c_int, V,
                                             V, V, c_size_t, V]),
    "krea2_gqa_attention_block_causal": (c_int, [_PD, c_int, c_int, c_int, c_int, V, V, V, V, V, V, V, V, V,
                                                 c_size_t, V]),
    "krea2_gqa_attention_noalloc": (c_int, [_PD, c_int, c_int, c_int, c_int, V, V, V, V, V, V, V, V]),
}


def load() -> ctypes.CDLL:
    """Load libkrea2.so; raises if it has not been built (there is no fallback path)."""
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m flow_matching_stream_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
