"""ctypes binding of libspec.so: the C ABI declared in include/spec.h, same names.

Argument marshalling only.  Every step of tree verification runs in the CUDA
kernels of libspec.so; importing this module fails loudly when the library has
not been built.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspec.so")

SPEC_OK = 0
SPEC_ERR_ARG = -1
SPEC_ERR_TREE = -2
SPEC_ERR_TOKEN = -3
SPEC_ERR_CAPACITY = -4
SPEC_ERR_ROOT = -5
SPEC_ERR_CUDA = -6
SPEC_ERR_TIMEOUT = -7
SPEC_ERR_STATE = -8
SPEC_ERR_RANGE = -9

SPEC_DTYPE_F32 = 0
SPEC_DTYPE_BF16 = 1

SPEC_DEVICE_OUTPUTS = 1
SPEC_DEBUG_LOGITS = 2
SPEC_NO_GRAPH = 4
SPEC_FEATURES = 8
SPEC_DRAFT_TOPK = 10

PROF_CLASSES = ("embed_meta", "gemm_qkv", "rope_kv_store", "attention", "gemm_o", "resid_norm", "gemm_gate_up",
                "gemm_down", "lm_head", "lm_reduce", "accept_walk", "kv_compact", "gemm_layer", "draft_fc", "topk",
                "features", "draft_tree")

ERR_NAMES = {0: "SPEC_OK", -1: "SPEC_ERR_ARG", -2: "SPEC_ERR_TREE", -3: "SPEC_ERR_TOKEN", -4: "SPEC_ERR_CAPACITY",
             -5: "SPEC_ERR_ROOT", -6: "SPEC_ERR_CUDA", -7: "SPEC_ERR_TIMEOUT", -8: "SPEC_ERR_STATE",
             -9: "SPEC_ERR_RANGE"}


class spec_config(ctypes.Structure):
    _fields_ = [
        ("n_layers", ctypes.c_int32), ("hidden", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32),
        ("vocab", ctypes.c_int32), ("dtype", ctypes.c_int32), ("rms_eps", ctypes.c_float),
        ("rope_theta", ctypes.c_float), ("max_batch", ctypes.c_int32), ("max_seq", ctypes.c_int32),
        ("max_nodes", ctypes.c_int32), ("draft_head", ctypes.c_int32),
        ("feature_layers", ctypes.c_int32 * 3), ("draft_vocab", ctypes.c_int32),
    ]


class spec_layer_weights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in
                ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "attn_norm", "mlp_norm")]


class spec_weights(ctypes.Structure):
    _fields_ = [
        ("embed", ctypes.c_void_p), ("final_norm", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
        ("layers", ctypes.POINTER(spec_layer_weights)),
        ("draft_fc_fuse", ctypes.c_void_p), ("draft_fc_in", ctypes.c_void_p),
        ("draft_layer", ctypes.POINTER(spec_layer_weights)), ("draft_final_norm", ctypes.c_void_p),
        ("draft_lm_head", ctypes.c_void_p), ("draft_vocab_ids", ctypes.c_void_p),
    ]


_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)
_vp = ctypes.c_void_p
_h = ctypes.c_void_p

_SIGNATURES = {
    "spec_kv_bytes": (ctypes.c_size_t, [ctypes.POINTER(spec_config)]),
    "spec_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(spec_config)]),
    "spec_init": (ctypes.c_int, [ctypes.POINTER(spec_config), ctypes.POINTER(spec_weights), _vp, ctypes.c_size_t,
                                 _vp, ctypes.c_size_t, _vp, ctypes.POINTER(_h)]),
    "spec_prefill": (ctypes.c_int, [_h, ctypes.c_int, _i32p, ctypes.c_int, _i32p]),
    "spec_prefill_features": (ctypes.c_int, [_h, ctypes.c_int, _i32p, ctypes.c_int, _i32p, _vp]),
    "spec_verify_tree": (ctypes.c_int, [_h, ctypes.c_int, _i32p, _i32p, ctypes.c_int, _i32p, _i32p, _i32p]),
    "spec_verify_tree_batch": (ctypes.c_int, [_h, ctypes.c_int, _i32p, _i32p, _i32p, _i32p, _vp, _vp, _vp, _vp,
                                              ctypes.c_int]),
    "spec_score_trees": (ctypes.c_int, [_h, ctypes.c_int, _i32p, _i32p, _i32p, _i32p, _i32p, _f32p, _f32p,
                                        ctypes.c_int]),
    "spec_set_debug_logits": (ctypes.c_int, [_h, _vp, ctypes.c_size_t]),
    "spec_set_sampling": (ctypes.c_int, [_h, ctypes.c_float, ctypes.c_uint64]),
    "spec_set_feature_out": (ctypes.c_int, [_h, _vp, ctypes.c_size_t]),
    "spec_truncate": (ctypes.c_int, [_h, ctypes.c_int, ctypes.c_int]),
    "spec_seq_len": (ctypes.c_int, [_h, ctypes.c_int, _i32p, _i32p]),
    "spec_sync": (ctypes.c_int, [_h]),
    "spec_validate_tree": (ctypes.c_int, [_i32p, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "spec_profile": (ctypes.c_int, [_h, ctypes.c_int]),
    "spec_profile_read": (ctypes.c_int, [_h, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]),
    "spec_step_launches": (ctypes.c_int, [_h]),
    "spec_set_trace": (ctypes.c_int, [_h, _vp, ctypes.c_size_t, ctypes.c_int]),
    "spec_info": (ctypes.c_int, [_h, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_char_p, ctypes.c_size_t]),
    "spec_io_bytes": (ctypes.c_int, [_h, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]),
    "spec_lm_head_argmax_noalloc": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_float, _vp, _vp, _vp, _vp]),
    "spec_draft_prefill": (ctypes.c_int, [_h, ctypes.c_int, _vp, _i32p, ctypes.c_int]),
    "spec_draft_step": (ctypes.c_int, [_h, ctypes.c_int, _i32p, _vp, _i32p, _i32p, _i32p, _vp, _vp, ctypes.c_int]),
    "spec_draft_len": (ctypes.c_int, [_h, ctypes.c_int, _i32p]),
    "spec_draft_append": (ctypes.c_int, [_h, ctypes.c_int, _vp, _i32p, ctypes.c_int]),
    "spec_draft_tree": (ctypes.c_int, [_h, ctypes.c_int, _i32p, _vp, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       _i32p, _i32p, _f32p]),
    "spec_wait_selftest": (ctypes.c_int, [_vp, ctypes.c_uint32, _i32p]),
    "spec_last_error": (ctypes.c_char_p, [_h]),
    "spec_free": (None, [_h]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libspec.so (built by speculative_decoding_06_b200.build); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libspec.so is not built; run `python -m speculative_decoding_06_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def declared_symbols():
    return list(_SIGNATURES)


class SpecError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("%s: %s" % (ERR_NAMES.get(code, str(code)), msg))
        self.code = code


def _bind(name):
    def call(*args):
        return getattr(lib(), name)(*args)
    call.__name__ = name
    return call


# one Python function per C entry point, same name
for _name in _SIGNATURES:
    globals()[_name] = _bind(_name)
del _name
