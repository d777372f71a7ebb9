"""ctypes view of the C ABI declared in include/tq.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# TQ_LIBRARY may point at another build of the same C ABI (e.g. a tuning variant).
LIB_PATH = os.environ.get("TQ_LIBRARY") or os.path.join(_HERE, "libtq_b200.so")

(TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_WORKSPACE, TQ_ERR_CUDA, TQ_ERR_DEVICE_BOUNDS,
 TQ_ERR_SCRATCH_LIMIT) = range(7)
TQ_NOALLOC_SCRATCH_BYTES = 64 << 20
TQ_DEV_POS_RANGE, TQ_DEV_NORM_OVERFLOW, TQ_DEV_LEN_RANGE, TQ_DEV_INTERNAL, TQ_DEV_CHANNEL_RANGE = 1, 2, 4, 8, 16
TQ_MAX_OUTLIERS = 16
TQ_F32, TQ_F16 = 0, 1
TQ_MAX_QUERY_TOKENS = 16

# Every symbol include/tq.h declares, with (restype, argtypes).
c_int, c_float, c_size_t, c_void_p = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p


class Codebook(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32),
                ("centroids", ctypes.c_float * 16),
                ("boundaries", ctypes.c_float * 15)]


class KVDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("seq_cap", ctypes.c_int32),
                ("sign_seed", ctypes.c_uint64),
                ("k_bits", ctypes.c_int32), ("v_bits", ctypes.c_int32)]


class VOutliers(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int32), ("channels", c_void_p), ("values", c_void_p)]


_P = ctypes.POINTER
SIGNATURES = {
    "tq_make_codebook": (c_int, [c_int, _P(Codebook)]),
    "tq_sign_vector": (c_int, [ctypes.c_uint64, c_void_p]),
    "tq_encode_kv": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_void_p, c_void_p, c_int, c_int,
                             c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "tq_decode_workspace_size": (c_size_t, [_P(KVDesc), c_int, c_float]),
    "tq_decode_attention": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_int, c_void_p, c_int,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_float,
                                    c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "tq_decode_attention_multi": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_int, c_int, c_void_p,
                                          c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float,
                                          c_float, c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "tq_decode_step": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_int, c_void_p, c_int,
                               c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_void_p, c_float, c_float, c_void_p, c_void_p, c_size_t, c_void_p,
                               c_void_p]),
    "tq_decode_attention_noalloc": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_int, c_void_p,
                                            c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                            c_float, c_float, c_void_p, c_void_p, c_void_p]),
    "tq_read_device_status": (c_int, [c_void_p, c_void_p, c_void_p]),
    "tq_pick_outlier_channels": (c_int, [_P(KVDesc), c_void_p, c_int, c_int, c_int, c_void_p, c_void_p]),
    "tq_encode_kv_v3": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_void_p, c_void_p, c_int, c_int,
                                c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, _P(VOutliers), c_void_p,
                                c_void_p]),
    "tq_encode_kv_v2": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_void_p, c_void_p, c_int, c_int,
                                c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "tq_decode_attention_v2": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_int, c_void_p, c_int,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_float,
                                       c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "tq_decode_attention_v3": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_int, c_void_p, c_int,
                                       c_void_p, c_void_p, c_void_p, c_void_p, _P(VOutliers), c_void_p,
                                       c_float, c_float, c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "tq_decode_attention_multi_v3": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_int, c_int,
                                             c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                             _P(VOutliers), c_void_p, c_float, c_float, c_void_p, c_void_p,
                                             c_size_t, c_void_p, c_void_p]),
    "tq_decode_attention_multi_v2": (c_int, [_P(KVDesc), _P(Codebook), _P(Codebook), c_int, c_int,
                                             c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                             c_void_p, c_float, c_float, c_void_p, c_void_p, c_size_t,
                                             c_void_p, c_void_p]),
    "tq_status_string": (ctypes.c_char_p, [c_int]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load the in-tree library; fail loudly if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m quantized_decode_attention_tq_b200.build`"
                " (there is no fallback implementation)")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


class TQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = lib().tq_status_string(status).decode()
        super().__init__(f"{fn} failed: status {status} ({msg})")
        self.status = status


def check(fn: str, status: int) -> None:
    if status != TQ_OK:
        raise TQError(fn, status)
