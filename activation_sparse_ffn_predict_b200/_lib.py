"""ctypes binding of libasffn.so (include/asffn.h).  Argument marshalling only."""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int32, c_int64, c_size_t, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libasffn.so")

ASF_OK = 0
ASF_ERR_INVALID_ARG = 1
ASF_ERR_MISALIGNED = 2
ASF_ERR_UNSUPPORTED = 3
ASF_ERR_CUDA = 4
ASF_ERR_DEVICE_INDEX = 5
ASF_ERR_TIMEOUT = 6
ASF_ERR_WORKSPACE = 7

ASF_F32 = 0
ASF_F16 = 1
ASF_ACT_RELU = 0
ASF_ACT_REGLU = 1
ASF_MAX_BATCH = 32
ASF_NOALLOC_SCRATCH_BYTES = 32 << 20
ASF_INJECT_NONE = 0
ASF_INJECT_WITHHOLD_FFN_COPIES = 1


class asf_predictor(ctypes.Structure):
    _fields_ = [("d", c_int32), ("r", c_int32), ("n", c_int32), ("wdtype", c_int),
                ("W1", c_void_p), ("b1", c_void_p), ("W2", c_void_p), ("b2", c_void_p)]


class asf_ffn(ctypes.Structure):
    _fields_ = [("d", c_int32), ("n", c_int32), ("wdtype", c_int), ("act", c_int),
                ("Wg", c_void_p), ("Wu", c_void_p), ("WdT", c_void_p), ("bias", c_void_p),
                ("hot_rows", c_int32), ("row_stride", c_int32),
                ("l2_next", c_void_p * 2), ("l2_next_bytes", ctypes.c_int64 * 2)]


ASF_MAX_PEERS = 8


class asf_peer_group(ctypes.Structure):
    _fields_ = [("world", c_int32), ("rank", c_int32), ("max_batch", c_int32), ("d", c_int32),
                ("pub", c_void_p * ASF_MAX_PEERS), ("flag", c_void_p * ASF_MAX_PEERS), ("epoch", c_void_p)]


# name -> (restype, argtypes), exactly the declarations of include/asffn.h
PROTOTYPES = {
    "asf_workspace_bytes": (c_size_t, [POINTER(asf_predictor), POINTER(asf_ffn), c_int32]),
    "asf_workspace_init": (c_int, [c_void_p, c_size_t, c_void_p]),
    "asf_predict": (c_int, [POINTER(asf_predictor), c_void_p, c_int32, c_float, c_void_p, c_void_p,
                            c_void_p, c_size_t, c_void_p]),
    "asf_sparse_ffn": (c_int, [POINTER(asf_ffn), c_void_p, c_int32, c_void_p, c_void_p, c_void_p,
                               c_void_p, c_size_t, c_void_p]),
    "asf_predict_sparse_ffn": (c_int, [POINTER(asf_predictor), POINTER(asf_ffn), c_void_p, c_int32, c_float,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "asf_predict_sparse_ffn_begin": (c_int, [POINTER(asf_predictor), POINTER(asf_ffn), c_void_p, c_int32,
                                             c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                             c_void_p]),
    "asf_predict_sparse_ffn_end": (c_int, [POINTER(asf_predictor), POINTER(asf_ffn), c_void_p, c_int32,
                                           c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                           c_void_p]),
    "asf_predict_sparse_ffn_exchange": (c_int, [POINTER(asf_predictor), POINTER(asf_ffn), c_void_p, c_int32,
                                                c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                                POINTER(asf_peer_group), c_void_p]),
    "asf_reduce_exchange": (c_int, [c_void_p, c_int64, c_int32, c_int32, c_int32, POINTER(asf_peer_group),
                                    c_int32, c_void_p, c_int64, c_void_p, c_size_t, c_void_p]),
    "asf_set_fault_injection": (c_int, [c_int32]),
    "asf_dense_ffn": (c_int, [POINTER(asf_ffn), c_void_p, c_int32, c_void_p, c_void_p, c_size_t,
                              c_void_p]),
    "asf_activation_counts": (c_int, [POINTER(asf_ffn), c_void_p, c_int32, c_void_p, c_void_p,
                                      c_size_t, c_void_p]),
    "asf_hot_permutation": (c_int, [POINTER(c_int64), c_int32, POINTER(c_int32)]),
    "asf_permute_rows": (c_int, [c_void_p, c_void_p, c_int32, c_int64, c_void_p, c_void_p]),
    "asf_gather_rows": (c_int, [c_void_p, c_int64, c_int32, c_void_p, c_int64, c_int32, c_int64, c_void_p,
                                c_void_p]),
    "asf_sparse_ffn_noalloc": (c_int, [POINTER(asf_ffn), c_void_p, c_int32, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p]),
    "asf_read_error": (c_int, [c_void_p, POINTER(c_int32), c_void_p]),
    "asf_status_string": (c_char_p, [c_int]),
    "asf_version": (c_int32, []),
}

_LIB = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libasffn.so once.  Raises if the library has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"libasffn.so is not built ({path}); run "
                           "`python -m activation_sparse_ffn_predict_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


class AsfError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        msg = load().asf_status_string(self.status).decode()
        super().__init__(f"{where}: {msg} (status {self.status})")


def check(status: int, where: str) -> None:
    if status != ASF_OK:
        raise AsfError(status, where)
