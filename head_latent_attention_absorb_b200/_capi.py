"""ctypes declarations of libmla_b200.so (the C ABI in include/mla_api.h).

Loading fails loudly when the library is missing: there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla_b200.so")

c_i32, c_i64, c_sz, c_f32, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p
c_i32p = ctypes.POINTER(ctypes.c_int32)
c_f32p = ctypes.POINTER(ctypes.c_float)

MLA_F32, MLA_BF16 = 0, 1
STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_CUDA",
          4: "MLA_ERR_INDEX", 5: "MLA_ERR_TIMEOUT", 6: "MLA_ERR_WORKSPACE", 7: "MLA_ERR_LENGTH"}
ABI_VERSION = 1


class MLADims(ctypes.Structure):
    _fields_ = [("n_h", c_i32), ("d_c", c_i32), ("d_r", c_i32), ("d_h", c_i32), ("d_v", c_i32)]


# name -> (restype, argtypes), in the order of include/mla_api.h
SIGNATURES = {
    "mla_abi_version": (c_i32, []),
    "mla_status_string": (ctypes.c_char_p, [c_i32]),
    "mla_last_error_message": (ctypes.c_char_p, []),
    "mla_absorb_q": (c_i32, [MLADims, c_i32, c_i32, c_vp, c_i64, c_vp, c_vp, c_vp]),
    "mla_decode_workspace_size": (c_sz, [MLADims, c_i32, c_i32, c_i32, c_i32]),
    "mla_decode_num_launches": (c_i32, [MLADims, c_i32, c_i32, c_i32, c_i32]),
    "mla_decode_absorb": (c_i32, [MLADims, c_i32, c_i32,
                                  c_vp, c_i64, c_vp, c_i64,
                                  c_vp, c_i64, c_i64, c_vp, c_i64, c_i64,
                                  c_i32, c_vp, c_vp, c_i32,
                                  c_f32, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "mla_decode_absorb_fp8kv": (c_i32, [MLADims, c_i32, c_vp, c_i64, c_vp, c_i64,
                                        c_vp, c_i64, c_i64, c_vp, c_i64, c_i64, c_vp, c_i64, c_i64,
                                        c_i32, c_vp, c_f32, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "mla_decode_absorb_multi": (c_i32, [MLADims, c_i32, c_i32, c_i32,
                                        c_vp, c_i64, c_vp, c_i64,
                                        c_vp, c_i64, c_i64, c_vp, c_i64, c_i64,
                                        c_i32, c_vp, c_f32, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "mla_decode_absorb_multi_topk": (c_i32, [MLADims, c_i32, c_i32, c_i32,
                                             c_vp, c_i64, c_vp, c_i64,
                                             c_vp, c_i64, c_i64, c_vp, c_i64, c_i64,
                                             c_i32, c_vp, c_vp, c_i32, c_f32, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "mla_decode_absorb_static": (c_i32, [MLADims, c_i32, c_i32,
                                         c_vp, c_i64, c_vp, c_i64,
                                         c_vp, c_i64, c_i64, c_vp, c_i64, c_i64,
                                         c_i32, c_vp, c_f32, c_vp, c_vp, c_vp, c_vp]),
    "mla_out_up": (c_i32, [MLADims, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "mla_absorb_q_fp8": (c_i32, [MLADims, c_i32, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "mla_out_up_fp8": (c_i32, [MLADims, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "mla_prefill_workspace_size": (c_sz, [MLADims, c_i32, c_i32, c_i32]),
    "mla_prefill_naive": (c_i32, [MLADims, c_i32, c_i32, c_i32, c_vp, c_vp, c_i64, c_vp, c_i64, c_vp,
                                  c_f32, c_i32, c_vp, c_vp, c_sz, c_vp]),
    "mla_cache_append": (c_i32, [MLADims, c_i32, c_i32, c_vp, c_i64, c_vp, c_f32, c_f32, c_vp, c_i32,
                                 c_vp, c_i64, c_i64, c_vp, c_i64, c_i64, c_vp, c_vp]),
    "mla_check_topk": (c_i32, [c_i32, c_vp, c_i32, c_vp, c_i32, c_vp, c_vp]),
    "mla_prefill_sparse_workspace_size": (c_sz, [MLADims, c_i32, c_i32, c_i32]),
    "mla_prefill_sparse": (c_i32, [MLADims, c_i32, c_i32, c_i32, c_vp, c_vp, c_i64, c_vp, c_i64, c_vp,
                                   c_f32, c_vp, c_i32, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "mla_selftest_wait_timeout": (c_i32, [ctypes.c_uint64, c_vp, c_vp]),
    "mla_clear_device_error": (c_i32, [c_vp, c_vp]),
    "mla_get_device_error": (c_i32, [c_vp, c_i32p]),
}

_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """The loaded library with every signature declared.  Raises if it is not built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m head_latent_attention_absorb_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(L, name)
                f.restype, f.argtypes = res, args
            if L.mla_abi_version() != ABI_VERSION:
                raise RuntimeError(f"libmla_b200.so ABI {L.mla_abi_version()} != {ABI_VERSION}")
            _lib = L
    return _lib


class MLAError(RuntimeError):
    def __init__(self, status: int, where: str):
        L = lib()
        self.status = status
        msg = L.mla_last_error_message().decode()
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")


def check(status: int, where: str) -> None:
    if status != 0:
        raise MLAError(status, where)
