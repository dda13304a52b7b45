"""ctypes binding of libcsa.so (the C ABI declared in include/csa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. Loading fails loudly if the library has not been built; there is no
fallback.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcsa.so")

CSA_OK = 0
CSA_DTYPE_F32 = 0
CSA_DTYPE_BF16 = 1
CSA_DTYPE_E4M3 = 2
CSA_MAX_TOPK = 2048
CSA_STEP_CHAINED = 0
CSA_STEP_PERSISTENT = 1

# Every function the header declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
_LL = ctypes.c_longlong
_F = ctypes.c_float
_SZ = ctypes.c_size_t
SIGNATURES = {
    "csa_strerror": (ctypes.c_char_p, [_I]),
    "csa_compress": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _I, _I, _I, _LL, _LL, _LL, _I, _P]),
    "csa_compress_rope": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _I, _I, _I, _LL, _LL, _LL, _I, ctypes.c_double, _P, _I,
                               _P]),
    "csa_index_compress": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P, _I, _I, _I, _LL, _LL, _LL, _I, _I, _P]),
    "csa_hadamard_rows": (_I, [_P, _P, _P, _LL, _I, _I, _I, _P]),
    "csa_index_topk_workspace_bytes": (_SZ, [_I, _I, _I]),
    "csa_index_topk": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "csa_index_scores": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "csa_index_scores_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "csa_index_topk_fp8": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "csa_topk_workspace_bytes": (_SZ, [_I, _I, _I]),
    "csa_topk": (_I, [_P, _P, _I, _P, _I, _I, _P, _SZ, _P]),
    "csa_mqa_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "csa_sparse_mqa": (_I, [_P, _P, _P, _P, _P, _F, _P, _I, _I, _I, _I, _I, _I, _I, _P, _I, _I, _I, _P, _SZ, _P]),
    "hca_mqa": (_I, [_P, _P, _P, _P, _F, _P, _I, _I, _I, _I, _I, _P, _I, _P, _I, _I, _I, _P, _SZ, _P]),
    "csa_topk_sparse_mqa_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "csa_topk_sparse_mqa": (_I, [_P, _P, _I, _P, _P, _P, _P, _P, _F, _P, _I, _I, _I, _I, _I, _I, _P, _I, _I, _I, _P,
                                 _SZ, _P]),
    "csa_workspace_status": (_I, [_P, _P, ctypes.POINTER(ctypes.c_uint32)]),
    "csa_launch_count": (ctypes.c_ulonglong, []),
    "csa_index_topk_noalloc": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _P]),
    "csa_num_entries": (_LL, [_LL, _I, _I]),
    "csa_last_cuda_error": (_I, []),
    "csa_cuda_error_string": (ctypes.c_char_p, [_I]),
    "csa_visible_counts_host": (_I, [_P, _LL, _I, _I, _P]),
    "csa_visible_counts": (_I, [_P, _LL, _I, _I, _P, _P]),
}



class DecodeStepArgs(ctypes.Structure):
    """csa_decode_step_args (include/csa.h), field for field."""
    _fields_ = [
        ("q", _P), ("kv_cmp", _P), ("kv_win", _P), ("win_end", _P), ("sink", _P), ("out", _P), ("n_cmp", _P),
        ("qi", _P), ("sq", _P), ("wi", _P), ("ki", _P), ("sk", _P), ("idx_out", _P),
        ("app_kv", _P), ("app_gate", _P), ("ape", _P), ("norm_w", _P), ("pos0", _P),
        ("scale", _F),
        ("Q", _I), ("B", _I), ("H", _I), ("D", _I), ("N_max", _I), ("win_len", _I), ("T_raw", _I),
        ("q_per_seq", _I), ("dtype", _I),
        ("index_dtype", _I), ("Hi", _I), ("Di", _I), ("k", _I),
        ("app_win", _I), ("app_stride", _I), ("app_T", _I), ("rope_dims", _I),
        ("app_kv_seq_stride", _LL), ("app_gate_seq_stride", _LL), ("app_row0", _LL),
        ("rope_theta", ctypes.c_double),
        ("variant", _I),
    ]


SIGNATURES["csa_decode_step_workspace_bytes"] = (_SZ, [ctypes.POINTER(DecodeStepArgs)])
SIGNATURES["csa_decode_step"] = (_I, [ctypes.POINTER(DecodeStepArgs), _P, _SZ, _P])

_lib = None


class CsaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        msg = f"{fn} failed: {strerror(code)}"
        if code == 4:  # CSA_ERR_CUDA: name the CUDA error behind it
            e = lib().csa_last_cuda_error()
            msg += f" ({e}: {lib().csa_cuda_error_string(e).decode()})"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """The loaded library (raises if libcsa.so is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is not built; run `python -m compressed_sparse_attention_15_b200.build` "
                "(the CUDA kernels are the only implementation of this path)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().csa_strerror(code).decode()


def check(fn: str, code: int) -> None:
    if code != CSA_OK:
        raise CsaError(fn, code)
