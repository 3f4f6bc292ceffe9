"""ctypes view of libeq.so (include/eq.h, include/eq_encode.h): structures and raw entry points.

Argument marshalling only.  Every step of the decode path runs in the library's CUDA kernels;
if the library cannot be built or loaded this module raises instead of falling back.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

from . import build as _build

EQ_OK, EQ_ERR_ARG, EQ_ERR_FORMAT, EQ_ERR_UNSUPPORTED, EQ_ERR_CUDA = 0, 1, 2, 3, 4
EQ_DEV_CORRUPT_STATE, EQ_DEV_OVERRUN, EQ_DEV_BAD_CODE = 1, 2, 4
EQ_DEV_COUNT_MISMATCH, EQ_DEV_TIMEOUT = 8, 16
EQ_SYM_E4M3, EQ_SYM_INT8 = 1, 2
EQ_TABLE_RANS, EQ_TABLE_HUFF, EQ_TABLE_RANS_PAIR_E4M3, EQ_TABLE_RANS_PAIR_INT8 = 1, 2, 3, 4
EQ_TABLE_RANS8_E4M3, EQ_TABLE_RANS8_INT8 = 5, 6
EQ_ABI_VERSION = 3

# every exported function of include/eq.h and include/eq_encode.h
EXPORTS = ("eq_table_bytes", "eq_build_tables", "eq_decode", "eq_decode_from_host", "eq_decode_gemv",
           "eq_huff_bf16_decode", "eq_huff_int_decode", "eq_mlp_scratch_bytes", "eq_mlp_decode", "eq_mlp_decode_noalloc", "eq_selftest_bounded_wait",
           "eq_status_string",
           "eq_abi_version", "eq_quantize_host", "eq_super_weights_host", "eq_quantize_excluding_host",
           "eq_rans_freqs_host", "eq_rans_encode_host", "eq_huff_lengths_host",
           "eq_huff_plan_host", "eq_huff_encode_host", "eq_free_host", "eq_rans_normalize_host",
           "eq_quantize_device", "eq_intq_quantize_host", "eq_huff_sym_plan_host",
           "eq_huff_sym_encode_host",
           "eq_histogram_device", "eq_rans_plan_device", "eq_rans_encode_device")


class EqError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})" if what else status_string(code))


class RansTensorDesc(C.Structure):
    """eq_rans_tensor"""
    _fields_ = [("version", C.c_uint32), ("symfmt", C.c_uint32), ("rows", C.c_uint32),
                ("cols", C.c_uint32), ("prob_bits", C.c_uint32), ("chunk_symbols", C.c_uint32),
                ("streams", C.c_uint32), ("run", C.c_uint32), ("num_chunks", C.c_uint64),
                ("states", C.c_void_p), ("word_off", C.c_void_p), ("words", C.c_void_p),
                ("scales", C.c_void_p), ("tables", C.c_void_p), ("n_patch", C.c_uint64),
                ("patch_idx", C.c_void_p), ("patch_val", C.c_void_p)]


class HuffTensorDesc(C.Structure):
    """eq_huff_tensor"""
    _fields_ = [("n", C.c_uint64), ("total_bits", C.c_uint64), ("bytes_per_thread", C.c_uint32),
                ("threads_per_block", C.c_uint32), ("enc_exp", C.c_void_p),
                ("sign_mant", C.c_void_p), ("gaps", C.c_void_p), ("block_out", C.c_void_p),
                ("tables", C.c_void_p)]


class HuffIntTensorDesc(C.Structure):
    """eq_huff_int_tensor"""
    _fields_ = [("n", C.c_uint64), ("total_bits", C.c_uint64), ("bytes_per_thread", C.c_uint32),
                ("threads_per_block", C.c_uint32), ("enc", C.c_void_p), ("gaps", C.c_void_p),
                ("block_out", C.c_void_p), ("tables", C.c_void_p), ("bits", C.c_uint32),
                ("zero", C.c_int32), ("scale", C.c_uint16), ("reserved16", C.c_uint16),
                ("reserved32", C.c_uint32)]


EQ_INTQ_ASYM, EQ_INTQ_UNSIGNED = 0, 1

_lib = None
_lock = threading.Lock()


def lib() -> C.CDLL:
    """Load libeq.so from the source tree, compiling it first if a source is newer."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            if not os.path.exists(path):
                raise RuntimeError(f"libeq.so missing at {path}")
            L = C.CDLL(path)
            p, u32, u64, i32 = C.c_void_p, C.c_uint32, C.c_uint64, C.c_int
            sig = {
                "eq_table_bytes": (C.c_size_t, [i32]),
                "eq_build_tables": (i32, [i32, p, u32, p, p]),
                "eq_decode": (i32, [p, u32, p, p, p]),
                "eq_decode_from_host": (i32, [p, p, p, p, u64, p, u32, p, p, p, p]),
                "eq_decode_gemv": (i32, [p, p, u32, p, p, p]),
                "eq_huff_bf16_decode": (i32, [p, p, p, p]),
                "eq_huff_int_decode": (i32, [p, p, p, p]),
                "eq_intq_quantize_host": (i32, [p, u64, u32, u32, p, p, p]),
                "eq_huff_sym_plan_host": (i32, [p, u64, p, C.POINTER(C.c_uint64)]),
                "eq_huff_sym_encode_host": (i32, [p, u64, p, u32, u64, p, p, p]),
                "eq_mlp_scratch_bytes": (C.c_size_t, [u32, u32]),
                "eq_mlp_decode": (i32, [p, p, p, p, u32, p, p, C.c_size_t, p, p]),
                "eq_mlp_decode_noalloc": (i32, [p, p, p, p, u32, p, p, p]),
                "eq_selftest_bounded_wait": (i32, [p, p]),
                "eq_status_string": (C.c_char_p, [i32]),
                "eq_abi_version": (u32, []),
                "eq_quantize_host": (i32, [p, u32, u32, u32, C.c_float, p, p, u32]),
                "eq_super_weights_host": (i32, [p, u32, u32, C.c_double, u64, p, p,
                                                C.POINTER(C.c_uint64)]),
                "eq_quantize_excluding_host": (i32, [p, u32, u32, u32, C.c_float, p, u64, p, p,
                                                     u32]),
                "eq_rans_freqs_host": (i32, [p, u64, u32, p]),
                "eq_rans_encode_host": (i32, [p, u32, u32, p, u32, u32, u32, u32, p, p,
                                              C.POINTER(C.c_void_p), C.POINTER(C.c_uint64)]),
                "eq_huff_lengths_host": (i32, [p, u32, p]),
                "eq_huff_plan_host": (i32, [p, u64, p, C.POINTER(C.c_uint64)]),
                "eq_huff_encode_host": (i32, [p, u64, p, u32, u64, p, p, p, p]),
                "eq_free_host": (None, [p]),
                "eq_rans_normalize_host": (i32, [p, u32, p]),
                "eq_quantize_device": (i32, [p, u32, u32, u32, C.c_float, p, p, p]),
                "eq_histogram_device": (i32, [p, u64, p, p]),
                "eq_rans_plan_device": (i32, [p, u32, u32, p, u32, u32, u32, p, p, p, p]),
                "eq_rans_encode_device": (i32, [p, u32, u32, p, u32, u32, u32, p, p, p, p]),
            }
            for name, (res, args) in sig.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            if L.eq_abi_version() != EQ_ABI_VERSION:
                raise RuntimeError("libeq.so ABI version mismatch")
            _lib = L
    return _lib


def status_string(code: int) -> str:
    try:
        return lib().eq_status_string(int(code)).decode()
    except Exception:  # noqa: BLE001 -- used while formatting another error
        return f"status {code}"


def check(code: int, what: str = "") -> None:
    if code != EQ_OK:
        raise EqError(code, what)
