"""CPU oracle for the anti-quant weight GEMM and its int8 sibling.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package; the product
path never does.  The arithmetic lives in ``wqmm_oracle.c`` (plain C, fp64),
which shares no code with the CUDA path; this module only builds it with gcc
and marshals numpy arrays into it.

Parity status of each oracle function (what pins it, see the tests):
  * ``wqmm``  -- pinned: exact rational brute force, page sample closed form
    (all-ones fp16 case -> 130), reductions to a library matmul, invariants.
  * ``qmm``   -- pinned: exact integer brute force, page sample closed form
    (all-ones int8 case -> 66), numpy int64 matmul.
  * format codecs -- pinned against numpy fp16, torch bf16 / fp8-e4m3fn and
    exact rational rounding.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wqmm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libwqmm_oracle.so")
_lock = threading.Lock()
_lib = None

F16, BF16, F32, I8, I4, FP8E4M3 = 1, 2, 3, 4, 5, 7
_ACT = {"f16": F16, "bf16": BF16}
_WDT = {"i8": I8, "i4": I4, "fp8": FP8E4M3, "f16": F16, "bf16": BF16}  # f16/bf16: non-quantised
_MODE = {"tensor": 0, "channel": 1, "group": 2, "none": 0}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, IEEE semantics: no fp contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", _LIB_PATH + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
            L.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
            L.oracle_f16_to_double.restype = D
            L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            L.oracle_bf16_to_double.restype = D
            L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            L.oracle_e4m3_to_double.restype = D
            L.oracle_double_to_f16.argtypes = [D]
            L.oracle_double_to_f16.restype = ctypes.c_uint16
            L.oracle_double_to_bf16.argtypes = [D]
            L.oracle_double_to_bf16.restype = ctypes.c_uint16
            L.oracle_weight_at.argtypes = [I32, P, I64, I64, I64, I64]
            L.oracle_weight_at.restype = D
            L.oracle_wqmm.argtypes = [I64, I64, I64, I32, P, I32, P, I64, I64, I32, I64, P, P, I64, I64,
                                      P, P, I64, P, I64, P, P, P]
            L.oracle_wqmm.restype = I32
            L.oracle_qmm.argtypes = [I64, I64, I64, P, P, I64, I64, P, I32, P, I64, P, I32, P,
                                     I64, P, I64, P, P, P, P]
            L.oracle_qmm.restype = I32
            L.oracle_num_threads.argtypes = []
            L.oracle_num_threads.restype = I32
            _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# ----------------------------------------------------------------- scalar codecs
def f16_to_double(bits: int) -> float:
    return lib().oracle_f16_to_double(int(bits))


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits))


def e4m3_to_double(bits: int) -> float:
    return lib().oracle_e4m3_to_double(int(bits))


def double_to_f16(x: float) -> int:
    return int(lib().oracle_double_to_f16(float(x)))


def double_to_bf16(x: float) -> int:
    return int(lib().oracle_double_to_bf16(float(x)))


def weight_at(wdt: str, x2: np.ndarray, s0: int, s1: int, kk: int, nn: int) -> float:
    x2 = np.ascontiguousarray(x2)
    return lib().oracle_weight_at(_WDT[wdt], _p(x2), s0, s1, kk, nn)


# ----------------------------------------------------------------- wqmm
def wqmm_raw(*, m, k, n, act, x1, wdt, x2, x2_strides, mode, group_size, scale, offset, scale_strides,
             bias=None, x3=None, rows: Optional[Sequence[int]] = None, cols: Optional[Sequence[int]] = None):
    """Evaluate the anti-quant GEMM on the selected rows x cols.
    Returns (y_exact float64 [R, C], y_rounded uint16 [R, C] in the activation format)."""
    x1 = np.ascontiguousarray(x1, dtype=np.uint16)
    x2 = np.ascontiguousarray(x2)
    scale = None if scale is None else np.ascontiguousarray(scale, dtype=np.uint16)
    offset = None if offset is None else np.ascontiguousarray(offset, dtype=np.uint16)
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
    x3 = None if x3 is None else np.ascontiguousarray(x3, dtype=np.uint16)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    R = m if r is None else len(r)
    C = n if c is None else len(c)
    ye = np.empty((R, C), dtype=np.float64)
    yr = np.empty((R, C), dtype=np.uint16)
    rc = lib().oracle_wqmm(m, k, n, _ACT[act], _p(x1), _WDT[wdt], _p(x2), int(x2_strides[0]), int(x2_strides[1]),
                           _MODE[mode], int(group_size), _p(scale), _p(offset), int(scale_strides[0]),
                           int(scale_strides[1]), _p(bias), _p(x3), R, _p(r), C, _p(c), _p(ye), _p(yr))
    if rc != 0:
        raise ValueError("oracle_wqmm rejected its arguments")
    return ye, yr


def wqmm(case, rows=None, cols=None):
    """Oracle for a ``workloads.WqmmCase`` (output flattened to (m, n) / sampled)."""
    return wqmm_raw(m=case.m, k=case.k, n=case.n, act=case.act, x1=case.x1, wdt=case.wdt, x2=case.x2,
                    x2_strides=case.x2_strides, mode=case.mode, group_size=case.group_size, scale=case.scale,
                    offset=case.offset, scale_strides=case.scale_strides, bias=case.bias, x3=case.x3,
                    rows=rows, cols=cols)


# ----------------------------------------------------------------- qmm
def qmm_raw(*, m, k, n, x1, x2, x2_strides, bias, dq_dtype, dequant_scale, pertoken, out, x3,
            rows=None, cols=None):
    """Evaluate the int8 GEMM on the selected rows x cols.
    Returns (acc int32 [R, C], y_exact float64 [R, C], y_rounded uint16 [R, C])."""
    x1 = np.ascontiguousarray(x1, dtype=np.int8)
    x2 = np.ascontiguousarray(x2, dtype=np.int8)
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.int32)
    dq = np.ascontiguousarray(dequant_scale, dtype=np.uint16 if dq_dtype == "bf16" else np.float32)
    pt = None if pertoken is None else np.ascontiguousarray(pertoken, dtype=np.float32)
    x3 = None if x3 is None else np.ascontiguousarray(x3, dtype=np.uint16)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    R = m if r is None else len(r)
    C = n if c is None else len(c)
    acc = np.empty((R, C), dtype=np.int32)
    ye = np.empty((R, C), dtype=np.float64)
    yr = np.empty((R, C), dtype=np.uint16)
    rc = lib().oracle_qmm(m, k, n, _p(x1), _p(x2), int(x2_strides[0]), int(x2_strides[1]), _p(bias),
                          BF16 if dq_dtype == "bf16" else F32, _p(dq), int(dq.size), _p(pt), _ACT[out], _p(x3),
                          R, _p(r), C, _p(c), _p(acc), _p(ye), _p(yr))
    if rc != 0:
        raise ValueError("oracle_qmm rejected its arguments")
    return acc, ye, yr


def qmm(case, rows=None, cols=None):
    """Oracle for a ``workloads.QmmCase``."""
    return qmm_raw(m=case.m, k=case.k, n=case.n, x1=case.x1, x2=case.x2, x2_strides=case.x2_strides,
                   bias=case.bias, dq_dtype=case.dq_dtype, dequant_scale=case.dequant_scale,
                   pertoken=case.pertoken_scale, out=case.out, x3=case.x3, rows=rows, cols=cols)
