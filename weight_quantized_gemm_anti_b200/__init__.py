"""Python binding of libwqmm (include/wqmm.h): argument marshalling only.

Every computation runs in the library's CUDA kernels; PyTorch is used for
device memory and streams.  There is no fallback: if ``libwqmm.so`` is missing
the import of the library raises.

Names mirror the C ABI (``wqmm_get_workspace_size``, ``wqmm_run``,
``qmm_get_workspace_size``, ``qmm_run``, ``wqmm_pack_weight_size``,
``wqmm_pack_weight``, ...); each takes :class:`WqmmTensor` descriptors and
returns the C status code.  :func:`weight_quant_matmul` and
:func:`quant_matmul` wrap both phases for torch tensors.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwqmm.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "wqmm.h")

# ---------------------------------------------------------------- constants (from include/wqmm.h)
SUCCESS = 0
ERR_PARAM_NULLPTR = 161001
ERR_PARAM_INVALID = 161002
ERR_INNER_TILING = 561002
ERR_CUDA = 500001
ERR_WORKSPACE = 500002
ERR_EXECUTOR = 500003
ERR_TIMEOUT = 500004

DT_F16, DT_BF16, DT_F32, DT_I8, DT_I4, DT_I32, DT_FP8E4M3, DT_I64, DT_U64 = 1, 2, 3, 4, 5, 6, 7, 8, 9
FORMAT_ND, FORMAT_PACKED = 0, 1


class WqmmError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"wqmm status {status}: {msg}")
        self.status = status


class WqmmTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 3), ("strides", ctypes.c_int64 * 3), ("format", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile libwqmm.so in-tree (nvcc, sm_100a)."""
    from . import buildlib as _b
    return _b.build(force=force)


def lib():
    """The loaded library.  Raises if it has not been built: there is no fallback path."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing; build it with weight_quantized_gemm_anti_b200.build()")
            L = ctypes.CDLL(LIB_PATH)
            T = ctypes.POINTER(WqmmTensor)
            P, I64, I32, U64P = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.POINTER(ctypes.c_uint64)
            EXP = ctypes.POINTER(ctypes.c_void_p)
            L.wqmm_get_workspace_size.argtypes = [T, T, T, T, T, T, ctypes.c_char_p, ctypes.c_char_p, I64, I64, I64,
                                                  T, U64P, EXP]
            L.wqmm_run.argtypes = [P, ctypes.c_uint64, P, P]
            L.qmm_get_workspace_size.argtypes = [T, T, T, T, T, T, ctypes.c_char_p, ctypes.c_char_p, I64, I64, T,
                                                 U64P, EXP]
            L.qmm_run.argtypes = [P, ctypes.c_uint64, P, P]
            L.wqmm_pack_weight_size.argtypes = [T, I32, U64P]
            L.wqmm_pack_weight.argtypes = [T, I32, P, P]
            L.wqmm_executor_destroy.argtypes = [P]
            L.wqmm_executor_destroy.restype = None
            L.wqmm_last_error.restype = ctypes.c_char_p
            L.wqmm_stream_wait.argtypes = [P, I32]
            L.wqmm_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), I32]
            L.wqmm_version.restype = ctypes.c_char_p
            L.qmm_debug_set_raw_accumulator.argtypes = [P, P]
            L.wqmm_debug_set_flag_wait.argtypes = [P, ctypes.c_uint64, I32]
            for name in ("wqmm_get_workspace_size", "wqmm_run", "qmm_get_workspace_size", "qmm_run",
                         "wqmm_pack_weight_size", "wqmm_pack_weight", "wqmm_stream_wait", "wqmm_device_error",
                         "qmm_debug_set_raw_accumulator", "wqmm_debug_set_flag_wait"):
                getattr(L, name).restype = I32
            _lib = L
    return _lib


def header_symbols(path: str = HEADER_PATH) -> list:
    """Names of the functions declared in include/wqmm.h."""
    src = open(path).read()
    return re.findall(r"^WQMM_API\s+[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)


# ---------------------------------------------------------------- descriptors
def _torch_dtype_code(t) -> int:
    import torch
    table = {torch.float16: DT_F16, torch.bfloat16: DT_BF16, torch.float32: DT_F32, torch.int8: DT_I8,
             torch.int32: DT_I32, torch.float8_e4m3fn: DT_FP8E4M3, torch.int64: DT_I64}
    if t.dtype not in table:
        raise TypeError(f"no wqmm dtype for {t.dtype}; pass dtype= explicitly")
    return table[t.dtype]


def desc(t=None, *, data: Optional[int] = None, dtype: Optional[int] = None, shape: Optional[Sequence[int]] = None,
         strides: Optional[Sequence[int]] = None, fmt: int = FORMAT_ND) -> WqmmTensor:
    """Describe a tensor.  For a torch tensor, pointer/shape/strides come from it
    unless given; int4 and packed weights pass dtype and the logical (k, n) shape."""
    d = WqmmTensor()
    if t is not None:
        data = t.data_ptr() if data is None else data
        dtype = _torch_dtype_code(t) if dtype is None else dtype
        if shape is None:
            shape = tuple(t.shape)
            strides = tuple(t.stride()) if strides is None else strides
    if shape is None or dtype is None:
        raise ValueError("shape and dtype are required")
    if strides is None:
        strides, acc = [], 1
        for s in reversed(shape):
            strides.insert(0, acc)
            acc *= s
    d.data = data or 0
    d.dtype = dtype
    d.ndim = len(shape)
    for i, (s, st) in enumerate(zip(shape, strides)):
        d.shape[i] = s
        d.strides[i] = st
    d.format = fmt
    d.reserved = 0
    return d


def _ref(d: Optional[WqmmTensor]):
    return None if d is None else ctypes.byref(d)


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


# ---------------------------------------------------------------- raw ABI
def wqmm_get_workspace_size(x1, x2, bias, antiquant_scale, antiquant_offset, x3, group, reduce_op, comm_turn,
                            stream_mode, antiquant_group_size, output):
    """Returns (status, workspace_size, executor handle or None)."""
    ws = ctypes.c_uint64(0)
    ex = ctypes.c_void_p(None)
    st = lib().wqmm_get_workspace_size(_ref(x1), _ref(x2), _ref(bias), _ref(antiquant_scale),
                                       _ref(antiquant_offset), _ref(x3), None if group is None else group.encode(),
                                       None if reduce_op is None else reduce_op.encode(), int(comm_turn),
                                       int(stream_mode), int(antiquant_group_size), _ref(output), ctypes.byref(ws),
                                       ctypes.byref(ex))
    return st, ws.value, ex.value


def wqmm_run(workspace: int, workspace_size: int, executor, stream=None) -> int:
    return lib().wqmm_run(workspace or None, workspace_size, executor, _stream_handle(stream))


def qmm_get_workspace_size(x1, x2, bias, x3, dequant_scale, pertoken_scale, group, reduce_op, comm_turn,
                           stream_mode, output):
    ws = ctypes.c_uint64(0)
    ex = ctypes.c_void_p(None)
    st = lib().qmm_get_workspace_size(_ref(x1), _ref(x2), _ref(bias), _ref(x3), _ref(dequant_scale),
                                      _ref(pertoken_scale), None if group is None else group.encode(),
                                      None if reduce_op is None else reduce_op.encode(), int(comm_turn),
                                      int(stream_mode), _ref(output), ctypes.byref(ws), ctypes.byref(ex))
    return st, ws.value, ex.value


def qmm_run(workspace: int, workspace_size: int, executor, stream=None) -> int:
    return lib().qmm_run(workspace or None, workspace_size, executor, _stream_handle(stream))


def wqmm_pack_weight_size(x2: WqmmTensor, for_int8_gemm: bool = False):
    nb = ctypes.c_uint64(0)
    st = lib().wqmm_pack_weight_size(ctypes.byref(x2), int(bool(for_int8_gemm)), ctypes.byref(nb))
    return st, nb.value


def wqmm_pack_weight(x2: WqmmTensor, for_int8_gemm: bool, packed: int, stream=None) -> int:
    return lib().wqmm_pack_weight(ctypes.byref(x2), int(bool(for_int8_gemm)), packed, _stream_handle(stream))


def wqmm_executor_destroy(executor) -> None:
    lib().wqmm_executor_destroy(executor)


def wqmm_last_error() -> str:
    return lib().wqmm_last_error().decode()


def wqmm_stream_wait(stream=None, timeout_ms: int = 10000) -> int:
    return lib().wqmm_stream_wait(_stream_handle(stream), int(timeout_ms))


def wqmm_device_error(reset: bool = False):
    code = ctypes.c_uint32(0)
    st = lib().wqmm_device_error(ctypes.byref(code), int(bool(reset)))
    return st, code.value


def wqmm_version() -> str:
    return lib().wqmm_version().decode()


def qmm_debug_set_raw_accumulator(executor, acc_ptr: int) -> int:
    return lib().qmm_debug_set_raw_accumulator(executor, acc_ptr)


def wqmm_debug_set_flag_wait(executor, wait_ns: int, mismatch: bool) -> int:
    return lib().wqmm_debug_set_flag_wait(executor, int(wait_ns), int(bool(mismatch)))


def wqmm_matmul_no_alloc(x1, x2, bias, antiquant_scale, antiquant_offset, x3, group, reduce_op, comm_turn,
                         stream_mode, antiquant_group_size, output, stream=None) -> int:
    """Both phases of the anti-quant GEMM in one call, with the library's fixed
    16 MiB device workspace instead of a caller-provided one (for callers that
    cannot allocate device memory).  Returns the C status."""
    L = lib()
    f = L.wqmm_matmul_no_alloc
    if f.argtypes is None:
        T = ctypes.POINTER(WqmmTensor)
        f.argtypes = [T, T, T, T, T, T, ctypes.c_char_p, ctypes.c_char_p, ctypes.c_int64, ctypes.c_int64,
                      ctypes.c_int64, T, ctypes.c_void_p]
        f.restype = ctypes.c_int32
    return f(_ref(x1), _ref(x2), _ref(bias), _ref(antiquant_scale), _ref(antiquant_offset), _ref(x3),
             None if group is None else group.encode(), None if reduce_op is None else reduce_op.encode(),
             int(comm_turn), int(stream_mode), int(antiquant_group_size), _ref(output), _stream_handle(stream))


def check(status: int) -> None:
    if status != SUCCESS:
        raise WqmmError(status, wqmm_last_error())


# ---------------------------------------------------------------- torch conveniences
def int4_desc(storage, k: int, n: int, transposed: bool = False) -> WqmmTensor:
    """Descriptor of an int4 (k, n) weight stored two per byte: ND -> storage (k, n/2)
    with pairs along n; transposed -> storage (n, k/2) with pairs along k."""
    strides = (1, k) if transposed else (n, 1)
    return desc(data=storage.data_ptr(), dtype=DT_I4, shape=(k, n), strides=strides)


def pack_weight(x2_desc: WqmmTensor, for_int8_gemm: bool = False, stream=None):
    """Pack a (k, n) weight for the GEMM kernels; returns (uint8 buffer, packed descriptor)."""
    import torch
    st, nbytes = wqmm_pack_weight_size(x2_desc, for_int8_gemm)
    check(st)
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    check(wqmm_pack_weight(x2_desc, for_int8_gemm, buf.data_ptr(), stream))
    k, n = x2_desc.shape[0], x2_desc.shape[1]
    return buf, desc(data=buf.data_ptr(), dtype=x2_desc.dtype, shape=(k, n), fmt=FORMAT_PACKED)


def _keep_until_done(t, stream) -> None:
    """A temporary used by work enqueued on `stream` stays allocated until that
    work is done (the caching allocator reuses freed blocks only in the order
    of the stream they are recorded on)."""
    if t is not None and stream is not None and hasattr(stream, "cuda_stream"):
        t.record_stream(stream)


def _workspace(nbytes: int, device):
    import torch
    if nbytes == 0:
        return None, 0
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, ws.data_ptr()


def weight_quant_matmul(x1, x2_desc: WqmmTensor, antiquant_scale, antiquant_offset=None, bias=None, x3=None,
                        antiquant_group_size: int = 0, out=None, stream=None):
    """out = x1 @ ((x2 + antiquant_offset) * antiquant_scale) + bias + x3 (both phases)."""
    import torch
    if out is None:
        out = torch.empty(tuple(x1.shape[:-1]) + (x2_desc.shape[1],), dtype=x1.dtype, device=x1.device)
    st, ws_size, ex = wqmm_get_workspace_size(
        desc(x1), x2_desc, None if bias is None else desc(bias),
        None if antiquant_scale is None else desc(antiquant_scale),
        None if antiquant_offset is None else desc(antiquant_offset), None if x3 is None else desc(x3), None, "sum",
        0, 1, antiquant_group_size, desc(out))
    check(st)
    ws, ws_ptr = _workspace(ws_size, x1.device)
    check(wqmm_run(ws_ptr, ws_size, ex, stream))
    _keep_until_done(ws, stream)
    return out


def quant_matmul(x1, x2_desc: WqmmTensor, dequant_scale, pertoken_scale=None, bias=None, x3=None,
                 out_dtype=None, out=None, raw_acc=None, stream=None):
    """out = dequant_scale * pertoken_scale * (x1 @ x2 + bias) + x3 for int8 x1, x2."""
    import torch
    if out is None:
        dt = out_dtype or (x3.dtype if x3 is not None else torch.bfloat16)
        out = torch.empty(tuple(x1.shape[:-1]) + (x2_desc.shape[1],), dtype=dt, device=x1.device)
    st, ws_size, ex = qmm_get_workspace_size(
        desc(x1), x2_desc, None if bias is None else desc(bias), None if x3 is None else desc(x3),
        desc(dequant_scale), None if pertoken_scale is None else desc(pertoken_scale), None, "sum", 0, 1, desc(out))
    check(st)
    if raw_acc is not None:
        rc = qmm_debug_set_raw_accumulator(ex, raw_acc.data_ptr())
        if rc != SUCCESS:
            wqmm_executor_destroy(ex)
            check(rc)
    ws, ws_ptr = _workspace(ws_size, x1.device)
    check(qmm_run(ws_ptr, ws_size, ex, stream))
    _keep_until_done(ws, stream)
    return out
