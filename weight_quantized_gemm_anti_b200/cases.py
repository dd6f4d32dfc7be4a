"""Marshalling of raw host arrays (bit patterns, packed int4 bytes) into device
tensors and ABI descriptors.  No arithmetic of the method happens here: the
bytes are copied as they are and described to the library.

A "case" is any object with the attributes of the seeded problem descriptions
(x1, x2, x2_transposed, scale, offset, bias, x3, ... as raw numpy storage);
see the ``workloads`` package for the layout of each field.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import (DT_BF16, DT_F16, DT_F32, DT_FP8E4M3, DT_I4, DT_I8, DT_I32, FORMAT_PACKED, WqmmTensor, check, desc,
               pack_weight, qmm_debug_set_raw_accumulator, qmm_get_workspace_size, qmm_run,
               wqmm_executor_destroy, wqmm_get_workspace_size, wqmm_run)

_ACT = {"f16": DT_F16, "bf16": DT_BF16}
_WDT = {"i8": DT_I8, "i4": DT_I4, "fp8": DT_FP8E4M3, "f16": DT_F16, "bf16": DT_BF16}  # f16/bf16: non-quantised


def _torch():
    import torch
    return torch


def _dev(a: np.ndarray, device, pin=False):
    torch = _torch()
    t = torch.from_numpy(np.ascontiguousarray(a))
    if pin:
        return t.pin_memory()
    return t.to(device)


def _act_view(t, act):
    torch = _torch()
    return t.view(torch.float16 if act == "f16" else torch.bfloat16)


@dataclass
class WqmmDevice:
    x1: object
    x2: object
    x2_desc: WqmmTensor
    scale: object
    scale_desc: WqmmTensor
    offset: object
    offset_desc: Optional[WqmmTensor]
    bias: object
    x3: object
    out: object
    group_size: int
    packed: Optional[object] = None
    keep: tuple = ()


def wqmm_to_device(case, device="cuda", pack=True, stream=None) -> WqmmDevice:
    """Copy a wqmm case to the device; optionally pre-pack the weight."""
    torch = _torch()
    k, n = case.k, case.n
    x1 = _act_view(_dev(case.x1.view(np.int16), device), case.act).reshape(case.x1_shape)
    if case.wdt in ("f16", "bf16"):
        x2s = _dev(case.x2.view(np.int16), device)
    else:
        x2s = _dev(case.x2.view(np.uint8) if case.x2.dtype != np.int8 else case.x2, device)
    strides = (1, k) if case.x2_transposed else (n, 1)
    x2d = desc(data=x2s.data_ptr(), dtype=_WDT[case.wdt], shape=(k, n), strides=strides)
    packed = None
    if pack and k > 0:
        packed, x2d = pack_weight(x2d, False, stream)
    sshape = None if case.scale is None else tuple(case.scale_shape)
    sc = None if case.scale is None else _act_view(_dev(case.scale.view(np.int16), device), case.act)
    of = None if case.offset is None else _act_view(_dev(case.offset.view(np.int16), device), case.act)
    if sc is None:
        pass
    elif case.mode == "group" and case.scale_transposed:
        ng = sshape[0]
        sc = sc.reshape(n, ng).t()
        of = None if of is None else of.reshape(n, ng).t()
    else:
        sc = sc.reshape(sshape)
        of = None if of is None else of.reshape(sshape)
    bias = None if case.bias is None else _act_view(_dev(case.bias.view(np.int16), device), case.act)
    x3 = None if case.x3 is None else _act_view(_dev(case.x3.view(np.int16), device), case.act).reshape(case.out_shape)
    out = torch.empty(case.out_shape, dtype=x1.dtype, device=device)
    return WqmmDevice(x1=x1, x2=x2s, x2_desc=x2d, scale=sc, scale_desc=None if sc is None else desc(sc), offset=of,
                      offset_desc=None if of is None else desc(of), bias=bias, x3=x3, out=out,
                      group_size=case.group_size, packed=packed)


def wqmm_call(d: WqmmDevice, stream=None, workspace=None):
    """Both phases of the anti-quant GEMM on device tensors; returns the workspace tensor used."""
    torch = _torch()
    st, ws_size, ex = wqmm_get_workspace_size(desc(d.x1), d.x2_desc, None if d.bias is None else desc(d.bias),
                                              d.scale_desc, d.offset_desc, None if d.x3 is None else desc(d.x3),
                                              None, "sum", 0, 1, d.group_size, desc(d.out))
    check(st)
    if ws_size and (workspace is None or workspace.numel() < ws_size):
        workspace = torch.empty(ws_size, dtype=torch.uint8, device=d.x1.device)
    ptr = workspace.data_ptr() if (ws_size and workspace is not None) else 0
    check(wqmm_run(ptr, ws_size, ex, stream))
    return workspace


@dataclass
class QmmDevice:
    x1: object
    x2: object
    x2_desc: WqmmTensor
    bias: object
    dq: object
    dq_desc: WqmmTensor
    pt: object
    x3: object
    out: object
    packed: Optional[object] = None


def qmm_to_device(case, device="cuda", pack=True, stream=None) -> QmmDevice:
    torch = _torch()
    k, n = case.k, case.n
    x1 = _dev(case.x1, device).reshape(case.x1_shape)
    x2s = _dev(case.x2, device)
    strides = (1, k) if case.x2_transposed else (n, 1)
    x2d = desc(data=x2s.data_ptr(), dtype=DT_I8, shape=(k, n), strides=strides)
    packed = None
    if pack:
        packed, x2d = pack_weight(x2d, True, stream)
    bias = None if case.bias is None else _dev(case.bias, device)
    if case.dq_dtype == "bf16":
        dq = _dev(case.dequant_scale.view(np.int16), device).view(torch.bfloat16)
    else:
        dq = _dev(case.dequant_scale, device)
    dq = dq.reshape(case.dequant_scale.shape)
    pt = None if case.pertoken_scale is None else _dev(case.pertoken_scale, device)
    x3 = None if case.x3 is None else _act_view(_dev(case.x3.view(np.int16), device), case.out).reshape(case.out_shape)
    out = torch.empty(case.out_shape, dtype=torch.bfloat16 if case.out == "bf16" else torch.float16, device=device)
    return QmmDevice(x1=x1, x2=x2s, x2_desc=x2d, bias=bias, dq=dq, dq_desc=desc(dq), pt=pt, x3=x3, out=out,
                     packed=packed)


def qmm_call(d: QmmDevice, stream=None, raw_acc=None, workspace=None):
    torch = _torch()
    st, ws_size, ex = qmm_get_workspace_size(desc(d.x1), d.x2_desc, None if d.bias is None else desc(d.bias),
                                             None if d.x3 is None else desc(d.x3), d.dq_desc,
                                             None if d.pt is None else desc(d.pt), None, "sum", 0, 1, desc(d.out))
    check(st)
    if raw_acc is not None:
        rc = qmm_debug_set_raw_accumulator(ex, raw_acc.data_ptr())
        if rc:
            wqmm_executor_destroy(ex)
            check(rc)
    if ws_size and (workspace is None or workspace.numel() < ws_size):
        workspace = torch.empty(ws_size, dtype=torch.uint8, device=d.x1.device)
    ptr = workspace.data_ptr() if (ws_size and workspace is not None) else 0
    check(qmm_run(ptr, ws_size, ex, stream))
    return workspace
