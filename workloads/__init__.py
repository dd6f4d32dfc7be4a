"""Seeded synthetic inputs for the anti-quant weight GEMM and its int8 sibling.

This module only *draws and encodes* inputs. It holds none of the method's
arithmetic (no dequantisation, no matmul, no rounding of results); both the CPU
oracle and the CUDA path consume the raw storage it returns, so the two sides
never share computation.

Storage conventions (the same bytes go to the oracle and to the GPU):
  * fp16 / bf16 tensors: ``np.uint16`` arrays holding the IEEE bit patterns.
  * fp32 tensors: ``np.float32``.
  * int8 weights / activations: ``np.int8``.
  * int4 weights: ``np.uint8``, two values per byte, two's-complement nibbles,
    the even index of the contiguous axis in bits 0-3 and the odd one in bits
    4-7 ("low nibble first").  For an ND (k, n) weight the pairs run along n;
    for a transposed weight (stored (n, k)) they run along k.
  * fp8-e4m3fn weights: ``np.uint8`` bit patterns.

Distributions follow the workloads of the weight-quant matmul pages
(aclnnWeightQuantMatmulAllReduce "计算公式" and aclnnQuantMatmulAllReduceV2
"Function"): N(0,1) activations, uniform integer weights, uniform scales and
integer offsets. Each tensor has its own sub-stream of a numpy ``SeedSequence``
spawned from the case seed, in the fixed order x1, x2, scale, offset, bias,
x3, dequant_scale, pertoken_scale, so adding an optional tensor never changes
the values drawn for the others.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np

STREAMS = ("x1", "x2", "scale", "offset", "bias", "x3", "dequant_scale", "pertoken_scale")


# --------------------------------------------------------------------------- encoders
def f16_bits(a: np.ndarray) -> np.ndarray:
    """float64 values -> IEEE fp16 bit patterns (numpy's correctly rounded cast)."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).view(np.uint16)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float64 values -> bf16 bit patterns: cast to fp32, then round-to-nearest-even
    on the upper 16 bits. Inputs here are finite, so no NaN handling is needed."""
    u = np.asarray(a, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def act_bits(a: np.ndarray, act: str) -> np.ndarray:
    if act == "f16":
        return f16_bits(a)
    if act == "bf16":
        return bf16_bits(a)
    raise ValueError(act)


def pack_int4_pairs(q: np.ndarray) -> np.ndarray:
    """Pack int4 values (int8 array with values in [-8, 7]) two per byte along the
    last axis, element 2j in the low nibble and 2j+1 in the high nibble."""
    q = np.asarray(q, dtype=np.int8)
    assert q.shape[-1] % 2 == 0
    u = (q.astype(np.int16) & 0xF).astype(np.uint8)
    return (u[..., 0::2] | (u[..., 1::2] << 4)).astype(np.uint8)


def e4m3_bits_from_codes(rng: np.random.Generator, size) -> np.ndarray:
    """Uniform over the finite fp8-e4m3fn codes (the NaN codes 0x7F/0xFF excluded)."""
    codes = rng.integers(0, 254, size=size, dtype=np.int64)
    codes = np.where(codes >= 0x7F, codes + 1, codes)  # skip 0x7F
    return codes.astype(np.uint8)


# --------------------------------------------------------------------------- cases
@dataclass
class WqmmCase:
    """One anti-quant GEMM problem, raw storage only."""
    name: str
    x1_shape: Tuple[int, ...]          # (m, k) or (b, s, k)
    k: int
    n: int
    act: str                           # "f16" | "bf16"
    wdt: str                           # "i8" | "i4" | "fp8"; == act: non-quantised
    mode: str                          # "tensor" | "channel" | "group" | "none"
    group_size: int
    x1: np.ndarray
    x2: np.ndarray                     # storage, see module docstring
    x2_transposed: bool
    scale: Optional[np.ndarray]        # None in the non-quantised scenario
    offset: Optional[np.ndarray]
    bias: Optional[np.ndarray]
    x3: Optional[np.ndarray]
    scale_transposed: bool = False     # per-group scale/offset stored (n, ng)
    seed: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def m(self) -> int:
        return int(np.prod(self.x1_shape[:-1]))

    @property
    def out_shape(self) -> Tuple[int, ...]:
        return tuple(self.x1_shape[:-1]) + (self.n,)

    # logical element strides of x2 viewed as (k, n)
    @property
    def x2_strides(self) -> Tuple[int, int]:
        return (1, self.k) if self.x2_transposed else (self.n, 1)

    @property
    def scale_shape(self) -> Tuple[int, ...]:
        return tuple(self.meta.get("scale_shape", self.scale.shape))

    @property
    def scale_strides(self) -> Tuple[int, int]:
        """Element strides of scale viewed as (rows, n)."""
        if self.mode == "none":
            return (0, 0)
        if self.mode == "group":
            ng = self.scale_shape[0]
            return (1, ng) if self.scale_transposed else (self.n, 1)
        return (0, 0) if self.mode == "tensor" else (0, 1)


@dataclass
class QmmCase:
    """One int8 x int8 problem, raw storage only."""
    name: str
    x1_shape: Tuple[int, ...]
    k: int
    n: int
    out: str                           # "f16" | "bf16"
    x1: np.ndarray                     # int8
    x2: np.ndarray                     # int8, (k, n) or (n, k) when transposed
    x2_transposed: bool
    bias: Optional[np.ndarray]         # int32 (n,)
    dq_dtype: str                      # "bf16" | "f32"
    dequant_scale: np.ndarray          # uint16 bits or float32, shape (1,), (n,) or (1, n)
    pertoken_scale: Optional[np.ndarray]  # float32 (m,)
    x3: Optional[np.ndarray]           # out dtype bits, out shape
    seed: int = 0

    @property
    def m(self) -> int:
        return int(np.prod(self.x1_shape[:-1]))

    @property
    def out_shape(self) -> Tuple[int, ...]:
        return tuple(self.x1_shape[:-1]) + (self.n,)

    @property
    def x2_strides(self) -> Tuple[int, int]:
        return (1, self.k) if self.x2_transposed else (self.n, 1)


def _rngs(seed: int):
    ss = np.random.SeedSequence(seed)
    return dict(zip(STREAMS, (np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(len(STREAMS)))))


def make_wqmm_case(*, name="case", x1_shape=(16, 256), n=128, act="bf16", wdt="i8",
                   mode="channel", group_size=0, offset=True, bias=True, x3=True,
                   x2_transposed=False, scale_2d=False, scale_transposed=False,
                   scale_range=(0.001, 0.02), offset_range=(-8, 8), offset_const=None,
                   scale_const=None, fractional_offset=False, seed=0) -> WqmmCase:
    """Draw one anti-quant case.

    x1 ~ N(0,1); weights uniform over their full integer range (int8 [-128,127],
    int4 [-8,7]) or over all finite fp8-e4m3 codes; scale ~ U[scale_range];
    offset ~ integer U[offset_range] (or U[a,b] continuous with
    ``fractional_offset``); bias, x3 ~ N(0,1). ``scale_const``/``offset_const``
    give per-tensor constants instead of draws.  ``wdt`` equal to ``act`` is
    the non-quantised scenario: x2 ~ N(0, 0.05^2) in the activation format, no
    scale or offset (``mode`` "none")."""
    r = _rngs(seed)
    k = x1_shape[-1]
    m = int(np.prod(x1_shape[:-1]))
    x1 = act_bits(r["x1"].standard_normal(size=x1_shape), act)

    if wdt == "i8":
        q = r["x2"].integers(-128, 128, size=(k, n), dtype=np.int64).astype(np.int8)
        x2 = np.ascontiguousarray(q.T) if x2_transposed else q
    elif wdt == "i4":
        q = r["x2"].integers(-8, 8, size=(k, n), dtype=np.int64).astype(np.int8)
        x2 = pack_int4_pairs(np.ascontiguousarray(q.T)) if x2_transposed else pack_int4_pairs(q)
    elif wdt == "fp8":
        c = e4m3_bits_from_codes(r["x2"], (k, n))
        x2 = np.ascontiguousarray(c.T) if x2_transposed else c
    elif wdt == act:
        w = act_bits(0.05 * r["x2"].standard_normal(size=(k, n)), act)
        x2 = np.ascontiguousarray(w.T) if x2_transposed else w
        mode = "none"
    else:
        raise ValueError(wdt)

    if mode == "none":
        sshape = None
    elif mode == "tensor":
        sshape = (1,)
    elif mode == "channel":
        sshape = (1, n) if scale_2d else (n,)
    elif mode == "group":
        ng = -(-k // group_size)
        sshape = (ng, n)
    else:
        raise ValueError(mode)

    if mode == "none":
        s = None
    elif scale_const is not None:
        s = np.full(sshape, scale_const, dtype=np.float64)
    else:
        s = r["scale"].uniform(scale_range[0], scale_range[1], size=sshape)
    if offset and wdt != "fp8" and mode != "none":
        if offset_const is not None:
            o = np.full(sshape, offset_const, dtype=np.float64)
        elif fractional_offset:
            o = r["offset"].uniform(offset_range[0], offset_range[1], size=sshape)
        else:
            o = r["offset"].integers(offset_range[0], offset_range[1] + 1, size=sshape).astype(np.float64)
    else:
        o = None

    scale_bits = None if s is None else act_bits(s, act)
    off_bits = None if o is None else act_bits(o, act)
    if mode == "group" and scale_transposed:
        scale_bits = np.ascontiguousarray(scale_bits.T)
        off_bits = None if off_bits is None else np.ascontiguousarray(off_bits.T)

    b = act_bits(r["bias"].standard_normal(size=(n,)), act) if bias else None
    out_shape = tuple(x1_shape[:-1]) + (n,)
    x3a = act_bits(r["x3"].standard_normal(size=out_shape), act) if x3 else None
    return WqmmCase(name=name, x1_shape=tuple(x1_shape), k=k, n=n, act=act, wdt=wdt, mode=mode,
                    group_size=group_size if mode == "group" else 0, x1=x1, x2=x2,
                    x2_transposed=x2_transposed, scale=scale_bits, offset=off_bits, bias=b, x3=x3a,
                    scale_transposed=scale_transposed and mode == "group", seed=seed,
                    meta={"scale_shape": sshape})


def make_qmm_case(*, name="qcase", x1_shape=(32, 64), n=128, out="bf16", bias=True, x3=True,
                  pertoken=True, dq_per_tensor=False, dq_2d=False, x2_transposed=False,
                  dq_range=(1e-4, 1e-3), seed=0, x_range=(-127, 127), bias_range=(-1000, 1000)) -> QmmCase:
    """Draw one int8 x int8 case: x1, x2 ~ integer U[x_range]; bias ~ integer
    U[bias_range]; dequantScale ~ U[dq_range] (bf16 for bf16 output, fp32 for
    fp16 output); pertokenScale ~ U[0.5, 2] fp32; x3 ~ N(0,1)."""
    r = _rngs(seed)
    k = x1_shape[-1]
    m = int(np.prod(x1_shape[:-1]))
    x1 = r["x1"].integers(x_range[0], x_range[1] + 1, size=x1_shape, dtype=np.int64).astype(np.int8)
    q = r["x2"].integers(x_range[0], x_range[1] + 1, size=(k, n), dtype=np.int64).astype(np.int8)
    x2 = np.ascontiguousarray(q.T) if x2_transposed else q
    b = r["bias"].integers(bias_range[0], bias_range[1] + 1, size=(n,), dtype=np.int64).astype(np.int32) if bias else None
    dshape = (1,) if dq_per_tensor else ((1, n) if dq_2d else (n,))
    dq = r["dequant_scale"].uniform(dq_range[0], dq_range[1], size=dshape)
    if out == "bf16":
        dq_dtype, dqa = "bf16", bf16_bits(dq)
    else:
        dq_dtype, dqa = "f32", dq.astype(np.float32)
    pt = r["pertoken_scale"].uniform(0.5, 2.0, size=(m,)).astype(np.float32) if pertoken else None
    out_shape = tuple(x1_shape[:-1]) + (n,)
    x3a = act_bits(r["x3"].standard_normal(size=out_shape), out) if x3 else None
    return QmmCase(name=name, x1_shape=tuple(x1_shape), k=k, n=n, out=out, x1=x1, x2=x2,
                   x2_transposed=x2_transposed, bias=b, dq_dtype=dq_dtype, dequant_scale=dqa,
                   pertoken_scale=pt, x3=x3a, seed=seed)


# --------------------------------------------------------------------------- the named workloads
# The first five are the benchmark configurations of the operator's headline
# comparison; the rest widen it: fp8-e4m3 weights (per-channel only, no
# offset), a medium-m point, and the non-quantised scenario at the headline's
# size.
WORKLOADS = {
    "tiny_w8a16_perchannel_f16": "x1 f16 (16,256); x2 i8 (256,128); per-channel scale/offset; bias; no x3",
    "w8a16_pertensor_bf16_2048x4096x4096": "x1 bf16 (2048,4096); x2 i8 (4096,4096); scale=0.01 offset=3; bias; x3",
    "w4a16_g128_bf16_4096x4096x4096": "x1 bf16 (4096,4096); x2 i4 (4096,4096); g=128 scale/offset; no bias/x3",
    "decode_w4a16_g64_bf16_1x16x8192x28672": "x1 bf16 (1,16,8192); x2 i4 (8192,28672); g=64; bias",
    "w8a8_pertoken_4x2048x8192x1024": "x1 i8 (4,2048,8192); x2 i8 (8192,1024); bias i32; bf16 dq; pertoken; x3",
    "fp8_perchannel_bf16_4096x4096x4096": "x1 bf16 (4096,4096); x2 fp8-e4m3 (4096,4096); per-channel scale; no offset",
    "w4a16_g128_bf16_256x4096x4096": "x1 bf16 (256,4096); x2 i4 (4096,4096); g=128 scale/offset; no bias/x3",
    "nonquant_bf16_4096x4096x4096": "x1 bf16 (4096,4096); x2 bf16 (4096,4096); no antiquant; no bias/x3",
}
WORKLOAD_NAMES = list(WORKLOADS)


def workload(name: str):
    """Build one of the named workloads (seed = its index in WORKLOAD_NAMES)."""
    i = WORKLOAD_NAMES.index(name)
    if i == 0:
        return make_wqmm_case(name=name, x1_shape=(16, 256), n=128, act="f16", wdt="i8", mode="channel",
                              scale_range=(0.001, 0.02), offset_range=(-8, 8), bias=True, x3=False, seed=0)
    if i == 1:
        return make_wqmm_case(name=name, x1_shape=(2048, 4096), n=4096, act="bf16", wdt="i8", mode="tensor",
                              scale_const=0.01, offset_const=3.0, bias=True, x3=True, seed=1)
    if i == 2:
        return make_wqmm_case(name=name, x1_shape=(4096, 4096), n=4096, act="bf16", wdt="i4", mode="group",
                              group_size=128, scale_range=(0.005, 0.05), offset_range=(-4, 4),
                              bias=False, x3=False, seed=2)
    if i == 3:
        return make_wqmm_case(name=name, x1_shape=(1, 16, 8192), n=28672, act="bf16", wdt="i4", mode="group",
                              group_size=64, scale_range=(0.005, 0.05), offset_range=(-4, 4),
                              bias=True, x3=False, seed=3)
    if i == 4:
        return make_qmm_case(name=name, x1_shape=(4, 2048, 8192), n=1024, out="bf16", bias=True, x3=True,
                             pertoken=True, seed=4)
    if i == 5:
        return make_wqmm_case(name=name, x1_shape=(4096, 4096), n=4096, act="bf16", wdt="fp8", mode="channel",
                              scale_range=(0.001, 0.02), offset=False, bias=False, x3=False, seed=5)
    if i == 6:
        return make_wqmm_case(name=name, x1_shape=(256, 4096), n=4096, act="bf16", wdt="i4", mode="group",
                              group_size=128, scale_range=(0.005, 0.05), offset_range=(-4, 4),
                              bias=False, x3=False, seed=6)
    if i == 7:
        return make_wqmm_case(name=name, x1_shape=(4096, 4096), n=4096, act="bf16", wdt="bf16",
                              bias=False, x3=False, seed=7)
    raise KeyError(name)
