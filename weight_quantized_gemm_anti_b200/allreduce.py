"""Row-parallel anti-quant GEMM with the operator's AllReduce over ranks.

The fused operator of aclnnWeightQuantMatmulAllReduce ("计算公式") is

    output = AllReduce( x1 @ ((x2 + antiquantOffset) * antiquantScale) + bias + x3 )

over the ranks of a communication domain (reduceOp "sum").  The torch_npu
npu_mm_all_reduce_base page describes its tensor-parallel use: x1 and x2 are
split along k (row-parallel), so rank r holds x1[..., k_r] and x2[k_r, :]
with the scale/offset rows of its k range.  Every rank computes its full
local result -- bias and x3 included, since the formula adds them inside the
AllReduce -- and the AllReduce sums the ranks' outputs, elementwise, in the
output tensor's dtype.

One process per GPU: each rank runs this library's GEMM on its shard, then
torch.distributed.all_reduce(SUM) on the output (ncclAllReduce with the NCCL
backend, on the process group's own stream, which waits for the stream the
GEMM was enqueued on).  At world size 1 the AllReduce is the identity and
nothing is launched for it.

Shards: a rank's k range starts on a multiple of lcm(64, G) (G = the
per-group size, or 1): whole 64-wide k steps of the packed weight and whole
scale/offset group rows.  The last rank's range ends at k.
"""
from __future__ import annotations

import math
from typing import List, Optional, Tuple

from . import desc, int4_desc, pack_weight, weight_quant_matmul


def k_shard_unit(group_size: int = 0) -> int:
    """Granularity of the k split: whole 64-wide k steps and whole groups."""
    return 64 if group_size <= 0 else 64 * group_size // math.gcd(64, group_size)


def k_ranges(k: int, world: int, group_size: int = 0) -> List[Tuple[int, int]]:
    """The [k0, k1) range of every rank: units of k_shard_unit dealt as evenly
    as possible (the first ranks take one more when they do not divide), the
    last range ending at k.  Every rank gets at least one unit."""
    if world < 1:
        raise ValueError("world size must be >= 1")
    unit = k_shard_unit(group_size)
    units = -(-k // unit)
    if units < world:
        raise ValueError(f"k = {k} has {units} units of {unit}: too few for {world} ranks")
    base, extra = divmod(units, world)
    out, u = [], 0
    for r in range(world):
        cnt = base + (1 if r < extra else 0)
        out.append((u * unit, min((u + cnt) * unit, k)))
        u += cnt
    return out


def shard_x1(x1, k0: int, k1: int):
    """This rank's columns of x1 ((m, k) or (b, s, k)), contiguous."""
    return x1[..., k0:k1].contiguous()


def shard_weight(x2, k0: int, k1: int, *, int4: bool = False, transposed: bool = False):
    """This rank's rows of a (k, n) weight, contiguous, in the same storage form:
    ND storage (k, n) -- or (k, n/2) bytes for int4 -- gives rows k0:k1;
    transposed storage (n, k) -- or (n, k/2) bytes -- gives columns k0:k1."""
    if int4:
        if k0 % 2 or (k1 - k0) % 2:
            raise ValueError("int4 shards must start and end on even k")
        return (x2[:, k0 // 2:k1 // 2] if transposed else x2[k0:k1]).contiguous()
    return (x2[:, k0:k1] if transposed else x2[k0:k1]).contiguous()


def shard_group_rows(t, k0: int, k1: int, group_size: int, *, transposed: bool = False):
    """This rank's rows of a per-group scale/offset ((ceil(k/G), n), or (n, ceil(k/G))
    when transposed): the groups that cover k0:k1.  Other modes are replicated."""
    if t is None or group_size <= 0:
        return t
    g0, g1 = k0 // group_size, -(-k1 // group_size)
    return (t[:, g0:g1] if transposed else t[g0:g1]).contiguous()


def all_reduce_output(out, group=None, stream=None):
    """Sum `out` over the ranks of `group` in place (the operator's AllReduce,
    reduceOp "sum"); the identity when there is one rank or no process group.
    The collective is ordered after the work already enqueued on `stream` (a
    torch.cuda.Stream; None: the current stream)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        if stream is not None and hasattr(stream, "cuda_stream"):
            import torch
            with torch.cuda.stream(stream):
                dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
        else:
            dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


def pack_shard(x2_shard, k: int, n: int, *, int4: bool = False, transposed: bool = False,
               dtype: Optional[int] = None, stream=None):
    """Pack this rank's weight shard (as shard_weight returns it, logical (k, n))
    once, for every later call; returns (buffer, packed descriptor).  `dtype`:
    the weight's DT_* code when the storage tensor's own dtype does not say it
    (fp8 bits held as uint8)."""
    if int4:
        d = int4_desc(x2_shard, k, n, transposed=transposed)
    else:
        d = desc(x2_shard, dtype=dtype, shape=(k, n), strides=(1, k) if transposed else (n, 1))
    return pack_weight(d, False, stream)


def matmul_all_reduce(x1, x2_desc, antiquant_scale=None, antiquant_offset=None, bias=None, x3=None,
                      antiquant_group_size: int = 0, out=None, group=None, stream=None):
    """This rank's part of the fused operator: the anti-quant GEMM on the local
    shard (x1: this rank's k columns; x2_desc: its k rows, e.g. from
    pack_shard; scale/offset: its group rows, or the full per-channel /
    per-tensor tensors), then the AllReduce(sum) of the output over `group`.
    antiquant_scale None: the non-quantised scenario (x2 of the x1 dtype).
    `stream`: a torch.cuda.Stream (or None for the current stream) that both the
    GEMM and the AllReduce are ordered on."""
    if stream is not None and not hasattr(stream, "cuda_stream"):
        raise TypeError("stream must be a torch.cuda.Stream or None")
    out = weight_quant_matmul(x1, x2_desc, antiquant_scale, antiquant_offset, bias, x3, antiquant_group_size, out,
                              stream)
    return all_reduce_output(out, group, stream)
