"""Row-parallel shards of a seeded anti-quant case, for the CPU all-reduce
tests and the GPU shard tests: each rank's inputs cut with the package's
shard helpers, and each rank's exact local result from the CPU oracle (test
infrastructure only)."""
import numpy as np
import torch

from weight_quantized_gemm_anti_b200 import allreduce as AR


def shard_case(case, rank, world, int4):
    """This rank's inputs, cut with the package's shard helpers (torch CPU tensors)."""
    k0, k1 = AR.k_ranges(case.k, world, case.group_size)[rank]
    t = torch.from_numpy
    x1 = AR.shard_x1(t(case.x1.view(np.int16)).reshape(case.x1_shape), k0, k1)
    x2 = AR.shard_weight(t(np.ascontiguousarray(case.x2)), k0, k1, int4=int4, transposed=case.x2_transposed)
    sc = None if case.scale is None else t(case.scale.view(np.int16))
    of = None if case.offset is None else t(case.offset.view(np.int16))
    if case.mode == "group":
        sc = AR.shard_group_rows(sc, k0, k1, case.group_size, transposed=case.scale_transposed)
        of = AR.shard_group_rows(of, k0, k1, case.group_size, transposed=case.scale_transposed)
    return k0, k1, x1, x2, sc, of


def local_oracle(case, rank, world, int4):
    """The rank's full local result (bias and x3 included), exact, from its shard."""
    import oracle
    k0, k1, x1, x2, sc, of = shard_case(case, rank, world, int4)
    kr = k1 - k0
    n = case.n
    if case.mode == "group":
        ng = sc.shape[1] if case.scale_transposed else sc.shape[0]
        ss = (1, ng) if case.scale_transposed else (n, 1)
    else:
        ss = case.scale_strides
    ye, _ = oracle.wqmm_raw(m=case.m, k=kr, n=n, act=case.act, x1=x1.numpy().view(np.uint16).reshape(case.m, kr),
                            wdt=case.wdt, x2=x2.numpy(), x2_strides=(1, kr) if case.x2_transposed else (n, 1),
                            mode=case.mode, group_size=case.group_size,
                            scale=None if sc is None else sc.numpy().view(np.uint16),
                            offset=None if of is None else of.numpy().view(np.uint16), scale_strides=ss,
                            bias=case.bias, x3=case.x3)
    return ye
