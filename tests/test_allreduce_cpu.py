"""Row-parallel split and the operator's AllReduce, on CPU (gloo, world size 2).

aclnnWeightQuantMatmulAllReduce ("计算公式") sums every rank's full result,
x1_r @ ((x2_r + offset_r) * scale_r) + bias + x3, over the communication
domain; in the row-parallel use of npu_mm_all_reduce_base each rank holds a k
range of x1 and x2 (and the scale/offset group rows of that range).  These
tests check the host side of that path without a GPU:
  * the k ranges (whole 64-wide steps and whole groups, balanced, covering k);
  * the shard helpers, against the unsharded storage decoded independently;
  * two gloo ranks that each evaluate their shard with the CPU oracle and sum
    the results with the same all-reduce call the GPU path uses: the sum
    equals the oracle of the whole problem plus (world - 1) * (bias + x3),
    since every rank's result carries bias and x3.
"""
import os
import socket

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from weight_quantized_gemm_anti_b200 import allreduce as AR
from rowparallel_cases import local_oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2

# (name, case arguments, weight stored two per byte)
SPECS = [
    ("i4_g64", dict(x1_shape=(6, 512), n=96, act="bf16", wdt="i4", mode="group", group_size=64, seed=41), True),
    ("i4_g128_transposed", dict(x1_shape=(2, 3, 768), n=64, act="f16", wdt="i4", mode="group", group_size=128,
                                x2_transposed=True, scale_transposed=True, seed=42), True),
    ("i8_chan", dict(x1_shape=(5, 320), n=64, act="bf16", wdt="i8", mode="channel", seed=43), False),
    ("fp8_chan", dict(x1_shape=(4, 256), n=32, act="bf16", wdt="fp8", mode="channel", offset=False, seed=44), False),
    ("nonquant", dict(x1_shape=(3, 192), n=32, act="bf16", wdt="bf16", seed=45), False),
]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import workloads as WL
        for name, kw, int4 in SPECS:
            case = WL.make_wqmm_case(name=name, **kw)
            y = torch.from_numpy(local_oracle(case, rank, world, int4))
            AR.all_reduce_output(y)  # the AllReduce(sum) the GPU path runs on its output
            if rank == 0:
                np.save(os.path.join(outdir, f"{name}.npy"), y.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    outdir = str(tmp_path_factory.mktemp("allreduce"))
    import oracle
    oracle.build()  # build before spawning so the ranks only load it
    mp.spawn(_rank_main, args=(WORLD, _free_port(), outdir), nprocs=WORLD, join=True)
    return outdir


@pytest.mark.parametrize("spec", SPECS, ids=[s[0] for s in SPECS])
def test_two_rank_all_reduce_equals_whole_problem(two_ranks, spec):
    import oracle
    import workloads as WL
    name, kw, _ = spec
    case = WL.make_wqmm_case(name=name, **kw)
    whole, _ = oracle.wqmm(case)
    extra = np.zeros((case.m, case.n))
    dec = (lambda b: b.view(np.float16).astype(np.float64)) if case.act == "f16" else \
        (lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    if case.bias is not None:
        extra += dec(case.bias)[None, :]
    if case.x3 is not None:
        extra += dec(case.x3).reshape(case.m, case.n)
    want = whole + (WORLD - 1) * extra
    got = np.load(os.path.join(two_ranks, f"{name}.npy"))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


@pytest.mark.parametrize("k,world,g", [(4096, 2, 128), (4096, 3, 128), (4096, 8, 0), (320, 2, 0), (768, 4, 64),
                                       (8192, 8, 96), (640, 5, 128)])
def test_k_ranges_cover_k_in_whole_units(k, world, g):
    r = AR.k_ranges(k, world, g)
    unit = AR.k_shard_unit(g)
    assert len(r) == world and r[0][0] == 0 and r[-1][1] == k
    for (a, b), (c, _) in zip(r, r[1:]):
        assert b == c                                   # contiguous, no overlap
    for a, b in r:
        assert a % unit == 0 and b > a                  # starts on whole steps and groups
        assert a % 64 == 0 and (g == 0 or a % g == 0)
    sizes = [-(-(b - a) // unit) for a, b in r]
    assert max(sizes) - min(sizes) <= 1                 # balanced to one unit


def test_k_ranges_reject_too_many_ranks():
    with pytest.raises(ValueError):
        AR.k_ranges(256, 8, 128)                        # two 128-wide units for eight ranks
    assert AR.k_shard_unit(96) == 192 and AR.k_shard_unit(0) == 64 and AR.k_shard_unit(256) == 256


def test_int4_shards_hold_the_same_values():
    import workloads as WL
    for transposed in (False, True):
        case = WL.make_wqmm_case(x1_shape=(2, 256), n=64, act="bf16", wdt="i4", mode="channel",
                                 x2_transposed=transposed, seed=46)
        full = torch.from_numpy(np.ascontiguousarray(case.x2))

        def unpack(b, rows, cols):
            b = b.astype(np.int64)
            out = np.empty((rows, cols), dtype=np.int64)
            out[:, 0::2], out[:, 1::2] = b & 0xF, (b >> 4) & 0xF
            return np.where(out >= 8, out - 16, out)

        ref = unpack(case.x2, case.n, case.k).T if transposed else unpack(case.x2, case.k, case.n)
        for k0, k1 in AR.k_ranges(case.k, 2):
            s = AR.shard_weight(full, k0, k1, int4=True, transposed=transposed).numpy()
            got = unpack(s, case.n, k1 - k0).T if transposed else unpack(s, k1 - k0, case.n)
            assert np.array_equal(got, ref[k0:k1])


def test_matmul_all_reduce_takes_a_torch_stream_only():
    # the AllReduce is ordered on the stream the GEMM ran on, which needs a
    # torch.cuda.Stream (a raw handle cannot be waited on by the process group)
    with pytest.raises(TypeError):
        AR.matmul_all_reduce(None, None, stream=12345)


@settings(max_examples=200, deadline=None, derandomize=True)
@given(k_units=st.integers(1, 1024), world=st.integers(1, 8), g=st.sampled_from([0, 32, 64, 96, 128, 192, 256]),
       tail=st.integers(0, 63))
def test_k_ranges_properties(k_units, world, g, tail):
    # any k (a ragged tail included) and world: contiguous cover of [0, k),
    # starts on whole 64-wide steps and whole groups, balanced to one unit,
    # or a refusal when there are fewer units than ranks
    unit = AR.k_shard_unit(g)
    k = 64 * k_units + (tail // 32) * 32
    units = -(-k // unit)
    if units < world:
        with pytest.raises(ValueError):
            AR.k_ranges(k, world, g)
        return
    r = AR.k_ranges(k, world, g)
    assert r[0][0] == 0 and r[-1][1] == k and len(r) == world
    assert all(b == c for (_, b), (c, _) in zip(r, r[1:]))
    assert all(a % unit == 0 and b > a for a, b in r)
    sizes = [-(-(b - a) // unit) for a, b in r]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == units
