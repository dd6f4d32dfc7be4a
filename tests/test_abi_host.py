"""Host-side tests of the C ABI (no GPU): the library loads and exports every
symbol include/wqmm.h declares; phase-1 validation follows the pages' rules and
the seven unit-test cases the anti-quant page describes; executor life cycle
and workspace checks fail with a status and launch nothing."""
import os

import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

import weight_quantized_gemm_anti_b200 as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FAKE = 0x10000  # an aligned, never-dereferenced address: phase 1 reads descriptors only


@pytest.fixture(scope="module", autouse=True)
def built():
    W.build()


def T(shape, dtype, strides=None, data=FAKE, fmt=W.FORMAT_ND):
    return W.desc(data=data, dtype=dtype, shape=shape, strides=strides, fmt=fmt)


def wq(x1=((32, 64), W.DT_F16), x2=((64, 128), W.DT_I8), scale=((128,), None), offset=None, bias=None, x3=None,
       out=None, G=0, reduce_op="sum", comm_turn=0, stream_mode=1, x2_strides=None, scale_strides=None,
       x2_fmt=W.FORMAT_ND):
    adt = x1[1]
    x1d = T(x1[0], adt, data=FAKE if 0 not in x1[0] else 0)
    x2d = T(x2[0], x2[1], strides=x2_strides, data=FAKE if 0 not in x2[0] else 0, fmt=x2_fmt)
    sd = None if scale is None else T(scale[0], scale[1] or adt, strides=scale_strides)
    od = None if offset is None else T(offset[0], offset[1] or adt, strides=scale_strides)
    bd = None if bias is None else T(bias[0], bias[1] or adt)
    x3d = None if x3 is None else T(x3[0], x3[1] or adt)
    if out is None:
        out = (tuple(x1[0][:-1]) + (x2[0][1],), adt)
    outd = T(out[0], out[1])
    st, ws, ex = W.wqmm_get_workspace_size(x1d, x2d, bd, sd, od, x3d, "hcom", reduce_op, comm_turn, stream_mode, G,
                                           outd)
    if ex:
        W.wqmm_executor_destroy(ex)
    return st, ws


# ------------------------------------------------------------------ library / symbols
def test_library_exports_every_header_symbol():
    names = W.header_symbols()
    assert len(names) >= 12
    L = W.lib()
    for name in names:
        assert hasattr(L, name), name
    assert W.wqmm_version().startswith("wqmm")


def test_product_path_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(W, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(W, "_lib", None)
    with pytest.raises(ImportError):
        W.lib()


# ------------------------------------------------------------------ the page's UT cases
def _ut_cases():
    out = []
    for line in open(os.path.join(GOLDEN, "ut_cases_weight_quant_matmul.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, x1s, x2s, adt, wdt, ss, g, want = [f.strip() for f in line.split("|")]
        shp = lambda s: tuple(int(v) for v in s.split(","))
        out.append((name, shp(x1s), shp(x2s), adt, wdt, shp(ss), int(g), want))
    return out


@pytest.mark.parametrize("case", _ut_cases(), ids=lambda c: c[0])
def test_page_unit_test_cases(case):
    name, x1s, x2s, adt, wdt, ss, g, want = case
    a = {"f16": W.DT_F16, "bf16": W.DT_BF16}[adt]
    w = {"i8": W.DT_I8, "i4": W.DT_I4}[wdt]
    st, _ = wq(x1=(x1s, a), x2=(x2s, w), scale=(ss, None), G=g)
    assert st == {"SUCCESS": W.SUCCESS, "PARAM_INVALID": W.ERR_PARAM_INVALID}[want], (name, W.wqmm_last_error())


# ------------------------------------------------------------------ rules from the constraint text
def test_null_required_inputs():
    x1, x2, s, o = T((32, 64), W.DT_F16), T((64, 128), W.DT_I8), T((128,), W.DT_F16), T((32, 128), W.DT_F16)
    for args in [(None, x2, s, o), (x1, None, s, o), (x1, x2, None, o), (x1, x2, s, None)]:
        st, _, ex = W.wqmm_get_workspace_size(args[0], args[1], None, args[2], None, None, None, "sum", 0, 1, 0,
                                              args[3])
        assert st == W.ERR_PARAM_NULLPTR and ex is None
    st, _, _ = W.wqmm_get_workspace_size(x1, x2, None, s, None, None, None, None, 0, 1, 0, o)
    assert st == W.ERR_PARAM_NULLPTR


def test_dtype_rules():
    assert wq(x1=((32, 64), W.DT_I8))[0] == W.ERR_PARAM_INVALID                    # x1 not f16/bf16
    assert wq(x2=((64, 128), W.DT_F16))[0] == W.ERR_PARAM_INVALID                  # non-quant weight + scale
    assert wq(scale=((128,), W.DT_BF16))[0] == W.ERR_PARAM_INVALID                 # scale dtype != x1
    assert wq(offset=((128,), W.DT_BF16))[0] == W.ERR_PARAM_INVALID
    assert wq(bias=((128,), W.DT_F32))[0] == W.ERR_PARAM_INVALID
    assert wq(x3=((32, 128), W.DT_F32))[0] == W.ERR_PARAM_INVALID                  # illegal x3 dtype
    assert wq(out=((32, 128), W.DT_BF16))[0] == W.ERR_PARAM_INVALID
    assert wq(x1=((32, 64), W.DT_BF16), x2=((64, 128), W.DT_I4))[0] == W.SUCCESS
    assert wq(x2=((64, 128), W.DT_FP8E4M3))[0] == W.SUCCESS                         # per-channel fp8


def test_non_quantised_rules():
    # x2 of the x1 dtype: the non-quantised scenario, no antiquant factors
    st, ws = wq(x2=((64, 128), W.DT_F16), scale=None)
    assert st == W.SUCCESS and ws >= 64 * 128 * 2                                # the 16-bit weight re-laid
    assert wq(x1=((32, 64), W.DT_BF16), x2=((64, 128), W.DT_BF16), scale=None, bias=((128,), None),
              x3=((32, 128), None))[0] == W.SUCCESS
    assert wq(x2=((64, 128), W.DT_F16), scale=None, x2_strides=(1, 64))[0] == W.SUCCESS   # transposed
    assert wq(x2=((64, 128), W.DT_F16), scale=None, x2_fmt=W.FORMAT_PACKED)[0] == W.SUCCESS
    assert wq(x2=((64, 128), W.DT_F16), scale=None, offset=((128,), None))[0] == W.ERR_PARAM_INVALID
    assert wq(x2=((64, 128), W.DT_F16), scale=None, G=32)[0] == W.ERR_PARAM_INVALID
    assert wq(x2=((64, 128), W.DT_BF16))[0] == W.ERR_PARAM_INVALID                 # bf16 weight, f16 x1
    assert wq(x2=((64, 128), W.DT_BF16), scale=None)[0] == W.ERR_PARAM_NULLPTR     # then a scale is required
    assert wq(x2=((64, 128), W.DT_I8), scale=None)[0] == W.ERR_PARAM_NULLPTR
    assert wq(x2=((64, 100), W.DT_F16), scale=None)[0] == W.ERR_PARAM_INVALID      # n % 32
    st, nbytes = W.wqmm_pack_weight_size(T((64, 128), W.DT_BF16), 0)
    assert st == W.SUCCESS and nbytes == 64 * 128 * 2
    assert W.wqmm_pack_weight_size(T((64, 128), W.DT_BF16), 1)[0] == W.ERR_PARAM_INVALID  # int8 GEMM tiling


def test_attribute_rules():
    assert wq(reduce_op="max")[0] == W.ERR_PARAM_INVALID
    assert wq(stream_mode=0)[0] == W.ERR_PARAM_INVALID
    assert wq(comm_turn=2)[0] == W.ERR_PARAM_INVALID
    assert wq(scale=((1, 128), None), G=64)[0] == W.ERR_PARAM_INVALID              # G = k > k - 1
    assert wq(scale=((2, 128), None), G=-32)[0] == W.ERR_PARAM_INVALID
    # G = 32 <= k - 1 = 63, and G = 64 allowed for k = 128
    assert wq(x1=((32, 128), W.DT_F16), x2=((128, 128), W.DT_I8), scale=((2, 128), None), G=64)[0] == W.SUCCESS


def test_fp8_restrictions():
    assert wq(x2=((64, 128), W.DT_FP8E4M3), offset=((128,), None))[0] == W.ERR_PARAM_INVALID
    assert wq(x2=((64, 128), W.DT_FP8E4M3), scale=((1,), None))[0] == W.ERR_PARAM_INVALID
    assert wq(x2=((64, 128), W.DT_FP8E4M3), scale=((2, 128), None), G=32)[0] == W.ERR_PARAM_INVALID


def test_shape_rules():
    assert wq(x1=((32, 96), W.DT_F16))[0] == W.ERR_PARAM_INVALID                   # k mismatch
    assert wq(x1=((64,), W.DT_F16), out=((128,), W.DT_F16))[0] == W.ERR_PARAM_INVALID  # 1-D x1
    assert wq(x1=((2, 16, 64), W.DT_F16))[0] == W.SUCCESS                           # 3-D x1 -> (b, s, n)
    assert wq(x1=((2, 16, 64), W.DT_F16), out=((32, 128), W.DT_F16))[0] == W.ERR_PARAM_INVALID
    assert wq(scale=((2,), None))[0] == W.ERR_PARAM_INVALID                        # illegal per-tensor shape
    assert wq(scale=((1, 128), None))[0] == W.SUCCESS                               # (1, n) per-channel
    assert wq(scale=((3, 128), None), G=32)[0] == W.ERR_PARAM_INVALID              # ceil(64/32) = 2 rows
    assert wq(scale=((2, 128), None), offset=((2, 64), None), G=32)[0] == W.ERR_PARAM_INVALID
    assert wq(bias=((64,), None))[0] == W.ERR_PARAM_INVALID
    assert wq(x3=((32, 64), None))[0] == W.ERR_PARAM_INVALID
    assert wq(out=((16, 128), W.DT_F16))[0] == W.ERR_PARAM_INVALID
    big = 2 ** 31
    assert wq(x1=((big, 64), W.DT_F16))[0] == W.ERR_PARAM_INVALID                  # m > 2^31 - 1
    assert wq(x1=((32, 65536), W.DT_F16), x2=((65536, 128), W.DT_I8))[0] == W.ERR_PARAM_INVALID
    assert wq(x2=((64, 65536 + 32), W.DT_I8), scale=((65536 + 32,), None))[0] == W.ERR_PARAM_INVALID
    assert wq(x1=((32, 64), W.DT_F16), x2=((64, 0), W.DT_I8), scale=((0,), None))[0] == W.ERR_PARAM_INVALID


def test_alignment_rules():
    assert wq(x1=((32, 64), W.DT_F16), x2=((64, 96), W.DT_I8), scale=((96,), None))[0] == W.SUCCESS
    assert wq(x1=((32, 64), W.DT_F16), x2=((64, 100), W.DT_I8), scale=((100,), None))[0] == W.ERR_PARAM_INVALID
    assert wq(x1=((32, 64), W.DT_F16), x2=((64, 96), W.DT_I4), scale=((96,), None))[0] == W.ERR_PARAM_INVALID
    assert wq(x1=((32, 96), W.DT_F16), x2=((96, 128), W.DT_I4))[0] == W.ERR_PARAM_INVALID
    x1 = T((32, 64), W.DT_F16, data=FAKE + 8)
    st, _, _ = W.wqmm_get_workspace_size(x1, T((64, 128), W.DT_I8), None, T((128,), W.DT_F16), None, None, None,
                                         "sum", 0, 1, 0, T((32, 128), W.DT_F16))
    assert st == W.ERR_PARAM_INVALID and "aligned" in W.wqmm_last_error()


def test_layout_rules():
    # transposed x2 (strides (1, k)) with per-channel scale: fine
    assert wq(x2_strides=(1, 64))[0] == W.SUCCESS
    # non-contiguous x2 that is not a transpose
    assert wq(x2_strides=(256, 1))[0] == W.ERR_PARAM_INVALID
    # per-group: transposed x2 needs the scale/offset transposed with it, and vice versa
    assert wq(scale=((2, 128), None), G=32, x2_strides=(1, 64))[0] == W.ERR_PARAM_INVALID
    assert wq(scale=((2, 128), None), G=32, x2_strides=(1, 64), scale_strides=(1, 2))[0] == W.SUCCESS
    assert wq(scale=((2, 128), None), G=32, scale_strides=(1, 2))[0] == W.ERR_PARAM_INVALID
    # non-contiguous x1
    x1 = T((32, 64), W.DT_F16, strides=(1, 32))
    st, _, _ = W.wqmm_get_workspace_size(x1, T((64, 128), W.DT_I8), None, T((128,), W.DT_F16), None, None, None,
                                         "sum", 0, 1, 0, T((32, 128), W.DT_F16))
    assert st == W.ERR_PARAM_INVALID


def test_workspace_sizes():
    # an ND weight is re-laid into the workspace; a packed one needs none (one 64x128 int8 tile pair)
    st, ws = wq()
    assert st == W.SUCCESS and ws >= 8192
    st, ws = wq(x2_fmt=W.FORMAT_PACKED)
    assert st == W.SUCCESS
    # empty k: no GEMM, no workspace
    st, ws = wq(x1=((32, 0), W.DT_F16), x2=((0, 128), W.DT_I8))
    assert st == W.SUCCESS and ws == 0


def test_executor_lifecycle_without_gpu():
    x1, x2, s, o = T((32, 64), W.DT_F16), T((64, 128), W.DT_I8), T((128,), W.DT_F16), T((32, 128), W.DT_F16)
    st, ws, ex = W.wqmm_get_workspace_size(x1, x2, None, s, None, None, None, "sum", 0, 1, 0, o)
    assert st == W.SUCCESS and ws > 0
    # too-small workspace: error, executor consumed, nothing launched
    assert W.wqmm_run(0, 0, ex, stream=0) == W.ERR_WORKSPACE
    # a consumed executor cannot run again ("第二段接口不可重复调用")
    assert W.wqmm_run(0, 0, ex, stream=0) == W.ERR_EXECUTOR
    # the other operator's runner rejects it too
    st, ws, ex2 = W.wqmm_get_workspace_size(x1, x2, None, s, None, None, None, "sum", 0, 1, 0, o)
    assert W.qmm_run(0, 0, ex2, stream=0) == W.ERR_EXECUTOR
    W.wqmm_executor_destroy(ex2)
    assert W.wqmm_run(0, 0, ex2, stream=0) == W.ERR_EXECUTOR
    assert W.wqmm_run(0, 0, None, stream=0) == W.ERR_EXECUTOR


# ------------------------------------------------------------------ int8 path
def qq(x1=((32, 64), W.DT_I8), x2=((64, 128), W.DT_I8), bias=((128,), W.DT_I32), x3=((32, 128), W.DT_F16),
       dq=((128,), W.DT_F32), pt=((32,), W.DT_F32), out=((32, 128), W.DT_F16), reduce_op="sum"):
    d = lambda a: None if a is None else T(a[0], a[1])
    st, ws, ex = W.qmm_get_workspace_size(d(x1), d(x2), d(bias), d(x3), d(dq), d(pt), "hcom", reduce_op, 0, 1, d(out))
    if ex:
        W.wqmm_executor_destroy(ex)
    return st


def test_qmm_page_sample_arguments_accepted():
    assert qq() == W.SUCCESS                                                        # the p4 sample's shapes/dtypes
    assert qq(x1=((4, 8, 64), W.DT_I8), x3=((4, 8, 128), W.DT_F16), out=((4, 8, 128), W.DT_F16)) == W.SUCCESS
    assert qq(dq=((1,), W.DT_F32), pt=None) == W.SUCCESS
    assert qq(dq=((128,), W.DT_BF16), x3=((32, 128), W.DT_BF16), out=((32, 128), W.DT_BF16)) == W.SUCCESS


def test_qmm_rules():
    assert qq(x1=None) == W.ERR_PARAM_NULLPTR
    assert qq(dq=None) == W.ERR_PARAM_NULLPTR
    assert qq(x1=((32, 64), W.DT_F16)) == W.ERR_PARAM_INVALID
    assert qq(bias=((128,), W.DT_F32)) == W.ERR_PARAM_INVALID
    assert qq(dq=((128,), W.DT_I64)) == W.ERR_PARAM_INVALID                         # TransQuantParamV2 encoding
    assert qq(dq=((128,), W.DT_BF16)) == W.ERR_PARAM_INVALID                        # f16 output wants f32
    assert qq(dq=((128,), W.DT_F32), x3=((32, 128), W.DT_BF16), out=((32, 128), W.DT_BF16)) == W.ERR_PARAM_INVALID
    assert qq(pt=((16,), W.DT_F32)) == W.ERR_PARAM_INVALID
    assert qq(dq=((64,), W.DT_F32)) == W.ERR_PARAM_INVALID
    assert qq(x1=((32, 0), W.DT_I8), x2=((0, 128), W.DT_I8)) == W.ERR_PARAM_INVALID  # no empty tensors
    assert qq(x1=((0, 64), W.DT_I8), x3=None, pt=None, out=((0, 128), W.DT_F16)) == W.ERR_PARAM_INVALID
    assert qq(reduce_op="min") == W.ERR_PARAM_INVALID
    assert qq(x2=((64, 100), W.DT_I8)) == W.ERR_PARAM_INVALID


def test_pack_size_queries():
    st, nb = W.wqmm_pack_weight_size(T((4096, 4096), W.DT_I4))
    assert st == W.SUCCESS and nb == 4096 * 4096 // 2
    st, nb = W.wqmm_pack_weight_size(T((8192, 1024), W.DT_I8), True)
    assert st == W.SUCCESS and nb == 8192 * 1024
    st, nb = W.wqmm_pack_weight_size(T((96, 160), W.DT_I8))
    assert st == W.SUCCESS and nb == 2 * 2 * 8192                                   # 2 n-blocks x 2 k-tiles, padded
    st, nb = W.wqmm_pack_weight_size(T((64, 128), W.DT_F16))                  # non-quantised 16-bit weight
    assert st == W.SUCCESS and nb == 64 * 128 * 2
    st, _ = W.wqmm_pack_weight_size(T((64, 128), W.DT_F32))
    assert st == W.ERR_PARAM_INVALID


# ------------------------------------------------------------------ schedule
@pytest.mark.parametrize("m,k,n", [
    (4096, 4096, 4096),    # whole tiles (CTA pairs for int4): no workspace
    (2048, 4096, 4096),    # whole tiles
    (16, 8192, 28672),     # narrow tiles, last wave split, owners reduce inline
    (40, 512, 21760),      # 170 tiles: 148 whole + 22 split
    (16, 4096, 256),       # 2 tiles over many CTAs: fix-up kernel
    (300, 512, 256),       # wide tiles, fewer than the CTAs: two-step units
    (200, 448, 384),       # odd k-step count
    (384, 4096, 4096),     # medium m: 128-row tiles split over the SMs
    (512, 1024, 8192),     # medium m with enough 128-row tiles for whole waves: 256 rows
])
@pytest.mark.parametrize("nonquant", [False, True], ids=["int4", "nonquant"])
def test_schedule_mirror_matches_library_workspace(m, k, n, nonquant):
    import bench
    if nonquant:  # 16-bit weights: the general kernel at every m
        st, ws = wq(x1=((m, k), W.DT_BF16), x2=((k, n), W.DT_BF16), scale=None, x2_fmt=W.FORMAT_PACKED)
    else:
        st, ws = wq(x1=((m, k), W.DT_BF16), x2=((k, n), W.DT_I4), scale=((n,), None), x2_fmt=W.FORMAT_PACKED)
    assert st == W.SUCCESS
    sms = 148  # phase 1 without a GPU plans for a B200
    try:
        import torch
        if torch.cuda.is_available():
            sms = torch.cuda.get_device_properties(0).multi_processor_count
    except ImportError:
        pass
    s = bench.wqmm_schedule(m, n, k, sms, nonquant=nonquant)
    rnd = lambda b: -(-b // 256) * 256
    assert ws == rnd(s["partial_bytes"]) + rnd(s["flag_bytes"]), (s, ws)


@settings(max_examples=80, deadline=None, derandomize=True)
@given(m=st.integers(1, 3000), k_steps=st.integers(1, 160), n_blocks=st.integers(1, 400), nonquant=st.booleans())
def test_schedule_mirror_random_shapes(m, k_steps, n_blocks, nonquant):
    # the benchmark's restatement of the planner agrees with phase 1's
    # workspace (split-tile partials and flags) over random shapes
    import bench
    k, n = 64 * k_steps, 64 * n_blocks
    dt = W.DT_BF16 if nonquant else W.DT_I4
    st_, ws = wq(x1=((m, k), W.DT_BF16), x2=((k, n), dt), scale=None if nonquant else ((n,), None),
                 x2_fmt=W.FORMAT_PACKED)
    assert st_ == W.SUCCESS
    s = bench.wqmm_schedule(m, n, k, 148, nonquant=nonquant)
    rnd = lambda b: -(-b // 256) * 256
    assert ws == rnd(s["partial_bytes"]) + rnd(s["flag_bytes"]), (m, k, n, nonquant, s, ws)
