"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Tolerance: max|gpu - oracle| / max|oracle| <= 4e-3 for bf16 outputs and
<= 1e-3 for fp16 outputs, where `oracle` is the exact (fp64, pre-rounding)
result -- the budget of one rounding of each dequantised weight to the MMA
operand type plus one rounding of the output; the raw int32 accumulator of the
int8 path is compared bit for bit.  Small cases span several tiles plus ragged tails in
m, n and k and cover every mode, weight type, activation type and layout;
full-size workloads are checked on sampled outputs the oracle evaluates one by
one.
"""
import zlib

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import workloads as WL
import weight_quantized_gemm_anti_b200 as W
from weight_quantized_gemm_anti_b200 import cases as C

pytestmark = pytest.mark.gpu

TOL = {"bf16": 4e-3, "f16": 1e-3}


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    W.build()
    torch.cuda.init()
    yield


def dec(bits: np.ndarray, act: str) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    if act == "f16":
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gpu_bits(t) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1, t.shape[-1])


def no_device_error():
    st, code = W.wqmm_device_error(reset=True)
    assert st == W.SUCCESS and code == 0, f"device error word {code}"


def rel_err(got, exact):
    denom = np.abs(exact).max()
    return np.abs(got - exact).max() / (denom if denom > 0 else 1.0)


def run_wqmm(case, pack=True):
    d = C.wqmm_to_device(case, pack=pack)
    C.wqmm_call(d)
    torch.cuda.synchronize()
    no_device_error()
    return gpu_bits(d.out)


def check_wqmm(case, pack=True, rows=None, cols=None):
    got = run_wqmm(case, pack=pack)
    ye, _ = oracle.wqmm(case, rows=rows, cols=cols)
    if rows is not None:
        got = got[rows]
    if cols is not None:
        got = got[:, cols]
    g = dec(got, case.act)
    assert np.isfinite(g).all()
    err = rel_err(g, ye)
    assert err <= TOL[case.act], f"{case.name}: rel err {err:.3e}"
    return err


# ---------------------------------------------------------------- small cases
SMALL = [
    # name, x1_shape, n, act, wdt, mode, G, extras
    ("i8_chan_f16_m16", (16, 256), 128, "f16", "i8", "channel", 0, {}),
    ("i8_chan_bf16_ragged", (37, 96), 192, "bf16", "i8", "channel", 0, {}),
    ("i8_tensor_bf16_m200", (200, 320), 160, "bf16", "i8", "tensor", 0, {"scale_const": 0.01, "offset_const": 3.0}),
    ("i8_group32_bf16", (100, 192), 224, "bf16", "i8", "group", 32, {}),
    ("i8_group96_f16", (70, 288), 96, "f16", "i8", "group", 96, {}),
    ("i4_group128_bf16_m300", (300, 512), 320, "bf16", "i4", "group", 128, {"scale_range": (0.005, 0.05),
                                                                           "offset_range": (-4, 4)}),
    ("i4_group64_f16", (33, 256), 384, "f16", "i4", "group", 64, {}),
    ("i4_chan_bf16_m1", (1, 640), 256, "bf16", "i4", "channel", 0, {}),
    ("i4_tensor_f16", (129, 128), 128, "f16", "i4", "tensor", 0, {}),
    ("fp8_chan_bf16", (50, 256), 192, "bf16", "fp8", "channel", 0, {"offset": False}),
    ("fp8_chan_f16", (17, 128), 128, "f16", "fp8", "channel", 0, {"offset": False}),
    ("i8_chan_bf16_no_offset", (64, 128), 128, "bf16", "i8", "channel", 0, {"offset": False}),
    ("i8_chan_bf16_fractional", (40, 192), 128, "bf16", "i8", "channel", 0, {"fractional_offset": True}),
    ("i4_group64_bf16_fractional", (24, 256), 128, "bf16", "i4", "group", 64, {"fractional_offset": True}),
    ("i4_group64_f16_fractional", (24, 256), 128, "f16", "i4", "group", 64, {"fractional_offset": True}),
    ("i8_group32_f16_fractional", (24, 128), 64, "f16", "i8", "group", 32, {"fractional_offset": True}),
    ("i8_chan_bf16_big_offset", (20, 128), 96, "bf16", "i8", "channel", 0, {"offset_range": (113, 127)}),
    ("i4_3d_bf16", (2, 9, 256), 128, "bf16", "i4", "group", 64, {}),
    ("i8_chan_bf16_scale2d", (20, 64), 96, "bf16", "i8", "channel", 0, {"scale_2d": True}),
    ("i8_nobias_nox3", (48, 128), 128, "bf16", "i8", "channel", 0, {"bias": False, "x3": False}),
    ("i4_splitk_m16", (16, 4096), 256, "bf16", "i4", "group", 128, {}),
    ("i8_splitk_m5", (5, 2048), 128, "f16", "i8", "channel", 0, {}),
    ("i4_m64_bn64", (64, 512), 256, "bf16", "i4", "group", 64, {}),
    ("i4_m20_bn32", (20, 512), 512, "bf16", "i4", "group", 32, {}),
    ("i4_g128_bf16_m384_split128", (384, 512), 256, "bf16", "i4", "group", 128, {}),
]


@pytest.mark.parametrize("spec", SMALL, ids=[s[0] for s in SMALL])
def test_wqmm_small_parity(spec):
    name, x1s, n, act, wdt, mode, G, extra = spec
    case = WL.make_wqmm_case(name=name, x1_shape=x1s, n=n, act=act, wdt=wdt, mode=mode, group_size=G,
                             seed=zlib.crc32(name.encode()) % 10000, **extra)
    check_wqmm(case)


# ---------------------------------------------------------------- non-quantised scenario
# x2 of the x1 dtype, no antiquant factors: out = x1 @ x2 + bias + x3.  The
# 16-bit weight is re-laid into the packed tiles and copied into the MMA's
# tensor-memory operand as it is.  Narrow (split k steps), wide and ragged m
# tiles, a k tail, 3-D x1, no bias/x3, and the transposed storage.
NONQUANT = [
    # name, x1_shape, n, act, extras
    ("nq_bf16_m16_split", (16, 4096), 256, "bf16", {}),
    ("nq_f16_m40_ktail", (40, 320), 192, "f16", {}),
    ("nq_bf16_m300", (300, 512), 384, "bf16", {}),
    ("nq_f16_m200_transposed", (200, 256), 256, "f16", {"x2_transposed": True}),
    ("nq_bf16_3d", (2, 9, 256), 128, "bf16", {}),
    ("nq_f16_nobias_nox3", (64, 128), 128, "f16", {"bias": False, "x3": False}),
    ("nq_bf16_k96", (24, 96), 160, "bf16", {}),
]


@pytest.mark.parametrize("pack", [True, False], ids=["prepacked", "nd"])
@pytest.mark.parametrize("spec", NONQUANT, ids=[s[0] for s in NONQUANT])
def test_wqmm_non_quantised_parity(spec, pack):
    name, x1s, n, act, extra = spec
    case = WL.make_wqmm_case(name=name, x1_shape=x1s, n=n, act=act, wdt=act, seed=zlib.crc32(name.encode()) % 10000,
                             **extra)
    assert case.scale is None
    check_wqmm(case, pack=pack)


def test_pack_kernel_16bit_layout():
    # chunk c (k values 8c .. 8c+7 of the tile) of column r at (c * 128 + r) * 16
    case = WL.make_wqmm_case(x1_shape=(1, 128), n=192, act="bf16", wdt="bf16", seed=7)
    d = C.wqmm_to_device(case, pack=True)
    torch.cuda.synchronize()
    got = d.packed.cpu().numpy().view(np.uint16)
    k, n = 128, 192
    w = np.zeros((256, 128), dtype=np.uint16)  # (n padded to 2 blocks, k)
    w[:n, :k] = case.x2.T
    want = w.reshape(2, 128, 2, 8, 8).transpose(0, 2, 3, 1, 4).reshape(-1)  # (nb, kt, c, r, 8)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- row-parallel shards
# The operator's tensor-parallel form splits x1 and x2 along k; each rank runs
# the GEMM on its shard (bias and x3 included) and the AllReduce sums the
# outputs.  Here every rank's part runs on this one GPU through the package's
# shard helpers and matmul_all_reduce (no process group: the AllReduce is the
# identity); the outputs are summed as a sum AllReduce would, and the sum is
# held to the sum of the ranks' exact results.
ROWPAR = [
    ("rp_i4_g128_bf16", dict(x1_shape=(40, 1024), n=256, act="bf16", wdt="i4", mode="group", group_size=128,
                             scale_range=(0.005, 0.05), offset_range=(-4, 4), seed=51), True),
    ("rp_i4_g64_f16_transposed", dict(x1_shape=(24, 512), n=128, act="f16", wdt="i4", mode="group", group_size=64,
                                      x2_transposed=True, scale_transposed=True, seed=52), True),
    ("rp_i8_chan_bf16_m300", dict(x1_shape=(300, 640), n=192, act="bf16", wdt="i8", mode="channel", seed=53), False),
    ("rp_fp8_chan_bf16", dict(x1_shape=(64, 512), n=128, act="bf16", wdt="fp8", mode="channel", offset=False,
                              seed=55), False),
    ("rp_nonquant_bf16", dict(x1_shape=(16, 512), n=128, act="bf16", wdt="bf16", seed=54), False),
]


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("spec", ROWPAR, ids=[s[0] for s in ROWPAR])
def test_row_parallel_shards_sum_to_the_operator(spec, world):
    from rowparallel_cases import local_oracle, shard_case
    from weight_quantized_gemm_anti_b200 import allreduce as AR
    name, kw, int4 = spec
    case = WL.make_wqmm_case(name=name, **kw)
    adt = torch.bfloat16 if case.act == "bf16" else torch.float16
    wcode = {"i8": W.DT_I8, "fp8": W.DT_FP8E4M3, "bf16": W.DT_BF16, "f16": W.DT_F16}.get(case.wdt)
    dev = lambda t: None if t is None else t.cuda()
    bias = None if case.bias is None else torch.from_numpy(case.bias.view(np.int16)).cuda().view(adt)
    x3 = None if case.x3 is None else torch.from_numpy(case.x3.view(np.int16)).cuda().view(adt).reshape(case.out_shape)
    total = np.zeros((case.m, case.n))
    want = np.zeros((case.m, case.n))
    bound = 0.0
    for r in range(world):
        k0, k1, x1, x2, sc, of = shard_case(case, r, world, int4)
        x1 = x1.cuda().view(adt)
        buf, x2d = AR.pack_shard(x2.cuda(), k1 - k0, case.n, int4=int4, transposed=case.x2_transposed, dtype=wcode)
        sc, of = dev(sc), dev(of)
        sc = None if sc is None else sc.view(adt)
        of = None if of is None else of.view(adt)
        if case.mode == "group" and case.scale_transposed:
            sc, of = sc.t(), (None if of is None else of.t())
        elif case.mode != "group" and sc is not None:
            sc = sc.reshape(case.scale_shape)
            of = None if of is None else of.reshape(case.scale_shape)
        out = AR.matmul_all_reduce(x1, x2d, sc, of, bias, x3, case.group_size)
        torch.cuda.synchronize()
        no_device_error()
        total += dec(gpu_bits(out), case.act)
        ye = local_oracle(case, r, world, int4)
        want += ye
        bound += np.abs(ye).max()
    err = np.abs(total - want).max() / bound
    assert err <= TOL[case.act], f"{name} x{world}: {err:.3e}"


# ---------------------------------------------------------------- small m (m <= 32)
# The small-m kernel: dequantisation groups that issue their own MMAs, x1
# fetched per turn by the groups, per-group scale/offset rows staged with the
# weights.  Even k-step counts take two-step turns, odd ones single steps; the
# m tile is 16 rows (m <= 16) or 32.  k tails (k % 64 == 32) and ragged m and
# n, every weight type and mode, and a tile split over many CTAs (fix-up).
SMALLM = [
    # name, x1_shape, n, act, wdt, mode, G, extras
    ("sm_i4_g64_bf16_m16_odd_ksteps", (16, 320), 384, "bf16", "i4", "group", 64, {}),
    ("sm_i4_g32_f16_m7", (7, 1024), 256, "f16", "i4", "group", 32, {}),
    ("sm_i8_g64_bf16_m32_x3", (32, 768), 320, "bf16", "i8", "group", 64, {}),
    ("sm_i8_chan_bf16_k_tail", (12, 96), 160, "bf16", "i8", "channel", 0, {}),
    ("sm_i8_g32_f16_k_tail", (9, 160), 96, "f16", "i8", "group", 32, {}),
    ("sm_fp8_chan_bf16_m30", (30, 640), 256, "bf16", "fp8", "channel", 0, {"offset": False}),
    ("sm_i4_tensor_bf16_m3", (3, 2048), 512, "bf16", "i4", "tensor", 0, {}),
    ("sm_i4_g128_bf16_fractional", (16, 512), 256, "bf16", "i4", "group", 128, {"fractional_offset": True}),
    ("sm_i4_g64_bf16_m25_3d", (5, 5, 1024), 640, "bf16", "i4", "group", 64, {}),
    ("sm_i4_g64_bf16_many_owners_fixup", (16, 8192), 128, "bf16", "i4", "group", 64, {}),
    ("sm_i8_g96_bf16_rows_straddle", (20, 576), 128, "bf16", "i8", "group", 96, {}),
]


@pytest.mark.parametrize("spec", SMALLM, ids=[s[0] for s in SMALLM])
def test_wqmm_small_m_kernel_parity(spec):
    name, x1s, n, act, wdt, mode, G, extra = spec
    case = WL.make_wqmm_case(name=name, x1_shape=x1s, n=n, act=act, wdt=wdt, mode=mode, group_size=G,
                             seed=zlib.crc32(name.encode()) % 10000, **extra)
    check_wqmm(case)


@pytest.mark.parametrize("env", [{"WQMM_STREAMK": "0"}, {"WQMM_SMALLM": "0"}], ids=["whole_tiles", "general_kernel"])
@pytest.mark.parametrize("spec", [SMALLM[0], SMALLM[1], SMALLM[2], SMALLM[5], SMALLM[9]],
                         ids=[SMALLM[i][0] for i in (0, 1, 2, 5, 9)])
def test_wqmm_small_m_other_schedules(spec, env, monkeypatch):
    # the small-m kernel on whole tiles, and the general kernel's narrow m tiles
    for key, val in env.items():
        monkeypatch.setenv(key, val)
    name, x1s, n, act, wdt, mode, G, extra = spec
    case = WL.make_wqmm_case(name=name, x1_shape=x1s, n=n, act=act, wdt=wdt, mode=mode, group_size=G,
                             seed=zlib.crc32(name.encode()) % 10000, **extra)
    check_wqmm(case)


def test_split_tile_flag_wait_runs_out_and_reports(monkeypatch):
    # Failure detection without a GPU fault: the test hook makes the first
    # owner of each split tile wait (bounded, 1 ms) for a flag value that no
    # owner writes.  The kernel gives up, records code 4 (epilogue wait) in the
    # device error word and returns; the next normal call is correct.
    case = WL.make_wqmm_case(name="flag_timeout", x1_shape=(16, 2048), n=1024, act="bf16", wdt="i4", mode="group",
                             group_size=64, scale_range=(0.005, 0.05), offset_range=(-4, 4), seed=41)
    d = C.wqmm_to_device(case)
    no_device_error()
    D = W.desc
    st, ws_size, ex = W.wqmm_get_workspace_size(D(d.x1), d.x2_desc, None if d.bias is None else D(d.bias),
                                                d.scale_desc, d.offset_desc, None, None, "sum", 0, 1, d.group_size,
                                                D(d.out))
    assert st == W.SUCCESS and ws_size > 0  # split tiles: partials and flags in the workspace
    ws = torch.zeros(ws_size, dtype=torch.uint8, device="cuda")
    assert W.wqmm_debug_set_flag_wait(ex, 1_000_000, True) == W.SUCCESS
    assert W.wqmm_run(ws.data_ptr(), ws_size, ex, None) == W.SUCCESS
    assert W.wqmm_stream_wait(None, 10_000) == W.SUCCESS  # the kernel ended; nothing hung
    st, code = W.wqmm_device_error(reset=True)
    assert st == W.SUCCESS and code == 4
    # the same problem, a fresh launch, the same workspace: correct again
    C.wqmm_call(d, workspace=ws)
    torch.cuda.synchronize()
    no_device_error()
    ye, _ = oracle.wqmm(case)
    assert rel_err(dec(gpu_bits(d.out), "bf16"), ye) <= TOL["bf16"]


# ---------------------------------------------------------------- CTA pairs
# With the 192- or 256-row m tile (WQMM_BN), whole tiles per CTA (stream-K off)
# and WQMM_PAIR=1, two CTAs of a cluster share each MMA (cta_group::2), each
# holding half of the x1 slab and its own 128 weight columns.  Odd column-block counts leave
# the second CTA of the last pair without weights (its outputs are masked).
PAIRS = [
    # name, x1_shape, n, act, wdt, mode, G, extras
    ("pair_i4_group128_bf16_ragged", (400, 640), 384, "bf16", "i4", "group", 128,
     {"scale_range": (0.005, 0.05), "offset_range": (-4, 4)}),
    ("pair_i8_tensor_bf16_x3", (300, 320), 256, "bf16", "i8", "tensor", 0, {"scale_const": 0.01, "offset_const": 3.0}),
    ("pair_i8_chan_f16_oddblocks", (193, 256), 640, "f16", "i8", "channel", 0, {}),
    ("pair_i4_group64_f16_fractional", (250, 256), 256, "f16", "i4", "group", 64, {"fractional_offset": True}),
    ("pair_fp8_chan_bf16", (385, 128), 384, "bf16", "fp8", "channel", 0, {"offset": False}),
    ("pair_i8_group32_bf16_3d", (3, 70, 192), 512, "bf16", "i8", "group", 32, {}),
]


@pytest.fixture(params=["192", "256"])
def whole_tiles(request, monkeypatch):
    monkeypatch.setenv("WQMM_STREAMK", "0")
    monkeypatch.setenv("WQMM_PAIR", "1")
    monkeypatch.setenv("WQMM_BN", request.param)  # the m tiles CTA pairs are built for
    yield


@pytest.mark.parametrize("spec", PAIRS, ids=[s[0] for s in PAIRS])
def test_wqmm_cta_pair_parity(spec, whole_tiles):
    name, x1s, n, act, wdt, mode, G, extra = spec
    case = WL.make_wqmm_case(name=name, x1_shape=x1s, n=n, act=act, wdt=wdt, mode=mode, group_size=G,
                             seed=zlib.crc32(name.encode()) % 10000, **extra)
    check_wqmm(case)


# Whole tiles on single CTAs (m > 128: 128- and 192-row m tiles): with an even
# number of k steps the dequantisation groups take turns of two k steps (their
# per-turn waits, bookkeeping and scale/offset loads shared); with an odd number
# they take one step per turn.
WHOLE = [
    ("whole_i4_g128_bf16", (400, 1024), 256, "bf16", "i4", "group", 128, {"scale_range": (0.005, 0.05),
                                                                          "offset_range": (-4, 4)}),
    ("whole_i4_g32_bf16", (300, 512), 384, "bf16", "i4", "group", 32, {}),
    ("whole_i4_g96_f16_rows_straddle", (200, 768), 256, "f16", "i4", "group", 96, {}),
    ("whole_i4_g64_bf16_fractional", (257, 512), 128, "bf16", "i4", "group", 64, {"fractional_offset": True}),
    ("whole_i4_chan_bf16_odd_ksteps", (300, 320), 256, "bf16", "i4", "channel", 0, {}),
    ("whole_i8_tensor_bf16_x3", (330, 640), 192, "bf16", "i8", "tensor", 0, {"scale_const": 0.01,
                                                                             "offset_const": 3.0}),
    ("whole_i8_g64_f16", (140, 256), 160, "f16", "i8", "group", 64, {}),
    ("whole_i8_chan_bf16_k_ragged", (200, 352), 96, "bf16", "i8", "channel", 0, {}),
    ("whole_fp8_chan_bf16", (150, 512), 128, "bf16", "fp8", "channel", 0, {"offset": False}),
    ("whole_i4_g128_bf16_bn128", (100, 512), 256, "bf16", "i4", "group", 128, {}),
]


@pytest.mark.parametrize("bn", ["192", "256"])
@pytest.mark.parametrize("spec", WHOLE, ids=[s[0] for s in WHOLE])
def test_wqmm_whole_tiles_parity(spec, bn, monkeypatch):
    monkeypatch.setenv("WQMM_STREAMK", "0")
    monkeypatch.setenv("WQMM_PAIR", "0")
    if spec[1][0] > 128:  # the m tile of wide problems: two TMEM accumulators (192) or one (256)
        monkeypatch.setenv("WQMM_BN", bn)
    name, x1s, n, act, wdt, mode, G, extra = spec
    case = WL.make_wqmm_case(name=name, x1_shape=x1s, n=n, act=act, wdt=wdt, mode=mode, group_size=G,
                             seed=zlib.crc32(name.encode()) % 10000, **extra)
    check_wqmm(case)


# ---------------------------------------------------------------- split last wave
# Narrow m tiles, more tiles than CTAs, the last wave partly filled: whole tiles
# for the full waves, then the k steps of the remaining tiles split evenly over
# the CTAs.  With at most four owners per split tile the owner of its first k
# steps adds the others' partials itself (inline); with more, or with
# WQMM_SK_INLINE=0, every owner writes a partial and the fix-up kernel reduces.
# Wide tiles use stream-K only when there are fewer tiles than CTAs (then with
# two-step units and two-step dequantisation turns).  WQMM_GRID shrinks the
# persistent grid so that these schedules arise at sizes the oracle computes
# quickly.
# name, x1_shape, n, act, wdt, mode, G, extras, grid (None: all SMs), env
HYBRID = [
    # 18 tiles on 8 CTAs: 16 whole + 2 split four ways (inline)
    ("hyb_i4_g64_bf16_m40", (40, 512), 2304, "bf16", "i4", "group", 64, {"scale_range": (0.005, 0.05),
                                                                       "offset_range": (-4, 4)}, 8, {}),
    ("hyb_i4_g64_bf16_m40_fixup", (40, 512), 2304, "bf16", "i4", "group", 64, {}, 8, {"WQMM_SK_INLINE": "0"}),
    ("hyb_i8_chan_f16_m16", (16, 640), 1280, "f16", "i8", "channel", 0, {}, 4, {}),
    ("hyb_i4_g128_bf16_m64_bias_x3", (64, 1024), 1152, "bf16", "i4", "group", 128, {}, 4, {}),
    ("hyb_fp8_chan_bf16_m32", (32, 512), 640, "bf16", "fp8", "channel", 0, {"offset": False}, 2, {}),
    ("hyb_i8_tensor_bf16_m24_x3", (24, 640), 768, "bf16", "i8", "tensor", 0, {"scale_const": 0.01,
                                                                              "offset_const": 3.0}, 4, {}),
    # one split tile over eight owners: the fix-up kernel
    ("hyb_i8_g32_bf16_m20_eight_owners", (20, 1024), 1152, "bf16", "i8", "group", 32, {}, 8, {}),
    # wide tiles, fewer tiles than CTAs: every tile split (two-step units), inline
    ("sk_wide_i4_g128_bf16", (300, 512), 256, "bf16", "i4", "group", 128, {}, None, {}),
    ("sk_wide_i8_chan_f16_odd_ksteps", (200, 448), 384, "f16", "i8", "channel", 0, {}, None, {}),
]


@pytest.mark.parametrize("spec", HYBRID, ids=[s[0] for s in HYBRID])
def test_wqmm_split_last_wave_parity(spec, monkeypatch):
    name, x1s, n, act, wdt, mode, G, extra, grid, env = spec
    if grid:
        monkeypatch.setenv("WQMM_GRID", str(grid))
    monkeypatch.setenv("WQMM_PAIR", "0")
    for key, val in env.items():
        monkeypatch.setenv(key, val)
    case = WL.make_wqmm_case(name=name, x1_shape=x1s, n=n, act=act, wdt=wdt, mode=mode, group_size=G,
                             seed=zlib.crc32(name.encode()) % 10000, **extra)
    d = C.wqmm_to_device(case)
    ws = C.wqmm_call(d)
    torch.cuda.synchronize()
    no_device_error()
    assert ws is not None and ws.numel() > 0, "a stream-K plan keeps fp32 partials in the workspace"
    first = gpu_bits(d.out)
    ye, _ = oracle.wqmm(case)
    g = dec(first, case.act)
    assert np.isfinite(g).all()
    assert rel_err(g, ye) <= TOL[case.act], f"{name}: rel err {rel_err(g, ye):.3e}"
    # a second run repeats every bit (the fix-up sums partials in a fixed order)
    C.wqmm_call(d, workspace=ws)
    torch.cuda.synchronize()
    no_device_error()
    assert np.array_equal(first, gpu_bits(d.out)), f"{name}: repeated runs differ"
    # and whole tiles on the same grid agree within the tolerance
    monkeypatch.setenv("WQMM_STREAMK", "0")
    whole = dec(run_wqmm(case), case.act)
    assert rel_err(g, whole) <= TOL[case.act]


def test_wqmm_inline_stream_k_graph_replays(monkeypatch):
    # A launch recorded into a CUDA graph replays with the same flag token: each
    # replay must still wait for its own owners' partials (the first owner
    # clears the flags it consumed).  x1 changes between replays, so partials
    # left from an earlier replay would show in the result.
    import dataclasses
    monkeypatch.setenv("WQMM_GRID", "8")
    monkeypatch.setenv("WQMM_PAIR", "0")
    case = WL.make_wqmm_case(name="graph_sk", x1_shape=(40, 512), n=2304, act="bf16", wdt="i4", mode="group",
                             group_size=64, scale_range=(0.005, 0.05), offset_range=(-4, 4), seed=7)
    d = C.wqmm_to_device(case)
    ws = C.wqmm_call(d)
    torch.cuda.synchronize()
    assert ws is not None and ws.numel() > 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        C.wqmm_call(d, workspace=ws)
    for r in range(3):
        x1 = WL.act_bits(np.random.default_rng(100 + r).standard_normal(size=case.x1_shape), case.act)
        d.x1.view(torch.int16).copy_(torch.from_numpy(np.ascontiguousarray(x1).view(np.int16)).to(d.x1.device))
        g.replay()
        torch.cuda.synchronize()
        no_device_error()
        ye, _ = oracle.wqmm(dataclasses.replace(case, x1=x1))
        got = dec(gpu_bits(d.out), case.act)
        assert rel_err(got, ye) <= TOL[case.act], f"replay {r}: rel err {rel_err(got, ye):.3e}"
    del g


def test_wqmm_cta_pair_matches_single_cta(monkeypatch):
    # the same problem with and without CTA pairs: both within tolerance of the
    # oracle, and close to each other
    monkeypatch.setenv("WQMM_STREAMK", "0")
    monkeypatch.setenv("WQMM_PAIR", "1")
    monkeypatch.setenv("WQMM_BN", "192")
    case = WL.make_wqmm_case(name="pair_vs_single", x1_shape=(512, 1024), n=512, act="bf16", wdt="i4", mode="group",
                             group_size=128, scale_range=(0.005, 0.05), offset_range=(-4, 4), seed=11)
    a = dec(run_wqmm(case), case.act)
    monkeypatch.setenv("WQMM_PAIR", "0")
    b = dec(run_wqmm(case), case.act)
    ye, _ = oracle.wqmm(case)
    assert rel_err(a, ye) <= TOL[case.act]
    assert rel_err(b, ye) <= TOL[case.act]
    assert rel_err(a, b) <= TOL[case.act]


@pytest.mark.parametrize("wdt,mode,G", [("i8", "group", 32), ("i4", "group", 64), ("fp8", "channel", 0),
                                        ("i8", "channel", 0)])
def test_wqmm_transposed_weight(wdt, mode, G):
    case = WL.make_wqmm_case(name="t", x1_shape=(40, 256), n=192 if wdt != "i4" else 256, act="bf16", wdt=wdt,
                             mode=mode, group_size=G, x2_transposed=True, scale_transposed=(mode == "group"),
                             offset=(wdt != "fp8"), seed=7)
    check_wqmm(case, pack=True)
    check_wqmm(case, pack=False)


def test_nd_weight_packed_inside_run_matches_prepacked():
    case = WL.make_wqmm_case(x1_shape=(77, 256), n=192, act="bf16", wdt="i8", mode="group", group_size=64, seed=3)
    a = run_wqmm(case, pack=True)
    b = run_wqmm(case, pack=False)
    assert np.array_equal(a, b)


def test_empty_k_gives_bias_plus_x3():
    case = WL.make_wqmm_case(x1_shape=(10, 0), n=96, act="bf16", wdt="i8", mode="channel", seed=4)
    got = run_wqmm(case, pack=False)
    _, yr = oracle.wqmm(case)
    assert np.array_equal(got, yr)  # a single rounding of bias + x3 on both sides


def test_page_sample_all_ones_gives_130():
    case = WL.make_wqmm_case(x1_shape=(32, 64), n=128, act="f16", wdt="i8", mode="channel", seed=0)
    one = WL.f16_bits(np.ones(1))[0]
    for a in (case.x1, case.scale, case.offset, case.bias, case.x3):
        a[:] = one
    case.x2[:] = 1
    got = dec(run_wqmm(case, pack=False), "f16")
    assert (got == 130.0).all()


def test_repeated_runs_are_bitwise_deterministic():
    case = WL.make_wqmm_case(x1_shape=(16, 4096), n=256, act="bf16", wdt="i4", mode="group", group_size=128, seed=8)
    d = C.wqmm_to_device(case)
    outs = []
    for _ in range(3):
        C.wqmm_call(d)
        torch.cuda.synchronize()
        outs.append(gpu_bits(d.out).copy())
    no_device_error()
    assert all(np.array_equal(outs[0], o) for o in outs[1:])


# ---------------------------------------------------------------- pack kernel layout
def _np_pack_wq_int4(q: np.ndarray) -> np.ndarray:
    """Independent numpy statement of the anti-quant GEMM's int4 tile layout."""
    k, n = q.shape
    NB, KT = -(-n // 128), -(-k // 64)
    u = np.zeros((NB * 128, KT * 64), dtype=np.uint32)
    u[:n, :k] = (q.T.astype(np.int64) + 8) & 0xF
    u[n:, :] = 8
    u[:, k:] = 8
    out = np.zeros((NB, KT, 2, 128, 4), dtype=np.uint32)
    for c in range(2):
        for w in range(4):
            word = np.zeros((NB * 128, KT), dtype=np.uint32)
            for j in range(4):
                word |= u[:, c * 32 + 8 * w + 2 * j::64][:, :KT] << (4 * j)
                word |= u[:, c * 32 + 8 * w + 2 * j + 1::64][:, :KT] << (16 + 4 * j)
            out[:, :, c, :, w] = word.reshape(NB, 128, KT).transpose(0, 2, 1)
    return out.reshape(-1).view(np.uint8)


def test_pack_kernel_int4_layout():
    case = WL.make_wqmm_case(x1_shape=(1, 128), n=192, act="bf16", wdt="i4", mode="channel", seed=5)
    d = C.wqmm_to_device(case, pack=True)
    torch.cuda.synchronize()
    got = d.packed.cpu().numpy()
    lo, hi = case.x2 & 0xF, case.x2 >> 4
    q = np.empty((128, 192), dtype=np.int64)
    q[:, 0::2], q[:, 1::2] = lo, hi
    q = np.where(q >= 8, q - 16, q)
    assert np.array_equal(got, _np_pack_wq_int4(q))


def test_pack_kernel_int8_qmm_layout():
    case = WL.make_qmm_case(x1_shape=(4, 256), n=320, seed=6)
    d = C.qmm_to_device(case, pack=True)
    torch.cuda.synchronize()
    got = d.packed.cpu().numpy().reshape(-1)
    k, n = 256, 320
    NB, KT = 2, 2
    full = np.zeros((NB * 256, KT * 128), dtype=np.uint8)
    full[:n, :k] = case.x2.T.view(np.uint8)
    want = np.zeros((NB, KT, 256, 8, 16), dtype=np.uint8)
    for r in range(256):
        for c in range(8):
            want[:, :, r, c ^ (r & 7), :] = full.reshape(NB, 256, KT, 8, 16)[:, r, :, c, :]
    assert np.array_equal(got, want.reshape(-1))


# ---------------------------------------------------------------- int8 path
QSMALL = [
    ("q_bf16_pertoken", (32, 64), 128, "bf16", {}),
    ("q_f16_pertoken", (32, 64), 128, "f16", {}),
    ("q_bf16_ragged", (200, 160), 288, "bf16", {}),
    ("q_f16_no_pertoken", (129, 256), 256, "f16", {"pertoken": False}),
    ("q_bf16_tensor_dq", (3, 4, 96), 64, "bf16", {"dq_per_tensor": True}),
    ("q_bf16_no_bias_x3", (64, 128), 512, "bf16", {"bias": False, "x3": False}),
    ("q_f16_dq2d", (16, 64), 32, "f16", {"dq_2d": True}),
]


@pytest.mark.parametrize("spec", QSMALL, ids=[s[0] for s in QSMALL])
def test_qmm_small_parity_and_exact_accumulator(spec):
    name, x1s, n, out, extra = spec
    case = WL.make_qmm_case(name=name, x1_shape=x1s, n=n, out=out, seed=zlib.crc32(name.encode()) % 1000, **extra)
    d = C.qmm_to_device(case)
    acc = torch.empty((case.m, n), dtype=torch.int32, device="cuda")
    C.qmm_call(d, raw_acc=acc)
    torch.cuda.synchronize()
    no_device_error()
    a_ref, ye, _ = oracle.qmm(case)
    assert np.array_equal(acc.cpu().numpy(), a_ref)
    g = dec(gpu_bits(d.out), out)
    assert rel_err(g, ye) <= TOL[out]


# Clusters of two CTAs share each int8 MMA (M = 256 rows of x1, 128 per CTA;
# each CTA loads half of the 256-column weight tile).  WQMM_PAIR=1 selects it at
# any size; odd 128-row block counts leave the second CTA of the last pair
# without rows (its loads are zero-filled and its outputs masked).
QPAIR = [
    ("qp_bf16_odd_blocks", (300, 384), 512, "bf16", {}),
    ("qp_f16_no_pertoken", (256, 256), 256, "f16", {"pertoken": False}),
    ("qp_bf16_3d_no_bias_x3", (2, 200, 1024), 768, "bf16", {"bias": False, "x3": False}),
    ("qp_bf16_tensor_dq", (129, 128), 256, "bf16", {"dq_per_tensor": True}),
]


@pytest.mark.parametrize("spec", QPAIR, ids=[s[0] for s in QPAIR])
def test_qmm_cta_pair_parity_and_exact_accumulator(spec, monkeypatch):
    monkeypatch.setenv("WQMM_PAIR", "1")
    name, x1s, n, out, extra = spec
    case = WL.make_qmm_case(name=name, x1_shape=x1s, n=n, out=out, seed=zlib.crc32(name.encode()) % 1000, **extra)
    d = C.qmm_to_device(case)
    acc = torch.empty((case.m, n), dtype=torch.int32, device="cuda")
    C.qmm_call(d, raw_acc=acc)
    torch.cuda.synchronize()
    no_device_error()
    a_ref, ye, _ = oracle.qmm(case)
    assert np.array_equal(acc.cpu().numpy(), a_ref)
    g = dec(gpu_bits(d.out), out)
    assert rel_err(g, ye) <= TOL[out]


def test_qmm_transposed_weight_and_unpacked():
    case = WL.make_qmm_case(x1_shape=(40, 128), n=96, x2_transposed=True, seed=12)
    d = C.qmm_to_device(case, pack=False)
    acc = torch.empty((case.m, case.n), dtype=torch.int32, device="cuda")
    C.qmm_call(d, raw_acc=acc)
    torch.cuda.synchronize()
    a_ref, ye, _ = oracle.qmm(case)
    assert np.array_equal(acc.cpu().numpy(), a_ref)
    assert rel_err(dec(gpu_bits(d.out), "bf16"), ye) <= 4e-3


def test_qmm_page_sample_all_ones_gives_66():
    case = WL.make_qmm_case(x1_shape=(32, 64), n=128, out="f16", seed=0)
    case.x1[:] = 1
    case.x2[:] = 1
    case.bias[:] = 1
    case.dequant_scale[:] = 1.0
    case.pertoken_scale[:] = 1.0
    case.x3[:] = WL.f16_bits(np.ones(1))[0]
    d = C.qmm_to_device(case)
    C.qmm_call(d)
    torch.cuda.synchronize()
    assert (dec(gpu_bits(d.out), "f16") == 66.0).all()


# ---------------------------------------------------------------- full-size workloads (sampled)
def _sample(m, n, nr, nc, seed):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, m - 1], rng.choice(m, size=min(nr, m), replace=False)]))
    cols = np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=min(nc, n), replace=False)]))
    return rows, cols


@pytest.mark.parametrize("name", [nm for nm in WL.WORKLOAD_NAMES if not nm.startswith("w8a8")])
def test_full_size_workload_sampled(name):
    case = WL.workload(name)
    rows, cols = _sample(case.m, case.n, 96, 768, 1)
    check_wqmm(case, rows=rows, cols=cols)


def test_full_size_int8_workload_sampled():
    case = WL.workload("w8a8_pertoken_4x2048x8192x1024")
    d = C.qmm_to_device(case)
    acc = torch.empty((case.m, case.n), dtype=torch.int32, device="cuda")
    C.qmm_call(d, raw_acc=acc)
    torch.cuda.synchronize()
    no_device_error()
    rows, cols = _sample(case.m, case.n, 64, 512, 2)
    a_ref, ye, _ = oracle.qmm(case, rows=rows, cols=cols)
    assert np.array_equal(acc.cpu().numpy()[np.ix_(rows, cols)], a_ref)
    g = dec(gpu_bits(d.out)[np.ix_(rows, cols)], "bf16")
    assert rel_err(g, ye) <= 4e-3
