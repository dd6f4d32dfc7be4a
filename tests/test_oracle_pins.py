"""Pins for the CPU oracle: checks against things other than the oracle itself.

* format codecs vs numpy fp16, torch bf16 / fp8-e4m3fn and exact rational rounding;
* the anti-quant GEMM vs an exact rational (fractions.Fraction) brute force on
  tiny inputs, in every mode / weight type / layout, including a ragged last group;
* the page samples' closed forms (tests/golden);
* invariants that reduce to a library routine (torch fp64 matmul, numpy int64
  matmul) or to another mode of the same formula.
"""
import itertools
import math
import os
import zlib
from fractions import Fraction

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ independent decoders
def dec_f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def dec_bf16(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dec_act(bits, act):
    return dec_f16(bits) if act == "f16" else dec_bf16(bits)


def dec_e4m3(bits):
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def unpack_i4(packed, rows, cols):
    """Independent unpack: (rows, cols/2) bytes -> (rows, cols) int values, low nibble first."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    lo, hi = p & 0xF, (p >> 4) & 0xF
    out = np.empty((rows, cols), dtype=np.int64)
    out[:, 0::2], out[:, 1::2] = lo, hi
    return np.where(out >= 8, out - 16, out)


def weights_kn(case):
    """(k, n) float64 weight values decoded by the test's own code."""
    k, n = case.k, case.n
    if case.wdt == "i8":
        q = case.x2.astype(np.float64)
        return q.T if case.x2_transposed else q
    if case.wdt == "fp8":
        q = dec_e4m3(case.x2)
        return q.T if case.x2_transposed else q
    if case.x2_transposed:
        return unpack_i4(case.x2, n, k).T.astype(np.float64)
    return unpack_i4(case.x2, k, n).astype(np.float64)


def factors_kn(case, tensor):
    """Expand scale/offset to per-element (k, n) factors (repeat rows per group)."""
    k, n = case.k, case.n
    v = dec_act(tensor, case.act)
    if case.mode == "tensor":
        return np.full((k, n), v.reshape(-1)[0])
    if case.mode == "channel":
        return np.broadcast_to(v.reshape(1, n), (k, n))
    if case.scale_transposed:
        v = v.T
    return np.repeat(v, case.group_size, axis=0)[:k]


# ------------------------------------------------------------------ exact rational rounding
def rne_fraction(x: Fraction, p: int, emin: int, maxfinite: Fraction):
    """Round x to p significant bits, min normal exponent emin, ties to even; inf on overflow."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    E = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** E > a:
        E -= 1
    while Fraction(2) ** (E + 1) <= a:
        E += 1
    E = max(E, emin)
    q = Fraction(2) ** (E - (p - 1))
    r = a / q
    fl = r.numerator // r.denominator
    rem = r - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    v = fl * q
    if v > maxfinite:
        return math.inf * sign
    return sign * v


BF16_MAX = Fraction(255) * Fraction(2) ** 120
F16_MAX = Fraction(65504)


def rne_act(x: Fraction, act):
    return rne_fraction(x, 11, -14, F16_MAX) if act == "f16" else rne_fraction(x, 8, -126, BF16_MAX)


# ------------------------------------------------------------------ codec pins
def test_f16_decode_all_codes():
    codes = np.arange(65536, dtype=np.uint16)
    ref = dec_f16(codes)
    got = np.array([oracle.f16_to_double(c) for c in codes])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    m = ~np.isnan(ref)
    assert np.array_equal(ref[m], got[m])


def test_bf16_decode_all_codes():
    codes = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(codes.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_double(c) for c in codes])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    m = ~np.isnan(ref)
    assert np.array_equal(ref[m], got[m])


def test_e4m3_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = dec_e4m3(codes)
    got = np.array([oracle.e4m3_to_double(c) for c in codes])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    m = ~np.isnan(ref)
    assert np.array_equal(ref[m], got[m])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def _encode_samples():
    rng = np.random.default_rng(123)
    xs = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-9, 6, 3000))
    # exact halfway points between adjacent fp16 / bf16 values (ties), both parities
    for b in [1, 2, 3, 0x3C00, 0x3C01, 0x7BFE, 0x0400, 0x03FF]:
        a, c = float(np.uint16(b).view(np.float16)), float(np.uint16(b + 1).view(np.float16))
        xs += [(a + c) / 2, -(a + c) / 2]
    for b in [1, 2, 0x3F80, 0x3F81, 0x0080, 0x007F, 0x7F7E, 0x4300]:
        a, c = float(dec_bf16(b)), float(dec_bf16(b + 1))
        xs += [(a + c) / 2, -(a + c) / 2]
    xs += [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e-8, 6e-8, 3.0e38, 3.4e38, 1e-40]
    return xs


def test_f16_encode_matches_numpy_rne():
    for x in _encode_samples():
        with np.errstate(over="ignore"):
            want = np.float64(x).astype(np.float16).view(np.uint16)
        assert oracle.double_to_f16(x) == int(want), x


def test_bf16_encode_matches_exact_rational_rne():
    for x in _encode_samples():
        r = rne_act(Fraction(x), "bf16")
        got = float(dec_bf16(oracle.double_to_bf16(x)))
        if isinstance(r, float) and math.isinf(r):
            assert math.isinf(got) and (got > 0) == (r > 0), x
        else:
            assert got == float(r), x


def test_bf16_encode_matches_torch_on_fp32_values():
    rng = np.random.default_rng(5)
    xs = rng.standard_normal(5000).astype(np.float32) * np.float32(1000)
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([oracle.double_to_bf16(float(x)) for x in xs], dtype=np.uint16)
    assert np.array_equal(ref, got)


# ------------------------------------------------------------------ brute force (exact)
def brute_force_wqmm(case):
    """Exact rational y = x1 @ ((x2 + off) * scale) + bias + x3 over all outputs."""
    m, k, n = case.m, case.k, case.n
    x1 = [[Fraction(float(v)) for v in row] for row in dec_act(case.x1.reshape(m, k), case.act)]
    wq = weights_kn(case)
    s = factors_kn(case, case.scale)
    o = factors_kn(case, case.offset) if case.offset is not None else np.zeros((k, n))
    Wf = [[(Fraction(float(wq[a, b])) + Fraction(float(o[a, b]))) * Fraction(float(s[a, b])) for b in range(n)]
          for a in range(k)]
    bias = dec_act(case.bias, case.act) if case.bias is not None else np.zeros(n)
    x3 = dec_act(case.x3.reshape(m, n), case.act) if case.x3 is not None else np.zeros((m, n))
    y = [[sum((x1[i][a] * Wf[a][j] for a in range(k)), Fraction(0)) + Fraction(float(bias[j])) +
          Fraction(float(x3[i, j])) for j in range(n)] for i in range(m)]
    return y


BF_CASES = []
for act, wdt, mode, transposed in itertools.product(["f16", "bf16"], ["i8", "i4", "fp8"],
                                                    ["tensor", "channel", "group"], [False, True]):
    if wdt == "fp8" and mode != "channel":
        continue
    BF_CASES.append((act, wdt, mode, transposed))


@pytest.mark.parametrize("act,wdt,mode,transposed", BF_CASES)
def test_wqmm_matches_exact_brute_force(act, wdt, mode, transposed):
    seed = zlib.crc32(f"{act}/{wdt}/{mode}/{transposed}".encode()) % 1000
    case = W.make_wqmm_case(x1_shape=(3, 64), n=6, act=act, wdt=wdt, mode=mode, group_size=32,
                            x2_transposed=transposed, scale_transposed=transposed, scale_range=(0.01, 0.2),
                            offset=(wdt != "fp8"), seed=seed, fractional_offset=(seed % 2 == 0))
    exact = brute_force_wqmm(case)
    ye, yr = oracle.wqmm(case)
    for i in range(case.m):
        for j in range(case.n):
            e = exact[i][j]
            assert abs(ye[i, j] - float(e)) <= 1e-13 * max(1.0, abs(float(e))), (i, j)
            want = rne_act(e, act)
            got = float(dec_act(yr[i, j], act))
            assert got == float(want), (i, j, got, float(want))


@settings(max_examples=25, deadline=None, derandomize=True)
@given(act=st.sampled_from(["f16", "bf16"]), wdt=st.sampled_from(["i8", "i4", "fp8"]),
       mode=st.sampled_from(["tensor", "channel", "group"]), transposed=st.booleans(),
       m=st.integers(1, 3), k_units=st.integers(1, 3), n_pairs=st.integers(1, 3), g_units=st.integers(1, 3),
       fractional=st.booleans(), seed=st.integers(0, 10_000))
def test_wqmm_brute_force_random_shapes(act, wdt, mode, transposed, m, k_units, n_pairs, g_units, fractional, seed):
    # random small shapes, modes and layouts, including group sizes that do not
    # divide k (a short last group): the oracle equals the exact rational value
    if wdt == "fp8":
        mode = "channel"
    k, n, G = 32 * k_units, 2 * n_pairs, 32 * g_units
    case = W.make_wqmm_case(x1_shape=(m, k), n=n, act=act, wdt=wdt, mode=mode, group_size=G,
                            x2_transposed=transposed, scale_transposed=transposed and mode == "group",
                            scale_range=(0.01, 0.2), offset=(wdt != "fp8"), fractional_offset=fractional, seed=seed)
    exact = brute_force_wqmm(case)
    ye, yr = oracle.wqmm(case)
    for i in range(m):
        for j in range(n):
            e = exact[i][j]
            assert abs(ye[i, j] - float(e)) <= 1e-13 * max(1.0, abs(float(e))), (i, j)
            assert float(dec_act(yr[i, j], act)) == float(rne_act(e, act)), (i, j)


def test_wqmm_ragged_last_group_brute_force():
    # group size 5 does not divide k = 13: the last group covers rows 10..12 only.
    case = W.make_wqmm_case(x1_shape=(2, 13), n=4, act="bf16", wdt="i8", mode="group", group_size=5,
                            scale_range=(0.01, 0.1), seed=77)
    assert case.scale.shape == (3, 4)
    exact = brute_force_wqmm(case)
    ye, _ = oracle.wqmm(case)
    for i in range(2):
        for j in range(4):
            assert abs(ye[i, j] - float(exact[i][j])) <= 1e-13 * max(1.0, abs(float(exact[i][j])))


def test_qmm_matches_exact_integer_brute_force():
    case = W.make_qmm_case(x1_shape=(5, 96), n=7, out="bf16", seed=3)
    acc, ye, yr = oracle.qmm(case)
    x1 = case.x1.astype(object)
    x2 = case.x2.astype(object)
    dq = dec_bf16(case.dequant_scale)
    x3 = dec_bf16(case.x3)
    for i in range(5):
        for j in range(7):
            a = sum(int(x1[i, t]) * int(x2[t, j]) for t in range(96)) + int(case.bias[j])
            assert acc[i, j] == a
            e = Fraction(a) * Fraction(float(dq[j])) * Fraction(float(case.pertoken_scale[i])) + Fraction(float(x3[i, j]))
            assert abs(ye[i, j] - float(e)) <= 1e-13 * max(1.0, abs(float(e)))
            assert float(dec_bf16(yr[i, j])) == float(rne_act(e, "bf16"))


@settings(max_examples=30, deadline=None, derandomize=True)
@given(m=st.integers(1, 6), k=st.integers(1, 80), n=st.integers(1, 6), out=st.sampled_from(["bf16", "f16"]),
       pertoken=st.booleans(), dq_per_tensor=st.booleans(), bias=st.booleans(), seed=st.integers(0, 10_000))
def test_qmm_random_shapes_exact_accumulator(m, k, n, out, pertoken, dq_per_tensor, bias, seed):
    # the int8 path's accumulator is the exact integer product plus bias (no
    # wrap at these sizes), over random shapes and options
    case = W.make_qmm_case(x1_shape=(m, k), n=n, out=out, bias=bias, x3=True, pertoken=pertoken,
                           dq_per_tensor=dq_per_tensor, seed=seed)
    acc, ye, _ = oracle.qmm(case)
    want = case.x1.astype(np.int64) @ case.x2.astype(np.int64)
    if case.bias is not None:
        want = want + case.bias.astype(np.int64)[None, :]
    assert np.array_equal(acc.astype(np.int64), want)


def test_qmm_int32_wraps_like_a_32bit_accumulator():
    case = W.make_qmm_case(x1_shape=(2, 32), n=3, out="bf16", seed=9, pertoken=False, x3=False)
    case.x1[:] = 127
    case.x2[:] = 127
    case.bias[:] = np.int32(2**31 - 1)
    acc, _, _ = oracle.qmm(case)
    s = 32 * 127 * 127 + (2**31 - 1)
    want = ((s + 2**31) % 2**32) - 2**31
    assert (acc == want).all() and want < 0


# ------------------------------------------------------------------ page sample closed forms
def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *rest = line.split()
                vals[key] = rest
    return vals


def test_page_sample_wqmm_all_ones_is_130():
    g = _read_golden("page_sample_wqmm_allones.txt")
    m, k = map(int, g["x1_shape"])
    n = int(g["x2"][2])
    one = W.f16_bits(np.ones(1))[0]
    case = W.make_wqmm_case(x1_shape=(m, k), n=n, act="f16", wdt="i8", mode="channel", seed=0)
    case.x1[:] = one
    case.x2[:] = 1
    case.scale[:] = one
    case.offset[:] = one
    case.bias[:] = one
    case.x3[:] = one
    ye, yr = oracle.wqmm(case)
    want = float(g["expected_every_output"][0])
    assert (ye == want).all()
    assert (dec_f16(yr) == want).all()


def test_page_sample_qmm_all_ones_is_66():
    g = _read_golden("page_sample_qmm_allones.txt")
    m, k = map(int, g["x1_shape"])
    n = int(g["x2_shape"][1])
    case = W.make_qmm_case(x1_shape=(m, k), n=n, out="f16", seed=0)
    case.x1[:] = 1
    case.x2[:] = 1
    case.bias[:] = 1
    case.dequant_scale[:] = 1.0
    case.pertoken_scale[:] = 1.0
    case.x3[:] = W.f16_bits(np.ones(1))[0]
    acc, ye, yr = oracle.qmm(case)
    want = float(g["expected_every_output"][0])
    assert (acc == 65).all() and (ye == want).all() and (dec_f16(yr) == want).all()


# ------------------------------------------------------------------ invariants
def test_zero_offset_unit_scale_is_plain_matmul():
    case = W.make_wqmm_case(x1_shape=(7, 96), n=40, act="bf16", wdt="i8", mode="tensor", scale_const=1.0,
                            offset_const=0.0, seed=11)
    ye, _ = oracle.wqmm(case)
    x1 = torch.from_numpy(dec_bf16(case.x1))
    q = torch.from_numpy(case.x2.astype(np.float64))
    ref = torch.matmul(x1, q) + torch.from_numpy(dec_bf16(case.bias)) + torch.from_numpy(dec_bf16(case.x3))
    np.testing.assert_allclose(ye, ref.numpy(), rtol=0, atol=1e-9)


def test_int4_zero_offset_unit_scale_is_plain_matmul():
    case = W.make_wqmm_case(x1_shape=(5, 128), n=64, act="f16", wdt="i4", mode="tensor", scale_const=1.0,
                            offset_const=0.0, bias=False, x3=False, seed=12)
    ye, _ = oracle.wqmm(case)
    q = torch.from_numpy(unpack_i4(case.x2, 128, 64).astype(np.float64))
    ref = torch.matmul(torch.from_numpy(dec_f16(case.x1)), q)
    np.testing.assert_allclose(ye, ref.numpy(), rtol=0, atol=1e-9)


@pytest.mark.parametrize("act,transposed", [("bf16", False), ("f16", False), ("bf16", True)])
def test_non_quantised_is_torch_fp64_matmul(act, transposed):
    # the non-quantised scenario (x2 of the x1 dtype, no antiquant factors):
    # out = x1 @ x2 + bias + x3, pinned against torch's float64 matmul on
    # values decoded by the test's own code
    case = W.make_wqmm_case(x1_shape=(2, 5, 96), n=48, act=act, wdt=act, x2_transposed=transposed, seed=21)
    assert case.mode == "none" and case.scale is None and case.offset is None
    ye, yr = oracle.wqmm(case)
    w = dec_act(case.x2, act)
    w = w.T if transposed else w
    ref = (torch.from_numpy(dec_act(case.x1, act).reshape(case.m, case.k)) @ torch.from_numpy(w)
           + torch.from_numpy(dec_act(case.bias, act)) + torch.from_numpy(dec_act(case.x3, act).reshape(case.m, case.n)))
    np.testing.assert_allclose(ye, ref.numpy(), rtol=0, atol=1e-12)
    # one rounding of the exact value: within half an ulp of the format
    got = dec_act(yr, act)
    ulp = np.exp2(np.floor(np.log2(np.abs(ye) + 1e-300)) - (10 if act == "f16" else 7))
    assert (np.abs(got - ye) <= 0.5 * ulp + 1e-300).all()


def test_non_quantised_rejects_antiquant_factors_and_mixed_dtypes():
    case = W.make_wqmm_case(x1_shape=(3, 64), n=32, act="bf16", wdt="bf16", seed=22)
    args = dict(m=case.m, k=case.k, n=case.n, act="bf16", wdt="bf16", x1=case.x1, x2=case.x2,
                x2_strides=case.x2_strides,
                mode="none", group_size=0, scale_strides=(0, 1))
    one = np.full((case.n,), 0x3F80, dtype=np.uint16)  # bf16 1.0
    with pytest.raises(ValueError):
        oracle.wqmm_raw(**args, scale=None, offset=one)             # an offset without a scale
    with pytest.raises(ValueError):
        oracle.wqmm_raw(**{**args, "act": "f16"}, scale=None, offset=None)  # x2 of another dtype
    with pytest.raises(ValueError):
        oracle.wqmm_raw(**{**args, "wdt": "i8"}, scale=None, offset=None)   # a quantised weight needs a scale


def test_identical_group_rows_equal_per_channel():
    g = W.make_wqmm_case(x1_shape=(6, 128), n=32, act="bf16", wdt="i4", mode="group", group_size=32, seed=13)
    c = W.make_wqmm_case(x1_shape=(6, 128), n=32, act="bf16", wdt="i4", mode="channel", seed=13)
    g.scale[:] = c.scale[None, :]
    g.offset[:] = c.offset[None, :]
    g.x1, g.x2, g.bias, g.x3 = c.x1, c.x2, c.bias, c.x3
    assert np.array_equal(oracle.wqmm(g)[0], oracle.wqmm(c)[0])


def test_group_size_k_equals_per_channel_on_oracle_core():
    c = W.make_wqmm_case(x1_shape=(4, 96), n=16, act="f16", wdt="i8", mode="channel", seed=14)
    ye_c, _ = oracle.wqmm(c)
    ye_g, _ = oracle.wqmm_raw(m=4, k=96, n=16, act="f16", x1=c.x1, wdt="i8", x2=c.x2, x2_strides=(16, 1),
                              mode="group", group_size=96, scale=c.scale.reshape(1, 16),
                              offset=c.offset.reshape(1, 16), scale_strides=(16, 1), bias=c.bias, x3=c.x3)
    assert np.array_equal(ye_c, ye_g)


def test_constant_per_channel_equals_per_tensor():
    t = W.make_wqmm_case(x1_shape=(5, 64), n=24, act="bf16", wdt="i8", mode="tensor", scale_const=0.03,
                         offset_const=-2.0, seed=15)
    c = W.make_wqmm_case(x1_shape=(5, 64), n=24, act="bf16", wdt="i8", mode="channel", seed=15)
    c.scale[:] = t.scale[0]
    c.offset[:] = t.offset[0]
    c.x1, c.x2, c.bias, c.x3 = t.x1, t.x2, t.bias, t.x3
    assert np.array_equal(oracle.wqmm(t)[0], oracle.wqmm(c)[0])


def test_linear_in_bias_and_x3():
    a = W.make_wqmm_case(x1_shape=(4, 64), n=16, act="bf16", wdt="i8", mode="channel", seed=16)
    y_full, _ = oracle.wqmm(a)
    b, x3 = a.bias, a.x3
    a.bias, a.x3 = None, None
    y_none, _ = oracle.wqmm(a)
    np.testing.assert_allclose(y_full - y_none, dec_bf16(b)[None, :] + dec_bf16(x3), rtol=0, atol=1e-12)


def test_transposed_storage_equals_nd_storage():
    for wdt in ["i8", "i4", "fp8"]:
        mode = "channel" if wdt == "fp8" else "group"
        nd = W.make_wqmm_case(x1_shape=(3, 128), n=64, act="bf16", wdt=wdt, mode=mode, group_size=64,
                              offset=(wdt != "fp8"), seed=17)
        tr = W.make_wqmm_case(x1_shape=(3, 128), n=64, act="bf16", wdt=wdt, mode=mode, group_size=64,
                              offset=(wdt != "fp8"), x2_transposed=True, scale_transposed=True, seed=17)
        assert np.array_equal(oracle.wqmm(nd)[0], oracle.wqmm(tr)[0]), wdt


def test_three_d_x1_equals_two_d():
    c3 = W.make_wqmm_case(x1_shape=(2, 3, 64), n=32, act="bf16", wdt="i8", mode="channel", seed=18)
    c2 = W.make_wqmm_case(x1_shape=(6, 64), n=32, act="bf16", wdt="i8", mode="channel", seed=18)
    c2.x1, c2.x3 = c3.x1.reshape(6, 64), c3.x3.reshape(6, 32)
    assert np.array_equal(oracle.wqmm(c3)[0], oracle.wqmm(c2)[0])


def test_empty_k_gives_bias_plus_x3():
    c = W.make_wqmm_case(x1_shape=(4, 0), n=8, act="bf16", wdt="i8", mode="channel", seed=19)
    ye, _ = oracle.wqmm(c)
    np.testing.assert_array_equal(ye, dec_bf16(c.bias)[None, :] + dec_bf16(c.x3))


def test_qmm_unit_scales_equal_numpy_int64_matmul():
    c = W.make_qmm_case(x1_shape=(9, 160), n=48, out="bf16", pertoken=False, x3=False, seed=20)
    c.dq_dtype = "f32"
    c.dequant_scale = np.ones(1, dtype=np.float32)
    acc, ye, _ = oracle.qmm(c)
    ref = c.x1.astype(np.int64) @ c.x2.astype(np.int64) + c.bias.astype(np.int64)
    assert np.array_equal(acc, ref) and np.array_equal(ye, ref.astype(np.float64))


def test_sampled_rows_cols_equal_full_evaluation():
    c = W.make_wqmm_case(x1_shape=(20, 128), n=48, act="bf16", wdt="i4", mode="group", group_size=64, seed=21)
    ye, yr = oracle.wqmm(c)
    rows, cols = [19, 0, 7], [47, 3, 3, 10]
    ye_s, yr_s = oracle.wqmm(c, rows=rows, cols=cols)
    assert np.array_equal(ye_s, ye[np.ix_(rows, cols)]) and np.array_equal(yr_s, yr[np.ix_(rows, cols)])
    q = W.make_qmm_case(x1_shape=(11, 64), n=40, seed=22)
    a, e, r = oracle.qmm(q)
    qrows, qcols = [10, 0, 4], [39, 3, 3, 10]
    a_s, e_s, r_s = oracle.qmm(q, rows=qrows, cols=qcols)
    assert np.array_equal(a_s, a[np.ix_(qrows, qcols)]) and np.array_equal(e_s, e[np.ix_(qrows, qcols)])
    with pytest.raises(ValueError):
        oracle.qmm(q, rows=[11])
    with pytest.raises(ValueError):
        oracle.wqmm(c, cols=[48])
