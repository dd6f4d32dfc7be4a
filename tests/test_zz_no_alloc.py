"""The no-allocation entry point, wqmm_matmul_no_alloc.

Some callers cannot allocate device memory -- code recorded into a CUDA graph,
components with a fixed memory budget, or foreign ABIs that pass tensors but no
allocator -- so they cannot provide the workspace wqmm_run needs.  For them the
library offers wqmm_matmul_no_alloc, which runs both phases with a fixed device
array of its own as the workspace.  These tests call it through the C ABI, twice
in a row (the array keeps the previous call's contents; a call on another problem runs
between them), and compare each result with the regular two-phase entry
point's and with the CPU oracle on the same inputs, within the tolerance the
parity tests use.  A problem too large for the array is refused
before anything is launched.

This file is named so that pytest collects it last.
"""
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
    yield


def _as_f64(t):
    return t.float().cpu().numpy().astype(np.float64).reshape(-1, t.shape[-1])


def _no_alloc(d, out):
    D = W.desc
    return W.wqmm_matmul_no_alloc(D(d.x1), d.x2_desc, None if d.bias is None else D(d.bias), d.scale_desc,
                                  d.offset_desc, None if d.x3 is None else D(d.x3), None, "sum", 0, 1, d.group_size,
                                  D(out))


def _workspace_bytes(d):
    st, ws, ex = W.wqmm_get_workspace_size(W.desc(d.x1), d.x2_desc, None if d.bias is None else W.desc(d.bias),
                                           d.scale_desc, d.offset_desc, None if d.x3 is None else W.desc(d.x3),
                                           None, "sum", 0, 1, d.group_size, W.desc(d.out))
    assert st == W.SUCCESS
    W.wqmm_executor_destroy(ex)
    return ws


def _other_call():
    # a different problem through the no-allocation entry point: it leaves its
    # own partials, flags and packed bytes in the shared array
    case = WL.make_wqmm_case(name="noalloc_other", x1_shape=(9, 1024), n=640, act="bf16", wdt="i8", mode="group",
                             group_size=32, seed=33)
    d = C.wqmm_to_device(case, pack=False)
    assert _no_alloc(d, d.out) == W.SUCCESS, W.wqmm_last_error()
    torch.cuda.synchronize()


def _check_twice(case, pack):
    d = C.wqmm_to_device(case, pack=pack)
    C.wqmm_call(d)  # the regular entry point, with a caller-provided workspace
    torch.cuda.synchronize()
    ref = _as_f64(d.out)
    ye, _ = oracle.wqmm(case)
    denom = max(np.abs(ref).max(), 1e-30)
    assert np.abs(ref - ye).max() / max(np.abs(ye).max(), 1e-30) <= TOL[case.act]
    for i in range(2):
        if i == 1:
            _other_call()
        out = torch.full_like(d.out, float("nan"))
        assert _no_alloc(d, out) == W.SUCCESS, W.wqmm_last_error()
        torch.cuda.synchronize()
        got = _as_f64(out)
        assert np.isfinite(got).all()
        assert np.abs(got - ref).max() / denom <= TOL[case.act]
        assert np.abs(got - ye).max() / max(np.abs(ye).max(), 1e-30) <= TOL[case.act]
    st, code = W.wqmm_device_error(reset=True)
    assert st == W.SUCCESS and code == 0
    return d


def test_no_alloc_small_m_stream_k_matches_regular_entry_point_and_oracle():
    # m = 16: the small-m schedule splits the k steps of its tiles over the SMs
    # and keeps fp32 partial tiles and "partial written" flags in the workspace
    case = WL.make_wqmm_case(name="noalloc_sk", x1_shape=(16, 2048), n=1024, act="bf16", wdt="i4", mode="group",
                             group_size=64, scale_range=(0.005, 0.05), offset_range=(-4, 4), seed=31)
    d = _check_twice(case, pack=True)
    # with the weight pre-packed and the scale contiguous, a non-zero workspace
    # holds nothing but split-tile partials and flags
    assert _workspace_bytes(d) > 0


def test_no_alloc_unpacked_weight_matches_regular_entry_point_and_oracle():
    # an unpacked (ND) weight is re-laid into the workspace before the GEMM
    case = WL.make_wqmm_case(name="noalloc_nd", x1_shape=(40, 512), n=384, act="f16", wdt="i8", mode="channel",
                             seed=32)
    _check_twice(case, pack=False)


def test_no_alloc_rejects_problems_larger_than_its_array():
    # an unpacked 4096 x 8192 int8 weight needs a 32 MiB packed copy: refused, nothing launched
    k, n = 4096, 8192
    x1 = torch.zeros((16, k), dtype=torch.bfloat16, device="cuda")
    x2 = torch.zeros((k, n), dtype=torch.int8, device="cuda")
    scale = torch.ones((n,), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((16, n), dtype=torch.bfloat16, device="cuda")
    st = W.wqmm_matmul_no_alloc(W.desc(x1), W.desc(x2), None, W.desc(scale), None, None, None, "sum", 0, 1, 0,
                                W.desc(out))
    assert st == W.ERR_WORKSPACE and "16 MiB" in W.wqmm_last_error()
