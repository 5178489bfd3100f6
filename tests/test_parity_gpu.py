"""Parity of the CUDA path with the fp64 oracle, element by element, through
the C ABI (via the Python binding). Inputs are seeded; the oracle receives
the exact bytes the GPU read. Every output lands in a guarded buffer whose
surroundings must stay untouched (out-of-bounds write detection)."""
import numpy as np
import pytest
import torch

import oracle
import transformer_row_normalization_b200 as rn
from transformer_row_normalization_b200 import workloads as wl
from tolerance import check, guarded_empty, to_f64

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.bfloat16]


def host(t):
    return t.detach().cpu()


def run_rms(x, w, eps, **kw):
    y, _, guard = guarded_empty(tuple(x.shape), x.dtype, **kw)
    rn.rms_norm(x, w, eps, out=y)
    torch.cuda.synchronize()
    guard()
    return y


def run_ln(x, w, b, eps, **kw):
    y, _, guard = guarded_empty(tuple(x.shape), x.dtype, **kw)
    rn.layer_norm(x, w, b, eps, out=y)
    torch.cuda.synchronize()
    guard()
    return y


def oracle_rms(x, w, eps):
    return oracle.rms_norm(host(x).reshape(-1, x.shape[-1]) if x.is_contiguous() else host(x),
                           None if w is None else host(w), eps)


def oracle_ln(x, w, b, eps):
    return oracle.layer_norm(host(x).reshape(-1, x.shape[-1]) if x.is_contiguous() else host(x),
                             None if w is None else host(w), None if b is None else host(b), eps)


# ---------------------------------------------------------------------------
# the workloads small enough to compare in full


def test_rms_f32_4x128x1024():
    w_ = wl.WORKLOADS["rms_f32_4x128x1024"]
    a = {k: v.cuda() for k, v in wl.make_inputs(w_).items()}
    y = run_rms(a["x"], a["w"], w_.eps)
    check(y.reshape(-1, w_.dim), oracle_rms(a["x"], a["w"], w_.eps), w_.dtype, what="c1")


def test_rms_page_iota_case_within_page_bound():
    # "Fused transformer kernels on Emily", Part 1, Correctness: iota / 100,
    # weight 1, eps 1e-6; the page expects |composed - fused| of about 1e-5.
    x = (torch.arange(4 * 128 * 1024, dtype=torch.float32) / 100.0).reshape(4, 128, 1024).cuda()
    w = torch.ones(1024, device="cuda")
    y = run_rms(x, w, 1e-6)
    worst, _ = check(y.reshape(-1, 1024), oracle_rms(x, w, 1e-6), torch.float32, what="iota")
    assert worst <= 1e-5


def test_ln_f32_1x1024x768():
    w_ = wl.WORKLOADS["ln_f32_1x1024x768"]
    a = {k: v.cuda() for k, v in wl.make_inputs(w_).items()}
    y = run_ln(a["x"], a["w"], a["b"], w_.eps)
    check(y.reshape(-1, w_.dim), oracle_ln(a["x"], a["w"], a["b"], w_.eps), w_.dtype,
          bias=a["b"], what="c2")


def test_dual_decode():
    w_ = wl.WORKLOADS["dual_bf16_decode"]
    a = {k: v.cuda() for k, v in wl.make_inputs(w_).items()}
    yq, _, gq = guarded_empty(tuple(a["q"].shape), w_.dtype)
    yk, _, gk = guarded_empty(tuple(a["k"].shape), w_.dtype)
    rn.dual_head_rms_norm(a["q"], a["k"], a["wq"], a["wk"], w_.eps, out_q=yq, out_k=yk)
    torch.cuda.synchronize()
    gq(), gk()
    rq, rk = oracle.dual_head_rms_norm(host(a["q"]).reshape(-1, 128), host(a["k"]).reshape(-1, 128),
                                       host(a["wq"]), host(a["wk"]), w_.eps)
    check(yq.reshape(-1, 128), rq, w_.dtype, what="decode q")
    check(yk.reshape(-1, 128), rk, w_.dtype, what="decode k")


# ---------------------------------------------------------------------------
# widths: tiny, ragged, around every family / chunk boundary, the maximum

WIDTHS = [1, 2, 3, 7, 8, 9, 31, 33, 64, 100, 127, 128, 129, 255, 256, 257, 768, 1000,
          1023, 1024, 1025, 1536, 2047, 2048, 2049, 4095, 4096, 4097, 8191, 8192, 16383, 16384]


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("dim", WIDTHS)
def test_widths_rms(dtype, dim):
    rows = 37
    x = wl.random_rows(rows, dim, dtype, seed=1000 + dim).cuda()
    w = wl.random_vector(dim, dtype, seed=2000 + dim).cuda()
    y = run_rms(x, w, 1e-6)
    check(y, oracle_rms(x, w, 1e-6), dtype, what=f"rms D={dim}")


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("dim", WIDTHS)
def test_widths_ln(dtype, dim):
    rows = 37
    x = wl.random_rows(rows, dim, dtype, seed=3000 + dim, mean=0.5, std=2.0).cuda()
    x[5] = x[5, :1]  # a constant row
    w = wl.random_vector(dim, dtype, seed=4000 + dim).cuda()
    b = wl.random_vector(dim, dtype, seed=5000 + dim, mean=0.0, std=0.1).cuda()
    y = run_ln(x, w, b, 1e-5)
    check(y, oracle_ln(x, w, b, 1e-5), dtype, bias=b, what=f"ln D={dim}")
    assert torch.equal(y[5], b), "a constant row must return exactly the bias"


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
def test_widest_rows(dtype):
    dim = 32768 if dtype == torch.bfloat16 else 16384
    x = wl.random_rows(9, dim, dtype, seed=7).cuda()
    w = wl.random_vector(dim, dtype, seed=8).cuda()
    b = wl.random_vector(dim, dtype, seed=9, mean=0.0, std=0.1).cuda()
    check(run_rms(x, w, 1e-6), oracle_rms(x, w, 1e-6), dtype, what="widest rms")
    check(run_ln(x, w, b, 1e-5), oracle_ln(x, w, b, 1e-5), dtype, bias=b, what="widest ln")


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("dim", [5, 128, 1000, 4097])
def test_null_weight_and_bias(dtype, dim):
    x = wl.random_rows(20, dim, dtype, seed=11).cuda()
    check(run_rms(x, None, 1e-6), oracle_rms(x, None, 1e-6), dtype, what="rms w=None")
    check(run_ln(x, None, None, 1e-5), oracle_ln(x, None, None, 1e-5), dtype,
          bias=torch.zeros(dim, dtype=dtype), what="ln w,b=None")
    b = wl.random_vector(dim, dtype, seed=12, mean=0.0, std=0.1).cuda()
    check(run_ln(x, None, b, 1e-5), oracle_ln(x, None, b, 1e-5), dtype, bias=b, what="ln w=None")


# ---------------------------------------------------------------------------
# layouts: strided and misaligned views, gaps between output rows, in place


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("dim,offset,pad", [(128, 1, 5), (1000, 3, 1), (4097, 0, 0),
                                            (4097, 1, 2), (768, 7, 9), (2048, 2, 3),
                                            (16384, 5, 1), (33, 1, 0)])
def test_misaligned_input_views(dtype, dim, offset, pad):
    rows = 29
    big = wl.random_rows(rows, offset + dim + pad, dtype, seed=dim + offset).cuda()
    x = big[:, offset:offset + dim]
    w = wl.random_vector(dim, dtype, seed=13).cuda()
    b = wl.random_vector(dim, dtype, seed=14, mean=0.0, std=0.1).cuda()
    xr = host(x).contiguous()
    check(run_rms(x, w, 1e-6), oracle.rms_norm(xr, host(w), 1e-6), dtype, what="rms view")
    check(run_ln(x, w, b, 1e-5), oracle.layer_norm(xr, host(w), host(b), 1e-5), dtype,
          bias=b, what="ln view")
    # output rows with gaps (and so a different 16-byte phase from x)
    check(run_rms(x, w, 1e-6, row_gap=3), oracle.rms_norm(xr, host(w), 1e-6), dtype,
          what="rms gapped out")


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("dim", [7, 128, 1000, 4097])
def test_misaligned_weight_and_bias(dtype, dim):
    x = wl.random_rows(16, dim, dtype, seed=21).cuda()
    wbuf = wl.random_vector(dim + 3, dtype, seed=22).cuda()
    bbuf = wl.random_vector(dim + 5, dtype, seed=23, mean=0.0, std=0.1).cuda()
    w, b = wbuf[1:1 + dim], bbuf[3:3 + dim]
    check(run_rms(x, w, 1e-6), oracle_rms(x, w, 1e-6), dtype, what="rms w view")
    check(run_ln(x, w, b, 1e-5), oracle_ln(x, w, b, 1e-5), dtype, bias=b, what="ln w,b views")


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("dim", [3, 128, 1024, 4097, 8192])
def test_in_place(dtype, dim):
    x = wl.random_rows(33, dim, dtype, seed=31).cuda()
    w = wl.random_vector(dim, dtype, seed=32).cuda()
    b = wl.random_vector(dim, dtype, seed=33, mean=0.0, std=0.1).cuda()
    ref_r = oracle_rms(x, w, 1e-6)
    ref_l = oracle_ln(x, w, b, 1e-5)
    x1 = x.clone()
    rn.rms_norm(x1, w, 1e-6, out=x1)
    x2 = x.clone()
    rn.layer_norm(x2, w, b, 1e-5, out=x2)
    torch.cuda.synchronize()
    check(x1, ref_r, dtype, what="rms in place")
    check(x2, ref_l, dtype, bias=b, what="ln in place")


def test_rows_zero_and_one():
    x = torch.empty(0, 64, device="cuda", dtype=torch.bfloat16)
    assert rn.rms_norm(x, None, 1e-6).shape == (0, 64)
    x = wl.random_rows(1, 4097, torch.bfloat16, seed=41).cuda()
    check(run_ln(x, None, None, 1e-5), oracle_ln(x, None, None, 1e-5), torch.bfloat16,
          bias=torch.zeros(4097), what="one row")


# ---------------------------------------------------------------------------
# properties of the definition, on the GPU


def test_eps_zero_scale_invariance():
    x = wl.random_rows(64, 1024, torch.float32, seed=51).cuda()
    w = wl.random_vector(1024, torch.float32, seed=52).cuda()
    y1 = rn.rms_norm(x, w, 0.0)
    y4 = rn.rms_norm(x * 4.0, w, 0.0)
    torch.cuda.synchronize()
    assert (y1 - y4).abs().max().item() <= 1e-5
    check(y1, oracle_rms(x, w, 0.0), torch.float32, what="eps 0")


def test_unit_rms_and_standardized_outputs():
    x = wl.random_rows(256, 4096, torch.float32, seed=53, mean=0.5, std=2.0).cuda()
    y = rn.rms_norm(x, None, 0.0)
    torch.cuda.synchronize()
    ms = (y.double() ** 2).mean(dim=1)
    assert torch.allclose(ms, torch.ones_like(ms), atol=1e-5)
    z = rn.layer_norm(x, None, None, 0.0)
    torch.cuda.synchronize()
    assert z.double().mean(dim=1).abs().max().item() < 1e-5
    assert torch.allclose(z.double().var(dim=1, unbiased=False), torch.ones(256, dtype=torch.float64,
                                                                             device="cuda"), atol=1e-5)


def test_errors_surface_as_exceptions():
    x = torch.zeros(4, 8, device="cuda")
    with pytest.raises(rn.RowNormError, match="RN_ERR_EPS"):
        rn.rms_norm(x, None, -1.0)
    with pytest.raises(rn.RowNormError, match="RN_ERR_OVERLAP"):
        rn.rms_norm(x[:, :4], None, 1e-6, out=x[:, 2:6])
    big = torch.zeros(1, 32769, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(rn.RowNormError, match="RN_ERR_UNSUPPORTED"):
        rn.add_rms_norm(big, big.clone(), None, 1e-6)  # fused ops: registers only
    with pytest.raises(rn.RowNormError, match="RN_ERR_UNSUPPORTED"):
        huge = torch.zeros(1, (1 << 22) + 1, device="cuda", dtype=torch.bfloat16)
        rn.rms_norm(huge, None, 1e-6)  # beyond the streaming limit
