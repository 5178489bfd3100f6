"""Parity of the fused residual-add RMSNorm and gated RMSNorm ("norm_fusion.rs",
module doc comment: the elementwise fusions kept composed until a kernel pins
the summation order) with the fp64 oracle, through the C ABI; their bits
against the unfused RMSNorm call; layouts, aliasing, every row at full size. Outputs land
in guard-banded buffers whose surroundings must stay untouched."""
import numpy as np
import pytest
import torch

import oracle
import transformer_row_normalization_b200 as rn
from transformer_row_normalization_b200 import workloads as wl
from fullsize import each_chunk
from tolerance import check, guarded_empty, to_f64

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.bfloat16]
WIDTHS = [1, 3, 7, 8, 9, 33, 64, 100, 128, 129, 768, 1000, 1024, 1025, 2048, 4096, 4097,
          8192, 16384]


def host(t):
    return t.detach().cpu()


def run_add(x, r, w, eps, row_gap=0, h=None):
    """h (the stored sum) must share x's 16-byte phase: a guarded dense
    buffer for dense x, else the caller's view laid out like x."""
    y, _, gy = guarded_empty(tuple(x.shape), x.dtype, row_gap=row_gap)
    gh = None
    if h is None:
        h, _, gh = guarded_empty(tuple(x.shape), x.dtype)
    rn.add_rms_norm(x, r, w, eps, out=y, out_h=h)
    torch.cuda.synchronize()
    gy()
    if gh is not None:
        gh()
    return y, h


def run_gated(x, z, w, eps, row_gap=0):
    y, _, gy = guarded_empty(tuple(x.shape), x.dtype, row_gap=row_gap)
    rn.gated_rms_norm(x, z, w, eps, out=y)
    torch.cuda.synchronize()
    gy()
    return y


def rows2d(t):
    return host(t).reshape(-1, t.shape[-1]) if t.is_contiguous() else host(t)


def check_add(x, r, w, eps, y, h, what):
    ref_y, ref_h = oracle.add_rms_norm(rows2d(x), rows2d(r), None if w is None else host(w), eps)
    got_h = to_f64(h).reshape(ref_h.shape)
    assert np.array_equal(got_h, ref_h), f"{what}: stored sum differs from the oracle"
    check(y.reshape(ref_y.shape), ref_y, x.dtype, what=what)
    # the contract: y is RMSNorm of the stored sum, bit for bit
    assert torch.equal(y, rn.rms_norm(h, w, eps)), f"{what}: y != rms_norm(h)"


def check_gated(x, z, w, eps, y, what):
    ref = oracle.gated_rms_norm(rows2d(x), rows2d(z), None if w is None else host(w), eps)
    check(y.reshape(ref.shape), ref, x.dtype, what=what, scaled=True)


def test_small_f32_workloads():
    for name in ("add_rms_f32_4x128x1024", "gated_rms_f32_4x128x1024"):
        w_ = wl.WORKLOADS[name]
        a = {k: v.cuda() for k, v in wl.make_inputs(w_).items()}
        if w_.op == "add_rms":
            y, h = run_add(a["x"], a["r"], a["w"], w_.eps)
            check_add(a["x"], a["r"], a["w"], w_.eps, y, h, name)
        else:
            y = run_gated(a["x"], a["z"], a["w"], w_.eps)
            check_gated(a["x"], a["z"], a["w"], w_.eps, y, name)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("dim", WIDTHS)
def test_add_rms_widths(dtype, dim):
    x = wl.random_rows(37, dim, dtype, seed=6000 + dim).cuda()
    r = wl.random_rows(37, dim, dtype, seed=7000 + dim, std=2.0).cuda()
    w = wl.random_vector(dim, dtype, seed=8000 + dim).cuda()
    y, h = run_add(x, r, w, 1e-6)
    check_add(x, r, w, 1e-6, y, h, f"add_rms D={dim}")


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("dim", WIDTHS)
def test_gated_rms_widths(dtype, dim):
    x = wl.random_rows(37, dim, dtype, seed=9000 + dim).cuda()
    z = wl.random_rows(37, dim, dtype, seed=9500 + dim, std=3.0).cuda()
    w = wl.random_vector(dim, dtype, seed=9900 + dim).cuda()
    y = run_gated(x, z, w, 1e-6)
    check_gated(x, z, w, 1e-6, y, f"gated D={dim}")


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("dim,offset,gap", [(1000, 3, 0), (4097, 1, 2), (128, 5, 1),
                                            (33, 1, 0), (2048, 2, 3)])
def test_misaligned_views_and_gapped_outputs(dtype, dim, offset, gap):
    # x and the second input start `offset` elements into wider rows (same
    # 16-byte phase); y rows carry a gap, so they may sit at another phase
    bx = wl.random_rows(29, dim + offset + 4, dtype, seed=dim + 1).cuda()
    b2 = wl.random_rows(29, dim + offset + 4, dtype, seed=dim + 2, std=2.0).cuda()
    x, s2 = bx[:, offset:offset + dim], b2[:, offset:offset + dim]
    w = wl.random_vector(dim, dtype, seed=dim + 3).cuda()
    # h laid out like x (same offset in equally wide rows), inside a buffer
    # whose other columns must stay untouched
    hb = torch.full_like(bx, float("nan"))
    y, h = run_add(x, s2, w, 1e-6, row_gap=gap, h=hb[:, offset:offset + dim])
    check_add(x, s2, w, 1e-6, y, h, f"add_rms view D={dim}")
    assert torch.isnan(hb[:, :offset]).all() and torch.isnan(hb[:, offset + dim:]).all()
    y = run_gated(x, s2, w, 1e-6, row_gap=gap)
    check_gated(x, s2, w, 1e-6, y, f"gated view D={dim}")


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("dim", [7, 128, 4096, 4097])
def test_in_place_residual_stream(dtype, dim):
    x = wl.random_rows(33, dim, dtype, seed=41 + dim).cuda()
    r = wl.random_rows(33, dim, dtype, seed=42 + dim).cuda()
    w = wl.random_vector(dim, dtype, seed=43).cuda()
    ref_y, ref_h = oracle.add_rms_norm(host(x), host(r), host(w), 1e-6)
    # h written over the residual, then over x
    r1 = r.clone()
    y1, _ = rn.add_rms_norm(x, r1, w, 1e-6, out_h=r1)
    x2 = x.clone()
    y2, _ = rn.add_rms_norm(x2, r, w, 1e-6, out_h=x2)
    torch.cuda.synchronize()
    for yy, hh, what in ((y1, r1, "h over residual"), (y2, x2, "h over x")):
        assert np.array_equal(to_f64(hh), ref_h), what
        check(yy, ref_y, dtype, what=what)
    # y written over x
    x3 = x.clone()
    y3, h3 = rn.add_rms_norm(x3, r, w, 1e-6, out=x3)
    g = x.clone()
    y4 = rn.gated_rms_norm(g, r, w, 1e-6, out=g)
    torch.cuda.synchronize()
    check(y3, ref_y, dtype, what="y over x")
    check_gated(x, r, w, 1e-6, y4, "gated y over x")


def test_null_weight_and_zero_inputs():
    x = wl.random_rows(20, 1000, torch.bfloat16, seed=51).cuda()
    r = wl.random_rows(20, 1000, torch.bfloat16, seed=52).cuda()
    y, h = run_add(x, r, None, 1e-6)
    check_add(x, r, None, 1e-6, y, h, "add_rms w=None")
    y, h = run_add(x, torch.zeros_like(x), None, 1e-6)
    assert torch.equal(h, x) and torch.equal(y, rn.rms_norm(x, None, 1e-6))
    y = run_gated(x, torch.zeros_like(x), None, 1e-6)
    assert torch.all(y == 0), "silu(0) = 0"
    y = run_gated(x, r, None, 1e-6)
    check_gated(x, r, None, 1e-6, y, "gated w=None")


def test_phase_mismatch_is_an_error():
    b = wl.random_rows(8, 130, torch.bfloat16, seed=53).cuda()
    x, r = b[:, 0:128], b[:, 1:129]  # r rows one element off x's phase
    with pytest.raises(rn.RowNormError, match="RN_ERR_ALIGN"):
        rn.add_rms_norm(x, r, None, 1e-6)
    with pytest.raises(rn.RowNormError, match="RN_ERR_ALIGN"):
        rn.gated_rms_norm(x, r, None, 1e-6)


@pytest.mark.parametrize("name", [n for n in wl.FUSED_SUITE
                                  if wl.WORKLOADS[n].op in ("add_rms", "gated_rms")])
def test_full_size(name):
    """Every row at the benchmark's size: y against the oracle, and the stored
    residual sum h equal to the oracle's rounded sum exactly."""
    w_ = wl.WORKLOADS[name]
    a = wl.make_inputs(w_, device="cuda")
    x = a["x"].reshape(-1, w_.dim)
    if w_.op == "add_rms":
        r = a["r"].reshape(-1, w_.dim)
        y, h = rn.add_rms_norm(x, r, a["w"], w_.eps)
        torch.cuda.synchronize()
        assert torch.equal(y, rn.rms_norm(h, a["w"], w_.eps))
        hx, hr, hy, hh, hw = host(x), host(r), host(y), host(h), host(a["w"])

        def part(r0, r1):
            ref_y, ref_h = oracle.add_rms_norm(hx[r0:r1], hr[r0:r1], hw, w_.eps)
            assert np.array_equal(to_f64(hh[r0:r1]), ref_h), f"{name} rows {r0}:{r1}: h"
            check(hy[r0:r1], ref_y, w_.dtype, what=f"{name} rows {r0}:{r1}")
    else:
        z = a["z"].reshape(-1, w_.dim)
        y = rn.gated_rms_norm(x, z, a["w"], w_.eps)
        torch.cuda.synchronize()
        hx, hz, hy, hw = host(x), host(z), host(y), host(a["w"])

        def part(r0, r1):
            ref = oracle.gated_rms_norm(hx[r0:r1], hz[r0:r1], hw, w_.eps)
            check(hy[r0:r1], ref, w_.dtype, what=f"{name} rows {r0}:{r1}", scaled=True)

    assert each_chunk(w_.rows, w_.dim, part) == w_.rows


@pytest.mark.parametrize("dim", [128, 1000, 4096, 4097])
def test_bitwise_repeatable_across_grids(dim):
    x = wl.random_rows(3000 if dim <= 1024 else 700, dim, torch.bfloat16, seed=dim + 61).cuda()
    r = wl.random_rows(x.shape[0], dim, torch.bfloat16, seed=dim + 62).cuda()
    w = wl.random_vector(dim, torch.bfloat16, seed=63).cuda()
    base_add = rn.add_rms_norm(x, r, w, 1e-6)
    base_gated = rn.gated_rms_norm(x, r, w, 1e-6)
    try:
        for grid in (1, 7, 148, 592):
            rn.set_grid_override(grid)
            y, h = rn.add_rms_norm(x, r, w, 1e-6)
            assert torch.equal(y, base_add[0]) and torch.equal(h, base_add[1]), grid
            assert torch.equal(rn.gated_rms_norm(x, r, w, 1e-6), base_gated), grid
    finally:
        rn.set_grid_override(0)
