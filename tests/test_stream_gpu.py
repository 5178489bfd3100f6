"""Rows wider than the register kernels hold (bf16 > 32768, f32 > 16384
columns) stream through a block per row ("Emily.Fast", rms_norm/3 and
layer_norm/4, whose statistic the page calls "Welford-style": two passes over
the row here, read again from L2). Parity with the fp64 oracle, constant rows,
layouts, in place, and bits independent of the grid."""
import numpy as np
import pytest
import torch

import oracle
import transformer_row_normalization_b200 as rn
from transformer_row_normalization_b200 import workloads as wl
from fullsize import each_chunk
from tolerance import check, guarded_empty

pytestmark = pytest.mark.gpu

CASES = [(torch.bfloat16, 32769), (torch.bfloat16, 40000), (torch.bfloat16, 65536),
         (torch.bfloat16, 100003), (torch.bfloat16, 262144), (torch.float32, 16385),
         (torch.float32, 32768), (torch.float32, 65537)]


def host(t):
    return t.detach().cpu()


@pytest.mark.parametrize("dtype,dim", CASES)
def test_wide_rows(dtype, dim):
    rows = 6
    x = wl.random_rows(rows, dim, dtype, seed=dim, mean=0.5, std=2.0).cuda()
    x[2] = x[2, :1]  # a constant row
    w = wl.random_vector(dim, dtype, seed=dim + 1).cuda()
    b = wl.random_vector(dim, dtype, seed=dim + 2, mean=0.0, std=0.1).cuda()
    assert rn.plan(rn.RN_OP_LN, x, weight=w, bias=b)["family"] == 2
    y, _, guard = guarded_empty((rows, dim), dtype)
    rn.rms_norm(x, w, 1e-6, out=y)
    torch.cuda.synchronize()
    guard()
    check(y, oracle.rms_norm(host(x), host(w), 1e-6), dtype, what=f"rms D={dim}")
    y, _, guard = guarded_empty((rows, dim), dtype)
    rn.layer_norm(x, w, b, 1e-5, out=y)
    torch.cuda.synchronize()
    guard()
    check(y, oracle.layer_norm(host(x), host(w), host(b), 1e-5), dtype, bias=b,
          what=f"ln D={dim}")
    assert torch.equal(y[2], b), "a constant row must return exactly the bias"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_wide_layouts(dtype):
    dim = 50001 if dtype == torch.bfloat16 else 20001
    big = wl.random_rows(5, dim + 7, dtype, seed=3).cuda()
    x = big[:, 3:3 + dim]                                   # rows off the 16-byte grid
    wbuf = wl.random_vector(dim + 2, dtype, seed=4).cuda()
    bbuf = wl.random_vector(dim + 3, dtype, seed=5, mean=0.0, std=0.1).cuda()
    w, b = wbuf[1:1 + dim], bbuf[2:2 + dim]                  # vectors off the grid too
    xr = host(x).contiguous()
    check(rn.rms_norm(x, w, 1e-6), oracle.rms_norm(xr, host(w), 1e-6), dtype, what="rms view")
    check(rn.layer_norm(x, w, b, 1e-5), oracle.layer_norm(xr, host(w), host(b), 1e-5), dtype,
          bias=b, what="ln view")
    y, _, guard = guarded_empty((5, dim), dtype, row_gap=5)  # y at other phases
    rn.layer_norm(x, None, None, 1e-5, out=y)
    torch.cuda.synchronize()
    guard()
    check(y, oracle.layer_norm(xr, None, None, 1e-5), dtype, bias=torch.zeros(dim),
          what="ln gapped out, null vectors")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_wide_shifted_vectors(dtype):
    """Rows off the 16-byte grid at every phase. With weight and bias at one
    common offset from the grid, their chunk columns come from two aligned
    words shifted into place. Those must give exactly the bits of
    element-by-element loads, taken when weight and bias sit at different
    offsets, and parity with the oracle."""
    dim = 40001 if dtype == torch.bfloat16 else 20001
    rows = 17  # every 16-byte phase of an odd width, twice
    x = wl.random_rows(rows, dim, dtype, seed=21, mean=0.5, std=2.0).cuda()
    wv = wl.random_vector(dim, dtype, seed=22).cuda()
    bv = wl.random_vector(dim, dtype, seed=23, mean=0.0, std=0.1).cuda()
    for off in (0, 1, 3):
        # common offset `off`: shifted loads (or, at 0, aligned ones)
        wbuf = torch.zeros(dim + 8, dtype=dtype, device="cuda")
        bbuf = torch.zeros(dim + 8, dtype=dtype, device="cuda")
        wbuf[off:off + dim] = wv
        bbuf[off:off + dim] = bv
        shifted = (rn.layer_norm(x, wbuf[off:off + dim], bbuf[off:off + dim], 1e-5),
                   rn.rms_norm(x, wbuf[off:off + dim], 1e-6))
        # bias one element further: weight and bias at different offsets
        b2 = torch.zeros(dim + 8, dtype=dtype, device="cuda")
        b2[off + 1:off + 1 + dim] = bv
        elementwise = rn.layer_norm(x, wbuf[off:off + dim], b2[off + 1:off + 1 + dim], 1e-5)
        torch.cuda.synchronize()
        assert torch.equal(shifted[0], elementwise), off
        check(shifted[0], oracle.layer_norm(host(x), host(wv), host(bv), 1e-5), dtype, bias=bv,
              what=f"ln offset {off}")
        check(shifted[1], oracle.rms_norm(host(x), host(wv), 1e-6), dtype, what=f"rms offset {off}")


@pytest.mark.parametrize("op,dtype,dim,threads", [
    ("ln", torch.bfloat16, 65536, 512), ("ln", torch.bfloat16, 98304, 512),
    ("ln", torch.bfloat16, 98305, 1024), ("ln", torch.bfloat16, 262144, 1024),
    ("ln", torch.float32, 49152, 512), ("ln", torch.float32, 49153, 1024),
    ("rms", torch.bfloat16, 65536, 1024), ("rms", torch.float32, 32768, 1024)])
def test_stream_block_size(op, dtype, dim, threads):
    """LayerNorm rows of at most 192 KB stream in blocks of 512 threads
    (several rows per SM); wider rows and RMSNorm in blocks of 1024 (one row
    per SM)."""
    x = torch.empty(2, dim, dtype=dtype, device="cuda")
    w = torch.empty(dim, dtype=dtype, device="cuda")
    kind = rn.RN_OP_LN if op == "ln" else rn.RN_OP_RMS
    p = rn.plan(kind, x, weight=w, bias=w if op == "ln" else None)
    assert p["family"] == 2 and p["threads_per_row"] == threads and p["block_threads"] == threads


def test_wide_in_place_and_grids():
    dim = 70000
    x = wl.random_rows(300, dim, torch.bfloat16, seed=9).cuda()
    w = wl.random_vector(dim, torch.bfloat16, seed=10).cuda()
    b = wl.random_vector(dim, torch.bfloat16, seed=11, mean=0.0, std=0.1).cuda()
    base = rn.layer_norm(x, w, b, 1e-5)
    try:
        for grid in (1, 7, 148, 300):
            rn.set_grid_override(grid)
            assert torch.equal(rn.layer_norm(x, w, b, 1e-5), base), grid
    finally:
        rn.set_grid_override(0)
    x2 = x.clone()
    rn.layer_norm(x2, w, b, 1e-5, out=x2)
    torch.cuda.synchronize()
    assert torch.equal(x2, base)
    idx = torch.tensor([0, 1, 150, 299])
    check(base[idx.cuda()], oracle.layer_norm(host(x)[idx], host(w), host(b), 1e-5),
          torch.bfloat16, bias=b, what="sampled rows")


@pytest.mark.parametrize("name", [n for n in wl.FUSED_SUITE if wl.WORKLOADS[n].op in ("rms", "ln")])
def test_full_size_streaming(name):
    """Every row of the streamed benchmark workloads against the oracle."""
    w_ = wl.WORKLOADS[name]
    a = wl.make_inputs(w_, device="cuda")
    x = a["x"].reshape(-1, w_.dim)
    if w_.op == "ln":
        y = rn.layer_norm(x, a["w"], a["b"], w_.eps)
    else:
        y = rn.rms_norm(x, a["w"], w_.eps)
    torch.cuda.synchronize()
    hx, hy, hw = host(x), host(y), host(a["w"])
    hb = host(a["b"]) if w_.op == "ln" else None
    del x, y, a
    torch.cuda.empty_cache()

    def part(r0, r1):
        if w_.op == "ln":
            check(hy[r0:r1], oracle.layer_norm(hx[r0:r1], hw, hb, w_.eps), w_.dtype, bias=hb,
                  what=f"{name} rows {r0}:{r1}")
        else:
            check(hy[r0:r1], oracle.rms_norm(hx[r0:r1], hw, w_.eps), w_.dtype,
                  what=f"{name} rows {r0}:{r1}")

    assert each_chunk(w_.rows, w_.dim, part) == w_.rows
