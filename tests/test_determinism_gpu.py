"""Bitwise determinism: repeated runs, every grid size, and the dual-output
q/k head norm against two single RMSNorm calls ("norm_fusion.rs": the fused
replay must reproduce the bits of the separate kernels over their inputs)."""
import pytest
import torch

import transformer_row_normalization_b200 as rn
from transformer_row_normalization_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CASES = [(torch.bfloat16, 128), (torch.bfloat16, 1000), (torch.bfloat16, 4097),
         (torch.bfloat16, 8192), (torch.float32, 768), (torch.float32, 2048)]


@pytest.fixture(autouse=True)
def reset_grid():
    yield
    rn.set_grid_override(0)


@pytest.mark.parametrize("dtype,dim", CASES)
def test_repeat_and_grid_independence(dtype, dim):
    x = wl.random_rows(601, dim, dtype, seed=dim, mean=0.5, std=2.0).cuda()
    w = wl.random_vector(dim, dtype, seed=1).cuda()
    b = wl.random_vector(dim, dtype, seed=2, mean=0.0, std=0.1).cuda()
    ref_r = rn.rms_norm(x, w, 1e-6)
    ref_l = rn.layer_norm(x, w, b, 1e-5)
    for _ in range(3):
        assert torch.equal(rn.rms_norm(x, w, 1e-6), ref_r)
        assert torch.equal(rn.layer_norm(x, w, b, 1e-5), ref_l)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for grid in (1, 7, sms, 4 * sms):
        rn.set_grid_override(grid)
        assert torch.equal(rn.rms_norm(x, w, 1e-6), ref_r), f"grid {grid}"
        assert torch.equal(rn.layer_norm(x, w, b, 1e-5), ref_l), f"grid {grid}"


@pytest.mark.parametrize("tokens", [1, 3, 8192])
def test_dual_equals_two_single_calls(tokens):
    q = wl.random_rows(tokens * 32, 128, torch.bfloat16, seed=tokens).cuda()
    k = wl.random_rows(tokens * 8, 128, torch.bfloat16, seed=tokens + 1).cuda()
    wq = wl.random_vector(128, torch.bfloat16, seed=3).cuda()
    wk = wl.random_vector(128, torch.bfloat16, seed=4).cuda()
    yq, yk = rn.dual_head_rms_norm(q, k, wq, wk, 1e-6)
    assert torch.equal(yq, rn.rms_norm(q, wq, 1e-6))
    assert torch.equal(yk, rn.rms_norm(k, wk, 1e-6))


@pytest.mark.parametrize("dq,dk", [(128, 64), (64, 256), (1000, 7), (1024, 1024)])
def test_dual_with_unequal_head_dims(dq, dk):
    q = wl.random_rows(77, dq, torch.bfloat16, seed=5).cuda()
    k = wl.random_rows(23, dk, torch.bfloat16, seed=6).cuda()
    wq = wl.random_vector(dq, torch.bfloat16, seed=7).cuda()
    wk = wl.random_vector(dk, torch.bfloat16, seed=8).cuda()
    yq, yk = rn.dual_head_rms_norm(q, k, wq, wk, 1e-6)
    assert torch.equal(yq, rn.rms_norm(q, wq, 1e-6))
    assert torch.equal(yk, rn.rms_norm(k, wk, 1e-6))


def test_dual_is_one_launch_plan():
    q = torch.zeros(8192 * 32, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(8192 * 8, 128, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(128, dtype=torch.bfloat16, device="cuda")
    p = rn.plan(rn.RN_OP_DUAL, q, weight=w, bias=w, k=k)
    assert p["family"] == 0 and p["grid_blocks"] >= 1


PATH_CASES = [
    # (dtype, rows, dim, offset) -- offset > 0 makes rows start off the 16-byte grid
    (torch.bfloat16, 3000, 128, 0), (torch.bfloat16, 2000, 768, 0), (torch.bfloat16, 2000, 1000, 0),
    (torch.float32, 1500, 1024, 0), (torch.bfloat16, 700, 4096, 0), (torch.bfloat16, 700, 4097, 0),
    (torch.bfloat16, 600, 8192, 0), (torch.bfloat16, 300, 16384, 0), (torch.bfloat16, 100, 32768, 0),
    (torch.float32, 500, 4099, 0), (torch.float32, 200, 16384, 0), (torch.bfloat16, 900, 2048, 3),
    (torch.bfloat16, 1100, 1536, 0), (torch.bfloat16, 801, 2048, 0), (torch.bfloat16, 700, 2056, 0),
    (torch.bfloat16, 1200, 64, 0), (torch.float32, 900, 1536, 1),
]


def ring_applies(dtype, dim, offset):
    """Under rn_set_path_override(2) the rings carry every RMSNorm and
    LayerNorm row the register kernels hold, except lane-group rows (dim <=
    2048 bf16, 1024 binary32: a warp of 32 lanes of at most 8 chunks) off
    the 16-byte grid: per-warp rings take lane-group rows whose rows all
    start on the grid with whole 16-byte chunks, block rings every wider
    row."""
    v = 8 if dtype == torch.bfloat16 else 4
    widest = 32768 if dtype == torch.bfloat16 else 16384
    lane_widest = 2048 if dtype == torch.bfloat16 else 1024
    if dim > lane_widest:
        return dim <= widest
    return dim % v == 0 and offset == 0


@pytest.mark.parametrize("dtype,rows,dim,offset", PATH_CASES)
def test_register_and_ring_kernels_agree_bitwise(dtype, rows, dim, offset):
    big = wl.random_rows(rows, dim + offset, dtype, seed=dim, mean=0.5, std=2.0).cuda()
    x = big[:, offset:offset + dim] if offset else big
    w = wl.random_vector(dim, dtype, seed=1).cuda()
    b = wl.random_vector(dim, dtype, seed=2, mean=0.0, std=0.1).cuda()
    out = {}
    try:
        for path in (1, 2, 3):
            rn.set_path_override(path)
            out[path] = (rn.rms_norm(x, w, 1e-6), rn.layer_norm(x, w, b, 1e-5),
                         rn.plan(rn.RN_OP_LN, x, weight=w, bias=b)["staged"])
    finally:
        rn.set_path_override(0)
    assert out[1][2] == 0 and out[3][2] == 0
    assert out[2][2] == int(ring_applies(dtype, dim, offset))
    for path in (2, 3):
        assert torch.equal(out[1][0], out[path][0]), path
        assert torch.equal(out[1][1], out[path][1]), path
    assert rn.device_error_count(reset=True) == 0


def test_ring_dual_agrees_with_register_dual():
    q = wl.random_rows(8192 * 4, 128, torch.bfloat16, seed=9).cuda()
    k = wl.random_rows(8192, 128, torch.bfloat16, seed=10).cuda()
    wq = wl.random_vector(128, torch.bfloat16, seed=11).cuda()
    wk = wl.random_vector(128, torch.bfloat16, seed=12).cuda()
    res = {}
    try:
        for path in (1, 2):
            rn.set_path_override(path)
            assert rn.plan(rn.RN_OP_DUAL, q, weight=wq, bias=wk, k=k)["staged"] == path - 1
            res[path] = rn.dual_head_rms_norm(q, k, wq, wk, 1e-6)
    finally:
        rn.set_path_override(0)
    assert torch.equal(res[1][0], res[2][0]) and torch.equal(res[1][1], res[2][1])
    assert rn.device_error_count(reset=True) == 0


@pytest.mark.parametrize("rows", [1, 2, 3, 31, 33, 597, 4096 + 3])
@pytest.mark.parametrize("dtype,dim", [(torch.bfloat16, 768), (torch.bfloat16, 1000),
                                       (torch.bfloat16, 128), (torch.bfloat16, 1536),
                                       (torch.bfloat16, 2048), (torch.float32, 1024),
                                       (torch.float32, 300)])
def test_ring_ragged_row_counts(rows, dtype, dim):
    """Row counts that leave partial tiles, warps without tiles and a ragged
    last round of lane groups give the register kernels' bits."""
    x = wl.random_rows(rows, dim, dtype, seed=rows + dim, mean=0.5, std=2.0).cuda()
    w = wl.random_vector(dim, dtype, seed=3).cuda()
    b = wl.random_vector(dim, dtype, seed=4, mean=0.0, std=0.1).cuda()
    res = {}
    try:
        for path in (1, 2):
            rn.set_path_override(path)
            res[path] = (rn.layer_norm(x, w, b, 1e-5), rn.rms_norm(x, None, 1e-6))
    finally:
        rn.set_path_override(0)
    assert torch.equal(res[1][0], res[2][0]) and torch.equal(res[1][1], res[2][1])
    assert rn.device_error_count(reset=True) == 0


def test_ring_strided_and_block_views():
    """Rows a stride apart (one copy per row) and head rows of a packed buffer
    through the rings, against the register kernels."""
    buf = wl.random_rows(3000, 1024 + 256, torch.bfloat16, seed=77, mean=0.5, std=2.0).cuda()
    x = buf[:, 256:256 + 768]                       # stride 1280, rows 16-byte aligned
    heads = buf.view(3000, 10, 128)[:, 2:8, :]      # 6 head rows per token, in blocks
    w = wl.random_vector(768, torch.bfloat16, seed=5).cuda()
    wh = wl.random_vector(128, torch.bfloat16, seed=6).cuda()
    res = {}
    try:
        for path in (1, 2):
            rn.set_path_override(path)
            assert rn.plan(rn.RN_OP_RMS, x, weight=w)["staged"] == path - 1
            res[path] = (rn.rms_norm(x, w, 1e-6), rn.rms_norm(heads, wh, 1e-6),
                         rn.layer_norm(x, w, None, 1e-5))
    finally:
        rn.set_path_override(0)
    for a, b in zip(res[1], res[2]):
        assert torch.equal(a, b)
    assert rn.device_error_count(reset=True) == 0


@pytest.mark.parametrize("dim", [768, 4097])
def test_ring_waits_run_out_and_the_context_survives(dim):
    """Under the wait test no ring stage completes: every warp (D = 768, warp
    rings) or block (D = 4097, block rings) gives up its first wait, waits
    for its copies, counts one timeout and stops without writing. The next
    normal launch gives the register kernels' bits, with no timeout."""
    rows = 4096
    x = wl.random_rows(rows, dim, torch.bfloat16, seed=dim, mean=0.5, std=2.0).cuda()
    w = wl.random_vector(dim, torch.bfloat16, seed=1).cuda()
    b = wl.random_vector(dim, torch.bfloat16, seed=2, mean=0.0, std=0.1).cuda()
    try:
        rn.set_path_override(1)
        ref = rn.layer_norm(x, w, b, 1e-5)
        rn.set_path_override(2)
        p = rn.plan(rn.RN_OP_LN, x, weight=w, bias=b)
        assert p["staged"] == 1, p
        rn.device_error_count(reset=True)
        rn.set_ring_wait_test(True)
        y = torch.full_like(x, float("nan"))
        rn.layer_norm(x, w, b, 1e-5, out=y)
        torch.cuda.synchronize()
        rn.set_ring_wait_test(False)
        if p["family"] == 0:  # a warp ring per warp, tiles of stage_bytes
            tiles = -(-rows // (p["stage_bytes"] // (2 * dim)))
            expect = min(p["grid_blocks"] * p["block_threads"] // 32, tiles)
        else:                 # a block ring per block, one row per stage
            expect = min(p["grid_blocks"], rows)
        assert rn.device_error_count(reset=True) == expect
        assert bool(torch.isnan(y).all())  # no stage completed, nothing written
        y2 = rn.layer_norm(x, w, b, 1e-5)
        torch.cuda.synchronize()
        assert torch.equal(y2, ref)
        assert rn.device_error_count(reset=True) == 0
    finally:
        rn.set_ring_wait_test(False)
        rn.set_path_override(0)


def test_ring_plans_for_the_large_workloads():
    """By default warp rings carry aligned bf16 lane-group rows that fill a
    warp (the narrow LayerNorm widths, two rows to a tile); block
    rings carry LayerNorm blocks of 512+ threads (D = 16384); the rest keep the
    register kernels unless the rings are forced."""
    for dim, ring in ((768, 1), (1000, 1), (4096, 0), (8192, 0), (16384, 1), (4097, 0)):
        x = torch.empty(65536, dim, dtype=torch.bfloat16, device="cuda")
        p = rn.plan(rn.RN_OP_LN, x)
        assert p["staged"] == ring, (dim, p)
        if ring:
            assert p["stages"] >= 2 and p["stage_bytes"] >= 2 * dim, p
        if dim in (768, 1000):  # whole-warp LayerNorm rows: two to a tile, 3 stages
            assert p["stage_bytes"] == 2 * 2 * dim and p["stages"] == 3, p
    q = torch.empty(8192 * 32, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(8192 * 8, 128, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(128, dtype=torch.bfloat16, device="cuda")
    # the plain dual head norm (4 lanes per row) stays on the register kernels
    assert rn.plan(rn.RN_OP_DUAL, q, weight=w, bias=w, k=k)["staged"] == 0
    # wide RMSNorm rows stay on the register kernels with their prefetch
    assert rn.plan(rn.RN_OP_RMS, torch.empty(1024, 16384, dtype=torch.bfloat16,
                                             device="cuda"))["staged"] == 0
    # binary32 rows and bf16 rows of 16 lanes stay on the register kernels
    assert rn.plan(rn.RN_OP_LN, torch.empty(4096, 1024, device="cuda"))["staged"] == 0
    x = torch.empty(4096, 512, dtype=torch.bfloat16, device="cuda")
    assert rn.plan(rn.RN_OP_LN, x)["staged"] == 0


@pytest.mark.parametrize("dim,layout", [(128, 2), (768, 2), (1000, 1), (1024, 2), (4096, 2),
                                        (4097, 0), (5120, 1), (8192, 2), (16384, 2)])
def test_layout_class_of_the_planned_launch(dim, layout):
    # 2: every thread owns all its chunk slots in every row (no slot tests);
    # 1: aligned rows with a ragged last round of slots, or more than four
    # chunks per thread; 0: rows off the 16-byte grid.
    x = torch.empty(4096, dim, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(dim, dtype=torch.bfloat16, device="cuda")
    assert rn.plan(rn.RN_OP_LN, x, weight=w, bias=w)["exact"] == layout


@pytest.mark.parametrize("dtype,dim", [(torch.bfloat16, 768), (torch.bfloat16, 8192),
                                       (torch.bfloat16, 1000), (torch.float32, 2048)])
def test_null_vectors_match_explicit_ones_and_zeros(dtype, dim):
    # A NULL weight (bias) is all ones (zeros). The kernels run separate row
    # loops for present and absent vectors; both must give the same bits.
    x = wl.random_rows(999, dim, dtype, seed=dim + 5, mean=0.5, std=2.0).cuda()
    ones = torch.ones(dim, dtype=dtype, device="cuda")
    zeros = torch.zeros(dim, dtype=dtype, device="cuda")
    b = wl.random_vector(dim, dtype, seed=6, mean=0.0, std=0.1).cuda()
    assert torch.equal(rn.rms_norm(x, None, 1e-6), rn.rms_norm(x, ones, 1e-6))
    assert torch.equal(rn.layer_norm(x, None, None, 1e-5), rn.layer_norm(x, ones, zeros, 1e-5))
    assert torch.equal(rn.layer_norm(x, None, b, 1e-5), rn.layer_norm(x, ones, b, 1e-5))
