"""The C-ABI library on the host (CPU only): it loads, exports every entry
point the header declares, and validates arguments before any CUDA call.
Only invalid calls and rows == 0 calls are made here; they return before the
library touches the CUDA runtime, so no GPU is needed."""
import ctypes

import numpy as np
import os
import re

import pytest

import transformer_row_normalization_b200 as rn
from transformer_row_normalization_b200 import rn_view

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rownorm.h")

FAKE = 0x7F0000000000  # a 256-byte-aligned address; never dereferenced


@pytest.fixture(scope="module")
def lib():
    from transformer_row_normalization_b200 import build_lib
    build_lib.build()
    return rn.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"RN_API\s+[\w\s\*]+?\b(rn_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("rn_rms_norm", "rn_layer_norm", "rn_dual_head_rms_norm", "rn_status_string",
              "rn_last_error", "rn_abi_version", "rn_plan", "rn_set_grid_override"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in rownorm.h but not exported"


def test_only_declared_symbols_are_exported(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", rn.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    exported = {e for e in exported if not e.startswith("_")}
    assert exported == set(declared_functions())


def test_status_strings_and_version(lib):
    assert lib.rn_abi_version() == 3
    assert lib.rn_status_string(0) == b"ok"
    for st in range(1, 9):
        assert lib.rn_status_string(st) not in (b"ok", b"unknown status")
    assert lib.rn_status_string(99) == b"unknown status"


def V(data=FAKE, rows=4, dim=64, stride=None, dtype=1):
    return rn_view(data, rows, dim, dim if stride is None else stride, dtype)


def rms(lib, x, y, w=None, eps=1e-6):
    return lib.rn_rms_norm(ctypes.byref(x) if x is not None else None, w, eps,
                           ctypes.byref(y) if y is not None else None, None)


def ln(lib, x, y, w=None, b=None, eps=1e-5):
    return lib.rn_layer_norm(ctypes.byref(x), w, b, eps, ctypes.byref(y), None)


def test_rejects_null_views_and_data(lib):
    assert rms(lib, None, V()) == 1
    assert rms(lib, V(), None) == 1
    assert rms(lib, V(data=None), V(data=FAKE + 4096)) == 1
    assert b"data is NULL" in lib.rn_last_error()


def test_rejects_bad_shapes(lib):
    y = V(data=FAKE + (1 << 20))
    assert rms(lib, V(rows=-1), y) == 2
    assert rms(lib, V(dim=0), V(data=FAKE + (1 << 20), dim=0)) == 2
    assert rms(lib, V(stride=63), y) == 2
    assert rms(lib, V(rows=4), V(data=FAKE + (1 << 20), rows=5)) == 2
    assert rms(lib, V(dim=64), V(data=FAKE + (1 << 20), dim=65)) == 2
    assert rms(lib, V(rows=1 << 40, stride=1 << 40), V(data=FAKE + (1 << 20))) == 2


def test_rejects_bad_dtypes(lib):
    assert rms(lib, V(dtype=7), V(data=FAKE + 4096, dtype=7)) == 3
    assert rms(lib, V(dtype=0), V(data=FAKE + 4096, dtype=1)) == 3


def test_rejects_bad_eps(lib):
    y = V(data=FAKE + 4096)
    for eps in (float("nan"), -1e-6, float("inf")):
        assert rms(lib, V(), y, eps=eps) == 4
        assert ln(lib, V(), y, eps=eps) == 4
    assert rms(lib, V(), V(data=FAKE + 4096, rows=0), eps=0.0) == 2  # rows differ
    assert rms(lib, V(rows=0), V(data=FAKE + 4096, rows=0), eps=0.0) == 0


def test_rejects_misalignment(lib):
    assert rms(lib, V(data=FAKE + 1), V(data=FAKE + 4096)) == 5
    assert rms(lib, V(dtype=0, data=FAKE + 2), V(dtype=0, data=FAKE + 4096)) == 5
    assert rms(lib, V(), V(data=FAKE + 4096), w=ctypes.c_void_p(FAKE + 8191)) == 5
    assert ln(lib, V(), V(data=FAKE + 4096), b=ctypes.c_void_p(FAKE + 8193)) == 5


def test_rejects_overlap_but_allows_in_place(lib):
    x = V(rows=0)  # rows == 0: an exact alias is OK and enqueues nothing
    assert rms(lib, x, V(rows=0)) == 0
    # partial overlap: y starts inside x
    assert rms(lib, V(), V(data=FAKE + 64)) == 6
    # same data, different stride: overlapping, not identical
    assert rms(lib, V(stride=128), V(stride=64)) == 6
    # output over the weight
    assert rms(lib, V(), V(data=FAKE + 4096), w=ctypes.c_void_p(FAKE + 4096 + 64)) == 6
    assert ln(lib, V(), V(data=FAKE + 4096), b=ctypes.c_void_p(FAKE + 4096 + 64)) == 6


def test_rejects_unsupported_widths(lib):
    # RMSNorm / LayerNorm stream rows up to RN_MAX_DIM_STREAM (4M) columns
    big = (1 << 22) + 1
    y = V(data=FAKE + (1 << 40), rows=2, dim=big, stride=big)
    assert rms(lib, V(rows=2, dim=big, stride=big), y) == 7
    assert ln(lib, V(rows=2, dim=big, stride=big), y) == 7
    # the fused ops hold rows in registers: 32768 bf16 / 16384 f32 at most
    x, r = V(rows=2, dim=32769, stride=32769), V(data=FAKE + (1 << 30), rows=2, dim=32769,
                                                 stride=32769)
    y, h = V(data=FAKE + (2 << 30), rows=2, dim=32769, stride=32769), \
        V(data=FAKE + (3 << 30), rows=2, dim=32769, stride=32769)
    assert add_rms(lib, x, r, y, h) == 7
    assert b"fused ops" in lib.rn_last_error()


def test_rows_zero_is_a_no_op(lib):
    assert rms(lib, V(rows=0), V(data=FAKE + 4096, rows=0)) == 0
    assert ln(lib, V(rows=0), V(data=FAKE + 4096, rows=0)) == 0


def dual(lib, q, k, yq, yk, wq=FAKE + (3 << 20), wk=FAKE + (3 << 20) + 4096, eps=1e-6):
    return lib.rn_dual_head_rms_norm(ctypes.byref(q), ctypes.byref(k),
                                     None if wq is None else ctypes.c_void_p(wq),
                                     None if wk is None else ctypes.c_void_p(wk), eps,
                                     ctypes.byref(yq), ctypes.byref(yk), None)


def test_dual_validation(lib):
    M = 1 << 20
    q, k = V(rows=0, dim=128), V(data=FAKE + M, rows=0, dim=128)
    yq, yk = V(data=FAKE + 2 * M, rows=0, dim=128), V(data=FAKE + 2 * M + 8192, rows=0, dim=128)
    assert dual(lib, q, k, yq, yk) == 0
    assert dual(lib, q, k, yq, yk, wq=None) == 1
    assert dual(lib, q, k, yq, yk, wk=None) == 1
    assert dual(lib, q, V(data=FAKE + M, rows=0, dim=128, dtype=0), yq,
                V(data=FAKE + 2 * M + 8192, rows=0, dim=128, dtype=0)) == 3
    big = V(rows=0, dim=2048)
    assert dual(lib, big, k, V(data=FAKE + 2 * M, rows=0, dim=2048), yk) == 7
    # yq over k, yk over q
    q4, k4 = V(rows=4, dim=128), V(data=FAKE + M, rows=4, dim=128)
    assert dual(lib, q4, k4, V(data=FAKE + M, rows=4, dim=128),
                V(data=FAKE + 2 * M, rows=4, dim=128)) == 6
    assert dual(lib, q4, k4, V(data=FAKE + 2 * M, rows=4, dim=128),
                V(data=FAKE, rows=4, dim=128)) == 6
    # yq and yk over each other
    assert dual(lib, q4, k4, V(data=FAKE + 2 * M, rows=4, dim=128),
                V(data=FAKE + 2 * M + 256, rows=4, dim=128)) == 6
    assert dual(lib, q, k, yq, yk, eps=float("nan")) == 4


def test_testing_controls(lib):
    assert lib.rn_set_grid_override(-1) == 2
    assert lib.rn_set_grid_override(0) == 0
    assert lib.rn_set_path_override(4) == 2
    assert lib.rn_set_path_override(0) == 0
    assert lib.rn_set_ring_wait_test(2) == 2
    assert lib.rn_set_ring_wait_test(-1) == 2
    assert lib.rn_set_ring_wait_test(0) == 0
    assert lib.rn_device_error_count(None, 0) == 1


@pytest.mark.parametrize("shape,strides,want", [
    ((4, 128, 1024), (128 * 1024, 1024, 1), (512, 1024, 1024)),
    ((1024,), (1,), (1, 1024, 1024)),
    ((8, 7), (10, 1), (8, 7, 10)),
    ((2, 1, 3, 5), (30, 99, 10, 1), (6, 5, 10)),
    ((1, 1, 9), (9, 9, 1), (1, 9, 9)),
    ((0, 16), (16, 1), (0, 16, 16)),
])
def test_view_params_folds_leading_axes(shape, strides, want):
    assert rn.view_params(shape, strides) == want


@pytest.mark.parametrize("shape,strides", [
    ((4, 8), (8, 2)),          # last axis not contiguous
    ((2, 3, 8), (40, 8, 1)),   # leading axes do not fold (40 != 3 * 8)
    ((4, 8), (4, 1)),          # rows overlap
])
def test_view_params_rejects(shape, strides):
    with pytest.raises(ValueError):
        rn.view_params(shape, strides)


def test_cpu_tensors_are_rejected_loudly():
    import torch
    x = torch.zeros(2, 8)
    with pytest.raises(TypeError, match="CUDA"):
        rn.rms_norm(x, None, 1e-6)


class _OnDevice:
    """Stands in for a CUDA tensor: the binding's device check reads only
    is_cuda and device, and raises before any other use."""

    is_cuda = True

    def __init__(self, index):
        import torch
        self.device = torch.device("cuda", index)


class _Stream:
    def __init__(self, index):
        import torch
        self.device = torch.device("cuda", index)


@pytest.mark.parametrize("call", [
    lambda a, b: rn.rms_norm(a, b, 1e-6),
    lambda a, b: rn.rms_norm(a, None, 1e-6, out=b),
    lambda a, b: rn.layer_norm(a, None, b, 1e-5),
    lambda a, b: rn.dual_head_rms_norm(a, b, a, a, 1e-6),
    lambda a, b: rn.dual_head_rms_norm(a, a, a, a, 1e-6, out_k=b),
    lambda a, b: rn.add_rms_norm(a, b, None, 1e-6),
    lambda a, b: rn.add_rms_norm(a, a, None, 1e-6, out_h=b),
    lambda a, b: rn.gated_rms_norm(a, b, None, 1e-6),
    lambda a, b: rn.dual_head_rms_norm_rope(a, a, a, a, 1e-6, b, 0, 8),
])
def test_tensors_on_another_device_are_rejected(call):
    with pytest.raises(TypeError, match="one device"):
        call(_OnDevice(0), _OnDevice(1))


def test_stream_on_another_device_is_rejected():
    with pytest.raises(TypeError, match="stream"):
        rn.rms_norm(_OnDevice(0), None, 1e-6, stream=_Stream(1))


def add_rms(lib, x, r, y, h, w=None, eps=1e-6):
    return lib.rn_add_rms_norm(ctypes.byref(x), ctypes.byref(r) if r is not None else None, w,
                               eps, ctypes.byref(y), ctypes.byref(h) if h is not None else None,
                               None)


def gated(lib, x, z, y, w=None, eps=1e-6):
    return lib.rn_gated_rms_norm(ctypes.byref(x), ctypes.byref(z) if z is not None else None, w,
                                 eps, ctypes.byref(y), None)


MB = 1 << 20


def test_add_rms_validation(lib):
    x, r = V(), V(data=FAKE + MB)
    y, h = V(data=FAKE + 2 * MB), V(data=FAKE + 3 * MB)
    assert add_rms(lib, x, None, y, h) == 1
    assert add_rms(lib, x, r, y, None) == 1
    assert add_rms(lib, x, V(data=FAKE + MB, rows=5), y, h) == 2
    assert add_rms(lib, x, V(data=FAKE + MB, dtype=0), y, h) == 3
    assert add_rms(lib, x, r, y, h, eps=float("nan")) == 4
    # the residual and h must share x's 16-byte phase on every row
    assert add_rms(lib, x, V(data=FAKE + MB + 2), y, h) == 5
    assert b"residual" in lib.rn_last_error()
    assert add_rms(lib, x, r, y, V(data=FAKE + 3 * MB + 8)) == 5
    assert add_rms(lib, x, V(data=FAKE + MB, stride=65), y, h) == 5
    # overlaps: y over h, y over the residual, h partly over x or the residual
    assert add_rms(lib, x, r, V(data=FAKE + 3 * MB), h) == 6
    assert add_rms(lib, x, r, V(data=FAKE + MB + 64), h) == 6
    assert add_rms(lib, x, r, y, V(data=FAKE + 64)) == 6
    assert add_rms(lib, x, r, y, V(data=FAKE + MB + 64)) == 6
    assert add_rms(lib, x, r, y, h, w=ctypes.c_void_p(FAKE + 3 * MB + 16)) == 6
    # h may be x or the residual exactly; y may be x unless h is
    z = dict(rows=0)
    assert add_rms(lib, V(**z), V(data=FAKE + MB, **z), V(data=FAKE + 2 * MB, **z), V(**z)) == 0
    assert add_rms(lib, V(**z), V(data=FAKE + MB, **z), V(data=FAKE + 2 * MB, **z),
                   V(data=FAKE + MB, **z)) == 0
    assert add_rms(lib, V(**z), V(data=FAKE + MB, **z), V(**z), V(data=FAKE + 3 * MB, **z)) == 0


def test_gated_rms_validation(lib):
    x, zv, y = V(), V(data=FAKE + MB), V(data=FAKE + 2 * MB)
    assert gated(lib, x, None, y) == 1
    assert gated(lib, x, V(data=FAKE + MB, dim=32), y) == 2
    assert gated(lib, x, zv, y, eps=-1.0) == 4
    assert gated(lib, x, V(data=FAKE + MB + 4), y) == 5
    assert gated(lib, x, zv, V(data=FAKE + MB)) == 6   # y over the gate
    assert gated(lib, x, zv, V(data=FAKE + 32)) == 6   # y partly over x
    z = dict(rows=0)
    assert gated(lib, V(**z), V(data=FAKE + MB, **z), V(**z)) == 0  # y == x


# ---------------------------------------------------------------------------
# RoPE: the host table builder, and validation of the fused entry


def test_rope_table_matches_the_math_library():
    import math
    t = rn.rope_table(8, 5, base=10000.0, scale=0.5)
    for p in range(5):
        for i in range(4):
            theta = p * 0.5 * (10000.0 ** (-2.0 * i / 8))
            assert t[p, i].item() == float(np.float32(math.cos(theta)))
            assert t[p, 4 + i].item() == float(np.float32(math.sin(theta)))
    f = [1.0, 0.25]
    t = rn.rope_table(4, 3000, inv_freq=f)
    assert t[2999, 0].item() == float(np.float32(math.cos(2999.0)))
    assert t[2999, 3].item() == float(np.float32(math.sin(2999.0 * 0.25)))


def test_rope_table_rejects_bad_schedules(lib):
    buf = (ctypes.c_float * 64)()
    assert lib.rn_rope_table(7, 10000.0, 1.0, None, 4, buf) == 2
    assert lib.rn_rope_table(8, 10000.0, 1.0, None, -1, buf) == 2
    assert lib.rn_rope_table(8, 10000.0, 1.0, None, 4, None) == 1
    assert lib.rn_rope_table(8, 0.0, 1.0, None, 4, buf) == 4
    assert lib.rn_rope_table(8, 10000.0, float("inf"), None, 4, buf) == 4


def rope_call(lib, q, k, yq, yk, rope, wq=FAKE + (3 << 20), wk=FAKE + (3 << 20) + 4096):
    return lib.rn_dual_head_rms_norm_rope(
        ctypes.byref(q), ctypes.byref(k), ctypes.c_void_p(wq), ctypes.c_void_p(wk), 1e-6,
        ctypes.byref(rope) if rope is not None else None, ctypes.byref(yq), ctypes.byref(yk), None)


def test_rope_validation(lib):
    table = FAKE + (5 << 20)
    R = lambda **kw: rn.rn_rope(**{**dict(table=table, n_pos=4096, offset=0, dims=64,
                                           traditional=0, heads_q=4, heads_k=2), **kw})
    q, k = V(rows=8, dim=64), V(data=FAKE + MB, rows=4, dim=64)
    yq, yk = V(data=FAKE + 2 * MB, rows=8, dim=64), V(data=FAKE + 3 * MB, rows=4, dim=64)
    assert rope_call(lib, q, k, yq, yk, None) == 1
    assert rope_call(lib, q, k, yq, yk, R(heads_q=0)) == 2
    assert rope_call(lib, q, k, yq, yk, R(heads_q=3)) == 2          # 8 rows, 3 heads
    assert rope_call(lib, q, k, yq, yk, R(heads_k=4)) == 2          # 2 tokens vs 1
    assert rope_call(lib, q, k, yq, yk, R(dims=63)) == 2
    assert rope_call(lib, q, k, yq, yk, R(dims=66)) == 2
    assert rope_call(lib, q, k, yq, yk, R(offset=4095)) == 2        # needs 2 positions
    assert b"positions" in lib.rn_last_error()
    assert rope_call(lib, q, k, yq, yk, R(table=None)) == 1
    assert rope_call(lib, q, k, yq, yk, R(table=table + 2)) == 5
    # an output over the table
    assert rope_call(lib, q, k, V(data=table + 256, rows=8, dim=64), yk, R()) == 6
    z = dict(rows=0, dim=64)
    assert rope_call(lib, V(**z), V(data=FAKE + MB, **z), V(data=FAKE + 2 * MB, **z),
                     V(data=FAKE + 3 * MB, **z), R()) == 0


# ---------------------------------------------------------------------------
# head rows in blocks (e.g. a slice of a packed QKV buffer)


@pytest.mark.parametrize("shape,strides,want", [
    ((2, 3, 8), (40, 8, 1), (6, 8, 8, 3, 40)),
    ((5, 32, 128), (48 * 128, 128, 1), (160, 128, 128, 32, 48 * 128)),   # q of a QKV
    ((2, 4, 3, 16), (400, 100, 16, 1), (24, 16, 16, 3, 100)),            # blocks fold
    ((4, 128, 1024), (128 * 1024, 1024, 1), (512, 1024, 1024, 0, 0)),  # one stride
])
def test_view_layout_blocks(shape, strides, want):
    assert rn.view_layout(shape, strides) == want


@pytest.mark.parametrize("shape,strides", [
    ((2, 3, 8), (20, 8, 1)),         # blocks overlap (20 < 2 * 8 + 8)
    ((2, 3, 8), (40, 4, 1)),         # rows overlap
    ((2, 2, 3, 8), (50, 100, 8, 1)),  # block axes do not fold
])
def test_view_layout_rejects(shape, strides):
    with pytest.raises(ValueError):
        rn.view_layout(shape, strides)


def test_block_views_are_validated(lib):
    def B(data=FAKE, rows=12, dim=64, stride=64, inner=4, outer=512, dtype=1):
        return rn_view(data, rows, dim, stride, dtype, inner, outer)
    y = V(data=FAKE + MB, rows=12, dim=64)
    assert rms(lib, B(outer=200), y) == 2          # blocks overlap
    assert rms(lib, B(inner=-1), y) == 2
    assert rms(lib, B(stride=32), y) == 2          # rows overlap inside a block
    # overlap is judged on each view's whole span (first to last row), so an
    # output anywhere inside the input's span, even between its blocks, is
    # refused unless it is the same view
    assert rms(lib, B(), B(data=FAKE + 512 * 2 + 2 * 64 * 2)) == 6
    assert rms(lib, B(), V(data=FAKE + 4 * 64 * 2, dim=64, rows=12)) == 6
    assert rms(lib, B(rows=0), B(rows=0)) == 0
