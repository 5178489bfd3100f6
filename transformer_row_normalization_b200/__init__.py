"""Fused last-axis row normalization on NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``librownorm.so`` (declared in
``include/rownorm.h``). This module only marshals arguments: it turns torch
CUDA tensors into ``rn_view`` descriptors (data pointer, rows, dim, row
stride, dtype, and for head rows sliced out of a packed buffer the block
layout), passes the current CUDA stream, and raises on a nonzero status.
Every step of the computation runs in the library's CUDA kernels; there is
no CPU or framework fallback, and calling with CPU tensors or without the
built library raises. Calls are asynchronous on the stream and may be
captured in CUDA graphs.

    rn_rms_norm(x, weight, eps, out=None)               RMSNorm
    rn_layer_norm(x, weight, bias, eps, out=None)       LayerNorm
    rn_dual_head_rms_norm(q, k, wq, wk, eps, ...)       q/k head RMSNorm, one launch
    rn_dual_head_rms_norm_rope(q, k, wq, wk, eps, table, offset, dims, ...)
                                                        ... followed by RoPE
    rn_add_rms_norm(x, residual, weight, eps, ...)      residual add + RMSNorm
    rn_gated_rms_norm(x, z, weight, eps, ...)           RMSNorm * silu(gate)
    rope_table(dims, n_pos, base, scale, inv_freq)      RoPE cos/sin table

The names without the ``rn_`` prefix are the same calls.
"""
import ctypes
import os

__all__ = [
    "RowNormError", "rn_rms_norm", "rn_layer_norm", "rn_dual_head_rms_norm",
    "rn_dual_head_rms_norm_rope", "rn_add_rms_norm", "rn_gated_rms_norm", "rope_table",
    "rms_norm", "layer_norm", "dual_head_rms_norm", "dual_head_rms_norm_rope",
    "add_rms_norm", "gated_rms_norm", "plan", "set_grid_override",
    "set_path_override", "set_ring_wait_test", "device_error_count",
    "library_path", "load_library", "view_params", "view_layout",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librownorm.so")

RN_F32, RN_BF16 = 0, 1
RN_OP_RMS, RN_OP_LN, RN_OP_DUAL, RN_OP_ADD_RMS, RN_OP_GATED_RMS = 0, 1, 2, 3, 4
STATUS_NAMES = {0: "RN_OK", 1: "RN_ERR_NULL", 2: "RN_ERR_SHAPE", 3: "RN_ERR_DTYPE",
                4: "RN_ERR_EPS", 5: "RN_ERR_ALIGN", 6: "RN_ERR_OVERLAP",
                7: "RN_ERR_UNSUPPORTED", 8: "RN_ERR_CUDA"}


class RowNormError(RuntimeError):
    def __init__(self, status, detail):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {detail}")


class rn_view(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("dim", ctypes.c_int64), ("row_stride", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("inner_rows", ctypes.c_int64),
                ("outer_stride", ctypes.c_int64)]


class rn_rope(ctypes.Structure):
    _fields_ = [("table", ctypes.c_void_p), ("n_pos", ctypes.c_int64),
                ("offset", ctypes.c_int64), ("dims", ctypes.c_int32),
                ("traditional", ctypes.c_int32), ("heads_q", ctypes.c_int32),
                ("heads_k", ctypes.c_int32)]


class rn_launch_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "family", "threads_per_row", "chunks_per_thread", "smem_bytes", "block_threads",
        "grid_blocks", "blocks_per_sm", "vector_y", "phase_period", "exact", "staged",
        "stages", "stage_bytes")]


_lib = None


def library_path() -> str:
    return LIB_PATH


def load_library():
    """Load librownorm.so (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is not built; build it with "
                "`python -m transformer_row_normalization_b200.build_lib`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, f32 = ctypes.c_void_p, ctypes.c_float
        pv = ctypes.POINTER(rn_view)
        lib.rn_rms_norm.argtypes = [pv, vp, f32, pv, vp]
        lib.rn_layer_norm.argtypes = [pv, vp, vp, f32, pv, vp]
        lib.rn_dual_head_rms_norm.argtypes = [pv, pv, vp, vp, f32, pv, pv, vp]
        lib.rn_add_rms_norm.argtypes = [pv, pv, vp, f32, pv, pv, vp]
        lib.rn_gated_rms_norm.argtypes = [pv, pv, vp, f32, pv, vp]
        lib.rn_dual_head_rms_norm_rope.argtypes = [pv, pv, vp, vp, f32,
                                                   ctypes.POINTER(rn_rope), pv, pv, vp]
        lib.rn_rope_table.argtypes = [ctypes.c_int32, f32, f32, vp, ctypes.c_int64, vp]
        lib.rn_plan.argtypes = [ctypes.c_int, pv, pv, pv, pv, vp, vp,
                                ctypes.POINTER(rn_launch_info)]
        lib.rn_set_grid_override.argtypes = [ctypes.c_int]
        lib.rn_set_path_override.argtypes = [ctypes.c_int]
        lib.rn_device_error_count.argtypes = [ctypes.POINTER(ctypes.c_uint), ctypes.c_int]
        lib.rn_set_ring_wait_test.argtypes = [ctypes.c_int]
        lib.rn_status_string.argtypes = [ctypes.c_int]
        lib.rn_status_string.restype = ctypes.c_char_p
        lib.rn_last_error.argtypes = []
        lib.rn_last_error.restype = ctypes.c_char_p
        for fn in (lib.rn_rms_norm, lib.rn_layer_norm, lib.rn_dual_head_rms_norm,
                   lib.rn_add_rms_norm, lib.rn_gated_rms_norm, lib.rn_plan,
                   lib.rn_dual_head_rms_norm_rope, lib.rn_rope_table,
                   lib.rn_set_grid_override, lib.rn_abi_version,
                   lib.rn_set_path_override, lib.rn_device_error_count,
                   lib.rn_set_ring_wait_test):
            fn.restype = ctypes.c_int
        _lib = lib
    return _lib


def _check(status):
    if status != 0:
        lib = load_library()
        raise RowNormError(status, lib.rn_last_error().decode())


def view_params(shape, strides):
    """(rows, dim, row_stride) of a [..., dim] layout whose last axis is
    contiguous and whose leading axes fold into one row axis; raises
    ValueError otherwise. Pure shape arithmetic (no copies)."""
    shape, strides = tuple(shape), tuple(strides)
    if len(shape) == 0:
        raise ValueError("a row view needs at least one dimension")
    dim = shape[-1]
    if dim > 1 and strides[-1] != 1:
        raise ValueError("the last axis must be contiguous (stride 1)")
    rows = 1
    for s in shape[:-1]:
        rows *= s
    if len(shape) == 1:
        return rows, dim, dim
    lead = [(n, st) for n, st in zip(shape[:-1], strides[:-1]) if n != 1]
    if not lead:
        return rows, dim, dim
    row_stride = lead[-1][1]
    expect = row_stride
    for n, st in reversed(lead):
        if st != expect:
            raise ValueError("leading axes do not fold into one row axis")
        expect = st * n
    if rows > 1 and row_stride < dim:
        raise ValueError("rows overlap (row stride < dim)")
    return rows, dim, row_stride


def _fold(axes):
    """Stride of one axis equivalent to the (size, stride) axes, or None."""
    if not axes:
        return None
    stride = axes[-1][1]
    expect = stride
    for n, st in reversed(axes):
        if st != expect:
            return None
        expect = st * n
    return stride


def view_layout(shape, strides):
    """(rows, dim, row_stride, inner_rows, outer_stride) of a [..., dim] layout
    whose last axis is contiguous: one row stride when the leading axes fold
    into one row axis (inner_rows = 0), else blocks of the last leading axis
    (inner_rows rows row_stride apart, blocks outer_stride apart) when the
    other leading axes fold into one block axis -- e.g. the heads of a packed
    QKV buffer. Raises ValueError otherwise. Pure shape arithmetic."""
    try:
        rows, dim, row_stride = view_params(shape, strides)
        return rows, dim, row_stride, 0, 0
    except ValueError as single:
        shape, strides = tuple(shape), tuple(strides)
        if len(shape) < 3 or (shape[-1] > 1 and strides[-1] != 1):
            raise single
        dim = shape[-1]
        lead = [(n, st) for n, st in zip(shape[:-1], strides[:-1]) if n != 1]
        if len(lead) < 2:
            raise single
        inner, row_stride = lead[-1]
        outer = _fold(lead[:-1])
        if outer is None:
            raise ValueError("leading axes do not fold into rows or blocks of rows")
        if row_stride < dim or outer < (inner - 1) * row_stride + dim:
            raise ValueError("rows overlap")
        rows = 1
        for n in shape[:-1]:
            rows *= n
        return rows, dim, row_stride, inner, outer


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return RN_F32
    if t.dtype == torch.bfloat16:
        return RN_BF16
    raise TypeError(f"row normalization supports float32 and bfloat16, not {t.dtype}")


def _require_cuda(*tensors, stream=None):
    """Every tensor argument lives on one CUDA device, that of the first (the
    input the kernel is launched for), and so does a caller's stream. The
    kernels dereference every pointer on that device, so a tensor on another
    GPU would be read through a peer mapping or fault; it is rejected here,
    before anything is launched."""
    device = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise TypeError("tensors must live on a CUDA device: this library has no CPU path")
        if device is None:
            device = t.device
        elif t.device != device:
            raise TypeError(f"all tensors of a call must be on one device: {t.device} is not "
                            f"{device}")
    if stream is not None and device is not None and stream.device != device:
        raise TypeError(f"stream is on {stream.device}, the tensors on {device}")


def _view(t):
    rows, dim, row_stride, inner, outer = view_layout(t.shape, t.stride())
    return rn_view(t.data_ptr() if t.numel() else None, rows, dim, row_stride, _dtype_code(t),
                   inner, outer)


def _vector(v, dim, like):
    if v is None:
        return None
    if v.dim() != 1 or v.shape[0] != dim or v.stride(0) != 1:
        raise ValueError(f"weight/bias must be a contiguous vector of length {dim}")
    if v.dtype != like.dtype or v.device != like.device:
        raise TypeError("weight/bias must match the input's dtype and device")
    return ctypes.c_void_p(v.data_ptr())


def _stream(t, stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream(t.device)
    return ctypes.c_void_p(s.cuda_stream)


def rn_rms_norm(x, weight, eps=1e-6, out=None, stream=None):
    """RMSNorm over the last axis of the CUDA tensor ``x``; returns ``out``."""
    import torch
    _require_cuda(x, weight, out, stream=stream)
    out = torch.empty_like(x) if out is None else out
    xv, yv = _view(x), _view(out)
    lib = load_library()
    with torch.cuda.device(x.device):
        _check(lib.rn_rms_norm(ctypes.byref(xv), _vector(weight, xv.dim, x), float(eps),
                               ctypes.byref(yv), _stream(x, stream)))
    return out


def rn_layer_norm(x, weight, bias, eps=1e-5, out=None, stream=None):
    """LayerNorm over the last axis of the CUDA tensor ``x``; returns ``out``."""
    import torch
    _require_cuda(x, weight, bias, out, stream=stream)
    out = torch.empty_like(x) if out is None else out
    xv, yv = _view(x), _view(out)
    lib = load_library()
    with torch.cuda.device(x.device):
        _check(lib.rn_layer_norm(ctypes.byref(xv), _vector(weight, xv.dim, x),
                                 _vector(bias, xv.dim, x), float(eps), ctypes.byref(yv),
                                 _stream(x, stream)))
    return out


def rn_dual_head_rms_norm(q, k, wq, wk, eps=1e-6, out_q=None, out_k=None, stream=None):
    """(RMSNorm(q, wq), RMSNorm(k, wk)) from one kernel launch; queries first."""
    import torch
    _require_cuda(q, k, wq, wk, out_q, out_k, stream=stream)
    out_q = torch.empty_like(q) if out_q is None else out_q
    out_k = torch.empty_like(k) if out_k is None else out_k
    qv, kv, yqv, ykv = _view(q), _view(k), _view(out_q), _view(out_k)
    if wq is None or wk is None:
        raise ValueError("dual head norm needs both wq and wk")
    lib = load_library()
    with torch.cuda.device(q.device):
        _check(lib.rn_dual_head_rms_norm(
            ctypes.byref(qv), ctypes.byref(kv), _vector(wq, qv.dim, q), _vector(wk, kv.dim, k),
            float(eps), ctypes.byref(yqv), ctypes.byref(ykv), _stream(q, stream)))
    return out_q, out_k


def rn_add_rms_norm(x, residual, weight, eps=1e-6, out=None, out_h=None, stream=None):
    """(y, h): h = x + residual stored in x's dtype, y = RMSNorm(h) * weight, in
    one pass. ``out_h`` may be ``x`` or ``residual`` (in-place residual stream)."""
    import torch
    _require_cuda(x, residual, weight, out, out_h, stream=stream)
    out = torch.empty_like(x) if out is None else out
    out_h = torch.empty_like(x) if out_h is None else out_h
    xv, rv, yv, hv = _view(x), _view(residual), _view(out), _view(out_h)
    lib = load_library()
    with torch.cuda.device(x.device):
        _check(lib.rn_add_rms_norm(ctypes.byref(xv), ctypes.byref(rv),
                                   _vector(weight, xv.dim, x), float(eps), ctypes.byref(yv),
                                   ctypes.byref(hv), _stream(x, stream)))
    return out, out_h


def rn_gated_rms_norm(x, z, weight, eps=1e-6, out=None, stream=None):
    """RMSNorm(x) * weight * silu(z) over the last axis, in one pass."""
    import torch
    _require_cuda(x, z, weight, out, stream=stream)
    out = torch.empty_like(x) if out is None else out
    xv, zv, yv = _view(x), _view(z), _view(out)
    lib = load_library()
    with torch.cuda.device(x.device):
        _check(lib.rn_gated_rms_norm(ctypes.byref(xv), ctypes.byref(zv),
                                     _vector(weight, xv.dim, x), float(eps), ctypes.byref(yv),
                                     _stream(x, stream)))
    return out


def rope_table(dims, n_pos, base=10000.0, scale=1.0, inv_freq=None, device=None):
    """The cos/sin table of a RoPE schedule ([n_pos, dims] float32: cos of plane
    i at [:, i], sin at [:, dims // 2 + i]), computed on the host by the
    library (angles in double, rounded once); moved to ``device`` if given."""
    import torch
    table = torch.empty((int(n_pos), int(dims)), dtype=torch.float32)
    f = None
    if inv_freq is not None:
        f = torch.as_tensor(inv_freq, dtype=torch.float32).contiguous().cpu()
        if f.numel() != dims // 2:
            raise ValueError("inv_freq must hold dims // 2 values")
    _check(load_library().rn_rope_table(int(dims), float(base), float(scale),
                                        None if f is None else ctypes.c_void_p(f.data_ptr()),
                                        int(n_pos), ctypes.c_void_p(table.data_ptr())
                                        if table.numel() else None))
    return table if device is None else table.to(device)


def rn_dual_head_rms_norm_rope(q, k, wq, wk, eps, table, offset, dims, heads_q=None,
                               heads_k=None, traditional=False, out_q=None, out_k=None,
                               stream=None):
    """(RoPE(RMSNorm(q, wq)), RoPE(RMSNorm(k, wk))) from one kernel launch.
    q [tokens, heads_q, D] and k [tokens, heads_k, Dk] (or 2-D head rows with
    the head counts given); ``table`` is a CUDA float32 rope_table."""
    import torch
    _require_cuda(q, k, wq, wk, table, out_q, out_k, stream=stream)
    if heads_q is None:
        heads_q = q.shape[-2] if q.dim() >= 3 else 1
    if heads_k is None:
        heads_k = k.shape[-2] if k.dim() >= 3 else 1
    if table.dtype != torch.float32 or not table.is_contiguous() or table.dim() != 2:
        raise ValueError("table must be a contiguous [n_pos, dims] float32 tensor")
    if table.shape[1] != dims:
        raise ValueError(f"table has {table.shape[1]} columns, dims is {dims}")
    out_q = torch.empty_like(q) if out_q is None else out_q
    out_k = torch.empty_like(k) if out_k is None else out_k
    qv, kv, yqv, ykv = _view(q), _view(k), _view(out_q), _view(out_k)
    if wq is None or wk is None:
        raise ValueError("dual head norm needs both wq and wk")
    rope = rn_rope(table.data_ptr() if table.numel() else None, table.shape[0], int(offset),
                   int(dims), int(bool(traditional)), int(heads_q), int(heads_k))
    lib = load_library()
    with torch.cuda.device(q.device):
        _check(lib.rn_dual_head_rms_norm_rope(
            ctypes.byref(qv), ctypes.byref(kv), _vector(wq, qv.dim, q), _vector(wk, kv.dim, k),
            float(eps), ctypes.byref(rope), ctypes.byref(yqv), ctypes.byref(ykv),
            _stream(q, stream)))
    return out_q, out_k


rms_norm = rn_rms_norm
layer_norm = rn_layer_norm
dual_head_rms_norm_rope = rn_dual_head_rms_norm_rope
dual_head_rms_norm = rn_dual_head_rms_norm
add_rms_norm = rn_add_rms_norm
gated_rms_norm = rn_gated_rms_norm


def plan(op, x, out=None, weight=None, bias=None, k=None, out_k=None):
    """The launch configuration the library picks (see rn_launch_info). For
    RN_OP_ADD_RMS ``k`` is the residual and ``out_k`` the stored sum h; for
    RN_OP_GATED_RMS ``k`` is the gate."""
    import torch
    out = torch.empty_like(x) if out is None else out
    xv, yv = _view(x), _view(out)
    info = rn_launch_info()
    lib = load_library()
    with torch.cuda.device(x.device):
        if op == RN_OP_DUAL:
            out_k = torch.empty_like(k) if out_k is None else out_k
            kv, ykv = _view(k), _view(out_k)
            _check(lib.rn_plan(op, ctypes.byref(xv), ctypes.byref(yv), ctypes.byref(kv),
                               ctypes.byref(ykv), _vector(weight, xv.dim, x),
                               _vector(bias, kv.dim, k), ctypes.byref(info)))
        elif op in (RN_OP_ADD_RMS, RN_OP_GATED_RMS):
            out_k = torch.empty_like(x) if out_k is None else out_k
            kv, ykv = _view(k), _view(out_k)
            _check(lib.rn_plan(op, ctypes.byref(xv), ctypes.byref(yv), ctypes.byref(kv),
                               ctypes.byref(ykv), _vector(weight, xv.dim, x), None,
                               ctypes.byref(info)))
        else:
            _check(lib.rn_plan(op, ctypes.byref(xv), ctypes.byref(yv), None, None,
                               _vector(weight, xv.dim, x), _vector(bias, xv.dim, x),
                               ctypes.byref(info)))
    return {n: getattr(info, n) for n, _ in rn_launch_info._fields_}


def set_grid_override(blocks: int):
    """Testing control: launch exactly ``blocks`` blocks (0 = automatic)."""
    _check(load_library().rn_set_grid_override(int(blocks)))


def set_path_override(path: int):
    """Testing control: 0 automatic, 1 register kernels, 2 per-warp bulk-copy
    rings where they apply, 3 register kernels with per-thread prefetch."""
    _check(load_library().rn_set_path_override(int(path)))


def set_ring_wait_test(on: bool):
    """Testing control: ring stages never complete, so their bounded waits
    run out (1 ms) and the timeout path runs; False restores the limits."""
    _check(load_library().rn_set_ring_wait_test(int(bool(on))))


def device_error_count(reset: bool = False) -> int:
    """Stage waits that timed out in the ring kernels (synchronizes)."""
    n = ctypes.c_uint(0)
    _check(load_library().rn_device_error_count(ctypes.byref(n), int(reset)))
    return n.value
