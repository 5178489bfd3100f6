"""fp64 CPU oracle for fused last-axis row normalization.

TEST INFRASTRUCTURE. Only the test suite, the entry module's ``smoke()`` and
the benchmark's CPU-baseline leg use this package. It shares no code with the
CUDA library (it neither imports it nor is imported by it); the arithmetic
lives in ``rownorm_oracle.c``, which states what each function follows on the
pages ("Fused transformer kernels on Emily", "Emily.Fast", "norm_fusion.rs"),
including the residual-add and gated RMSNorm fusions of "norm_fusion.rs".

Inputs are numpy arrays (or CPU torch tensors) holding the exact bytes the
GPU sees: float32 values, or bfloat16 as raw uint16/int16 bit patterns.
Outputs are dense float64 arrays.

Parity of every function here is pinned by ``tests/test_oracle.py`` (closed
forms, invariants, library special cases, brute force on tiny rows) and the
pins are themselves checked against planted mistakes by
``tests/test_oracle_mutants.py``.
"""
import ctypes

import numpy as np

from . import build as _build

F32 = 0
BF16 = 1


def _as_numpy(a):
    if a is None:
        return None
    if not isinstance(a, np.ndarray):  # a CPU torch tensor
        import torch
        if a.dtype == torch.bfloat16:
            a = a.view(torch.int16)
        a = a.detach().cpu().numpy()
    return a


def _dtype_code(a):
    if a.dtype == np.float32:
        return F32
    if a.dtype in (np.uint16, np.int16):
        return BF16
    raise TypeError(f"oracle takes float32 or bfloat16 bit patterns, got {a.dtype}")


def _view(x):
    """(array, rows, dim, row_stride) for a [..., dim] array. A 2-D array may
    carry a row stride larger than dim (a strided view of a wider buffer)."""
    x = _as_numpy(x)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    if x.ndim > 2:
        x = np.ascontiguousarray(x).reshape(-1, x.shape[-1])
    if x.strides[1] != x.itemsize or x.strides[0] % x.itemsize or x.strides[0] < 0:
        x = np.ascontiguousarray(x)
    rows, dim = x.shape
    row_stride = x.strides[0] // x.itemsize if rows > 1 else dim
    return x, rows, dim, row_stride


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _vector(w, dim, code):
    if w is None:
        return None
    w = np.ascontiguousarray(_as_numpy(w)).reshape(-1)
    if w.size != dim or _dtype_code(w) != code:
        raise ValueError("weight/bias must match the row length and dtype")
    return w


class Oracle:
    """ctypes front end over one build of the oracle C file."""

    def __init__(self, path):
        lib = ctypes.CDLL(path)
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_rms_norm.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp,
                                        ctypes.c_float, vp, ctypes.c_int]
        lib.oracle_layer_norm.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp,
                                          vp, ctypes.c_float, vp, ctypes.c_int]
        lib.oracle_dual_head_rms_norm.argtypes = [
            vp, i64, i64, i64, vp, i64, i64, i64, ctypes.c_int, vp, vp,
            ctypes.c_float, vp, vp, ctypes.c_int]
        lib.oracle_add_rms_norm.argtypes = [vp, vp, ctypes.c_int, i64, i64, i64, i64,
                                            vp, ctypes.c_float, vp, vp, ctypes.c_int]
        lib.oracle_gated_rms_norm.argtypes = [vp, vp, ctypes.c_int, i64, i64, i64, i64,
                                              vp, ctypes.c_float, vp, ctypes.c_int]
        lib.oracle_dual_head_rms_norm_rope.argtypes = [
            vp, i64, i64, i64, vp, i64, i64, i64, ctypes.c_int, vp, vp, ctypes.c_float,
            i64, i64, i64, i64, ctypes.c_int, ctypes.c_float, ctypes.c_float, vp, vp, vp,
            ctypes.c_int]
        lib.oracle_decode.argtypes = [vp, ctypes.c_int, i64, vp]
        for fn in (lib.oracle_rms_norm, lib.oracle_layer_norm,
                   lib.oracle_dual_head_rms_norm, lib.oracle_add_rms_norm,
                   lib.oracle_gated_rms_norm, lib.oracle_dual_head_rms_norm_rope):
            fn.restype = ctypes.c_int
        lib.oracle_decode.restype = None
        self._lib = lib
        self.path = path

    def rms_norm(self, x, weight, eps, nthreads=1):
        """RMSNorm of every row of ``x`` in fp64; float64 [rows, dim]."""
        x, rows, dim, stride = _view(x)
        code = _dtype_code(x)
        w = _vector(weight, dim, code)
        y = np.empty((rows, dim), dtype=np.float64)
        st = self._lib.oracle_rms_norm(_ptr(x), code, rows, dim, stride, _ptr(w),
                                       float(eps), _ptr(y), int(nthreads))
        if st:
            raise ValueError(f"oracle_rms_norm rejected its arguments (status {st})")
        return y

    def layer_norm(self, x, weight, bias, eps, nthreads=1):
        """LayerNorm of every row of ``x`` in fp64; float64 [rows, dim]."""
        x, rows, dim, stride = _view(x)
        code = _dtype_code(x)
        w = _vector(weight, dim, code)
        b = _vector(bias, dim, code)
        y = np.empty((rows, dim), dtype=np.float64)
        st = self._lib.oracle_layer_norm(_ptr(x), code, rows, dim, stride, _ptr(w),
                                         _ptr(b), float(eps), _ptr(y), int(nthreads))
        if st:
            raise ValueError(f"oracle_layer_norm rejected its arguments (status {st})")
        return y

    def dual_head_rms_norm(self, q, k, wq, wk, eps, nthreads=1):
        """(RMSNorm(q, wq), RMSNorm(k, wk)) in fp64, queries first."""
        q, qr, qd, qs = _view(q)
        k, kr, kd, ks = _view(k)
        code = _dtype_code(q)
        if _dtype_code(k) != code:
            raise TypeError("q and k must share a dtype")
        wq_ = _vector(wq, qd, code)
        wk_ = _vector(wk, kd, code)
        yq = np.empty((qr, qd), dtype=np.float64)
        yk = np.empty((kr, kd), dtype=np.float64)
        st = self._lib.oracle_dual_head_rms_norm(
            _ptr(q), qr, qd, qs, _ptr(k), kr, kd, ks, code, _ptr(wq_), _ptr(wk_),
            float(eps), _ptr(yq), _ptr(yk), int(nthreads))
        if st:
            raise ValueError(f"oracle_dual_head_rms_norm rejected its arguments ({st})")
        return yq, yk

    def add_rms_norm(self, x, residual, weight, eps, nthreads=1):
        """(y, h): h = x + residual stored in the input type (as fp64), and
        y = RMSNorm(h) * weight, in fp64; both float64 [rows, dim]."""
        x, rows, dim, xs = _view(x)
        r, rr, rd, rs = _view(residual)
        code = _dtype_code(x)
        if (rr, rd) != (rows, dim) or _dtype_code(r) != code:
            raise ValueError("x and residual must share shape and dtype")
        w = _vector(weight, dim, code)
        y = np.empty((rows, dim), dtype=np.float64)
        h = np.empty((rows, dim), dtype=np.float64)
        st = self._lib.oracle_add_rms_norm(_ptr(x), _ptr(r), code, rows, dim, xs, rs,
                                           _ptr(w), float(eps), _ptr(y), _ptr(h),
                                           int(nthreads))
        if st:
            raise ValueError(f"oracle_add_rms_norm rejected its arguments (status {st})")
        return y, h

    def gated_rms_norm(self, x, gate, weight, eps, nthreads=1):
        """RMSNorm(x) * weight * silu(gate) in fp64; float64 [rows, dim]."""
        x, rows, dim, xs = _view(x)
        z, zr, zd, zs = _view(gate)
        code = _dtype_code(x)
        if (zr, zd) != (rows, dim) or _dtype_code(z) != code:
            raise ValueError("x and gate must share shape and dtype")
        w = _vector(weight, dim, code)
        y = np.empty((rows, dim), dtype=np.float64)
        st = self._lib.oracle_gated_rms_norm(_ptr(x), _ptr(z), code, rows, dim, xs, zs,
                                             _ptr(w), float(eps), _ptr(y), int(nthreads))
        if st:
            raise ValueError(f"oracle_gated_rms_norm rejected its arguments (status {st})")
        return y

    def dual_head_rms_norm_rope(self, q, k, wq, wk, eps, heads_q, heads_k, offset, dims,
                                traditional=False, base=10000.0, scale=1.0, inv_freq=None,
                                nthreads=1):
        """(RoPE(RMSNorm(q, wq)), RoPE(RMSNorm(k, wk))) in fp64, queries first.
        Rows are head rows, token-major: row r is token r // heads. ``base``
        and ``scale`` travel as binary32; ``inv_freq`` (dims/2 float32) replaces
        base^(-2i/dims)."""
        q, qr, qd, qs = _view(q)
        k, kr, kd, ks = _view(k)
        code = _dtype_code(q)
        if _dtype_code(k) != code:
            raise TypeError("q and k must share a dtype")
        wq_ = _vector(wq, qd, code)
        wk_ = _vector(wk, kd, code)
        f = None
        if inv_freq is not None:
            f = np.ascontiguousarray(_as_numpy(inv_freq), dtype=np.float32).reshape(-1)
            if f.size != dims // 2:
                raise ValueError("inv_freq must hold dims / 2 values")
        yq = np.empty((qr, qd), dtype=np.float64)
        yk = np.empty((kr, kd), dtype=np.float64)
        st = self._lib.oracle_dual_head_rms_norm_rope(
            _ptr(q), qr, qd, qs, _ptr(k), kr, kd, ks, code, _ptr(wq_), _ptr(wk_), float(eps),
            int(heads_q), int(heads_k), int(offset), int(dims), int(bool(traditional)),
            float(base), float(scale), _ptr(f), _ptr(yq), _ptr(yk), int(nthreads))
        if st:
            raise ValueError(f"oracle_dual_head_rms_norm_rope rejected its arguments ({st})")
        return yq, yk

    def decode(self, a):
        """Exact fp64 values of a float32 or bfloat16-bits array."""
        a = np.ascontiguousarray(_as_numpy(a))
        out = np.empty(a.size, dtype=np.float64)
        self._lib.oracle_decode(_ptr(a), _dtype_code(a), a.size, _ptr(out))
        return out.reshape(a.shape)


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def rms_norm(x, weight, eps, nthreads=1):
    return default().rms_norm(x, weight, eps, nthreads)


def layer_norm(x, weight, bias, eps, nthreads=1):
    return default().layer_norm(x, weight, bias, eps, nthreads)


def dual_head_rms_norm(q, k, wq, wk, eps, nthreads=1):
    return default().dual_head_rms_norm(q, k, wq, wk, eps, nthreads)


def add_rms_norm(x, residual, weight, eps, nthreads=1):
    return default().add_rms_norm(x, residual, weight, eps, nthreads)


def gated_rms_norm(x, gate, weight, eps, nthreads=1):
    return default().gated_rms_norm(x, gate, weight, eps, nthreads)


def dual_head_rms_norm_rope(q, k, wq, wk, eps, heads_q, heads_k, offset, dims,
                            traditional=False, base=10000.0, scale=1.0, inv_freq=None,
                            nthreads=1):
    return default().dual_head_rms_norm_rope(q, k, wq, wk, eps, heads_q, heads_k, offset, dims,
                                             traditional, base, scale, inv_freq, nthreads)


def decode(a):
    return default().decode(a)
