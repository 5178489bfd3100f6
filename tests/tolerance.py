"""Parity tolerances and output guards shared by the GPU tests.

fp32 outputs: max |gpu - oracle| <= 1e-5 (the stated bar; "Fused transformer
kernels on Emily", Part 1, Correctness expects round-off of about 1e-5).

bf16 outputs: |gpu - oracle| <= one bfloat16 ulp of the exact value, i.e. the
spacing of bfloat16 numbers in the binade of |oracle| (8 significant bits:
2^(e-7) for |v| in [2^e, 2^(e+1)), relative 2^-8 .. 2^-7). The kernel rounds
a binary32 result once, so it sits within half an ulp plus binary32 error.
LayerNorm adds the bias after the product n*w; where n*w and b nearly cancel
the exact result is tiny while the binary32 error scales with |n*w| + |b|,
so LayerNorm also allows an absolute floor 1e-5 * (|n*w| + |b| + 1) (that is
~170 binary32 ulps of the operands, far below one bf16 ulp of them).

Gated RMSNorm in fp32 (``scaled=True``): its outputs reach |y| ~ 40 (the gate's
silu grows like the gate), where a fixed 1e-5 is below the binary32 error of
the product chain itself (four roundings; __expf within 2 + 1.2 |t| ulps and
__fdividef within 2 ulps: about 1e-6 relative for |t| < 20). Its bound is
1e-5 * (1 + |y|), ten times that error.

RMSNorm + RoPE (``rope=(dims, traditional)``): each rotated output mixes the
two values of its plane, y_a = o_a cos - o_b sin. Where the two terms cancel,
the exact result is far below the plane's size, while the binary32 error of
the chain (about 4e-7 relative) scales with the plane norm
sqrt(y_a^2 + y_b^2) (rotation keeps it). So bf16 also allows an absolute
floor of 1e-5 times the plane norm, 25 times that error.
"""
import numpy as np
import torch


def bf16_ulp(v):
    a = np.abs(np.asarray(v, dtype=np.float64))
    _, e = np.frexp(a)                  # a = m * 2**e with m in [0.5, 1)
    ulp = np.ldexp(1.0, e - 8)          # 8 significant bits
    return np.where(a < 2.0 ** -126, 2.0 ** -133, ulp)


def to_f64(t):
    return t.detach().to("cpu").double().numpy()


def plane_norms(ref, dims, traditional):
    """sqrt(y_a^2 + y_b^2) of each element's RoPE plane (|y| past dims)."""
    ref = np.asarray(ref, dtype=np.float64)
    out = np.abs(ref).copy()
    half = dims // 2
    for i in range(half):
        a, b = (2 * i, 2 * i + 1) if traditional else (i, i + half)
        n = np.sqrt(ref[:, a] ** 2 + ref[:, b] ** 2)
        out[:, a] = out[:, b] = n
    return out


def check(gpu, ref, dtype, bias=None, what="", scaled=False, rope=None):
    """Assert parity; returns (max_abs_err, max_err_in_ulps or None)."""
    got = to_f64(gpu).reshape(ref.shape)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got) == np.isfinite(ref)), f"{what}: finiteness differs"
    if dtype == torch.float32:
        worst = float(err.max()) if err.size else 0.0
        if scaled:
            bad = err > 1e-5 * (1.0 + np.abs(ref))
            assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond 1e-5 * (1 + |y|)"
        else:
            assert worst <= 1e-5, f"{what}: max abs err {worst:.3e} > 1e-5"
        return worst, None
    ulp = bf16_ulp(ref)
    bound = ulp.copy()
    if rope is not None:
        bound = np.maximum(bound, 1e-5 * plane_norms(ref, *rope))
    if bias is not None:
        b = np.broadcast_to(to_f64(bias), ref.shape)
        floor = 1e-5 * (np.abs(ref - b) + np.abs(b) + 1.0)
        bound = np.maximum(bound, floor)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements off; worst at {i}: "
                             f"gpu {got[i]!r} oracle {ref[i]!r} ulp {ulp[i]!r}")
    return (float(err.max()) if err.size else 0.0,
            float((err / ulp).max()) if err.size else 0.0)


SENTINEL = {torch.float32: 0x7FC0DEAD, torch.bfloat16: 0x7FAB}


def guarded_empty(shape, dtype, pad=2048, row_gap=0, device="cuda"):
    """An output tensor inside a buffer whose surroundings (pad elements before
    and after, and row_gap elements after each row) hold a NaN sentinel.
    Returns (view, buffer, check) where check() asserts the guard bands are
    untouched."""
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    dim = shape[-1]
    stride = dim + row_gap
    n = pad + rows * stride + pad
    itype = torch.int32 if dtype == torch.float32 else torch.int16
    sentinel = SENTINEL[dtype]
    if itype == torch.int16 and sentinel > 0x7FFF:
        sentinel -= 0x10000
    buf = torch.full((n,), sentinel, dtype=itype, device=device).view(dtype)
    view = buf[pad:pad + rows * stride].view(rows, stride)[:, :dim]
    if len(shape) != 2:
        assert row_gap == 0
        view = view.reshape(shape)

    def check():
        bits = buf.view(itype)
        assert torch.all(bits[:pad] == sentinel), "write before the output"
        assert torch.all(bits[pad + rows * stride:] == sentinel), "write after the output"
        if row_gap:
            gaps = bits[pad:pad + rows * stride].view(rows, stride)[:, dim:]
            assert torch.all(gaps == sentinel), "write into the gap between rows"
    return view, buf, check
