"""Pins for the fp64 oracle: checks against facts fixed by the pages and by the
mathematics, never against the oracle itself.

Every ``pin_*`` takes an oracle object (``oracle.Oracle``) and raises
``AssertionError`` when the oracle is wrong. ``test_oracle.py`` runs them on
the real oracle; ``test_oracle_mutants.py`` runs them on copies of the oracle
with planted mistakes and requires each mistake to trip at least one pin.

Kinds of pin used here:
  closed forms     -- the pages' worked rows ("Emily.Fast" doctests; the iota
                      input of "Fused transformer kernels on Emily", Part 1)
                      evaluated from hand-derived exact statistics with
                      50-digit decimals;
  invariants       -- unit output RMS, zero mean / unit variance, constant
                      rows give the bias, scale and shift invariance,
                      permutation equivariance, weight/bias linearity;
  library routines -- torch.nn.functional.layer_norm / rms_norm / silu in
                      fp64; torch's binary32 -> bfloat16 cast for the
                      stored residual sum;
  brute force      -- exact rational mean and variance on rows of 1..5.

The residual-add and gated RMSNorm fusions ("norm_fusion.rs", module doc
comment) are pinned the same ways: the stored sum against a library cast
(ties included), the normalized output against library routines, a zero gate,
a closed form with silu(1), and the identity silu(t) - silu(-t) = t.
"""
import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
getcontext().prec = 50


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def f32(v) -> float:
    """The binary32 value nearest v, as a Python float (exact)."""
    return float(np.float32(v))


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).view(torch.int16).numpy()


def _dec(v) -> Decimal:
    if isinstance(v, Fraction):
        return Decimal(v.numerator) / Decimal(v.denominator)
    return Decimal(float(v))


def _close(got, want, rel, abs_=0.0, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, f"{what}: shape {got.shape} != {want.shape}"
    err = np.abs(got - want)
    bound = rel * np.abs(want) + abs_
    bad = ~(err <= bound)
    assert not bad.any(), (f"{what}: max err {float(err.max()):.3e}; first bad "
                           f"index {np.argwhere(bad)[0].tolist()}")


# --------------------------------------------------------------------------
# closed forms from the pages' worked rows


def pin_doctest_rms(orc):
    g = _golden("emily_fast_doctest_rows.json")
    x = np.array(g["x"], dtype=np.float32)
    w = np.array(g["weight"], dtype=np.float32)
    eps = g["eps"]
    ms = Fraction(*g["rms_mean_square"])
    den = (_dec(ms) + _dec(f32(eps))).sqrt()
    want = [float(_dec(v) / den * _dec(wj)) for v, wj in zip(x[0], w)]
    y = orc.rms_norm(x, w, eps)
    assert list(y.shape) == g["output_shape"]
    _close(y[0], want, 1e-15, what="doctest rms_norm")


def pin_doctest_ln(orc):
    g = _golden("emily_fast_doctest_rows.json")
    x = np.array(g["x"], dtype=np.float32)
    w = np.array(g["weight"], dtype=np.float32)
    b = np.array(g["bias"], dtype=np.float32)
    mean = Fraction(*g["ln_mean"])
    var = Fraction(*g["ln_population_variance"])
    for eps in (g["eps"], 0.0):
        den = (_dec(var) + _dec(f32(eps))).sqrt()
        want = [float((_dec(Fraction(float(v)) - mean)) / den * _dec(wj) + _dec(bj))
                for v, wj, bj in zip(x[0], w, b)]
        y = orc.layer_norm(x, w, b, eps)
        assert list(y.shape) == g["output_shape"]
        _close(y[0], want, 1e-15, what=f"doctest layer_norm eps={eps}")
    # eps = 0: the population-variance reading gives +-3/sqrt(5), +-1/sqrt(5).
    y0 = orc.layer_norm(x, w, b, 0.0)[0]
    _close(y0, [-3 / math.sqrt(5), -1 / math.sqrt(5), 1 / math.sqrt(5), 3 / math.sqrt(5)],
           1e-15, what="doctest layer_norm population variance")


def _sum_sq_run(a, n):
    """sum of k^2 for k = a .. a + n - 1 (integers), via S2(m) = m(m+1)(2m+1)/6."""
    def s2(m):
        return m * (m + 1) * (2 * m + 1) // 6
    return s2(a + n - 1) - s2(a - 1)


def _iota_rows(shape, divisor):
    n = int(np.prod(shape))
    x = (np.arange(n, dtype=np.float32) / np.float32(divisor)).reshape(-1, shape[-1])
    return x


def pin_iota_rms_exact(orc):
    """iota / 128 is exact in binary32, so the closed form is exact."""
    D = 1024
    x = _iota_rows((4, 128, D), 128.0)
    eps = 1e-6
    y = orc.rms_norm(x, None, eps)
    for r in (0, 1, 200, 511):
        a = r * D
        ms = Fraction(_sum_sq_run(a, D), 128 * 128 * D)
        den = float((_dec(ms) + _dec(f32(eps))).sqrt())
        want = ((a + np.arange(D)) / 128.0) / den
        _close(y[r], want, 4e-16, what=f"iota/128 rms row {r}")


def pin_iota_rms_page_case(orc):
    """The page's own input, iota / 100 in f32: the oracle (fed the rounded
    f32 inputs) sits within the page's round-off bound of the closed form of
    the unrounded input n / 100."""
    g = _golden("emily_iota_rms_case.json")
    D = g["shape"][-1]
    x = _iota_rows(tuple(g["shape"]), g["divisor"])
    y = orc.rms_norm(x, np.ones(D, np.float32), g["eps"])
    worst = 0.0
    for r in (0, 3, 255, 511):
        a = r * D
        ms = Fraction(_sum_sq_run(a, D), 100 * 100 * D)
        den = float((_dec(ms) + _dec(f32(g["eps"]))).sqrt())
        want = ((a + np.arange(D)) / 100.0) / den
        worst = max(worst, float(np.abs(y[r] - want).max()))
    assert worst <= g["page_bound_max_abs_diff"], worst
    assert worst <= 1e-6, worst  # what f32 input rounding alone allows


def pin_iota_ln_closed_form(orc):
    """Rows of consecutive integers / 128: mean (a + (D-1)/2) / 128 and
    population variance (D^2 - 1) / 12 / 128^2 (discrete uniform)."""
    rng = np.random.default_rng(7)
    for D in (768, 1024, 5):
        a = 1000 * D
        x = ((a + np.arange(3 * D, dtype=np.float64)) / 128.0).astype(np.float32).reshape(3, D)
        w = rng.uniform(0.5, 1.5, D).astype(np.float32)
        b = rng.uniform(-0.1, 0.1, D).astype(np.float32)
        eps = 1e-5
        y = orc.layer_norm(x, w, b, eps)
        for r in range(3):
            start = a + r * D
            mean = Fraction(2 * start + D - 1, 2 * 128)
            var = Fraction(D * D - 1, 12 * 128 * 128)
            den = (_dec(var) + _dec(f32(eps))).sqrt()
            want = [float((_dec(Fraction(start + j, 128) - mean)) / den * _dec(w[j]) + _dec(b[j]))
                    for j in range(D)]
            _close(y[r], want, 1e-14, 1e-15, what=f"iota ln D={D} row {r}")


# --------------------------------------------------------------------------
# invariants


def _rows(seed, rows, dim, dtype="f32", mean=0.0, std=1.0):
    g = torch.Generator().manual_seed(seed)
    t = torch.randn(rows, dim, generator=g) * std + mean
    if dtype == "bf16":
        return _bf16_bits(t)
    return t.numpy().astype(np.float32)


def pin_rms_unit_output_rms(orc):
    for dtype in ("f32", "bf16"):
        x = _rows(11, 16, 1000, dtype, 0.3, 2.0)
        y = orc.rms_norm(x, None, 0.0)
        _close(np.mean(y * y, axis=1), np.ones(16), 1e-14, what=f"unit rms {dtype}")
        eps = 0.5
        xv = orc.decode(x)
        ms = np.mean(xv * xv, axis=1)
        y = orc.rms_norm(x, None, eps)
        _close(np.mean(y * y, axis=1), ms / (ms + f32(eps)), 1e-13,
               what=f"rms with eps {dtype}")


def pin_ln_standardized(orc):
    for dtype in ("f32", "bf16"):
        x = _rows(12, 16, 777, dtype, 0.5, 2.0)
        y = orc.layer_norm(x, None, None, 0.0)
        assert np.all(np.abs(np.mean(y, axis=1)) <= 1e-14), "ln row mean not 0"
        _close(np.mean(y * y, axis=1), np.ones(16), 1e-13, what=f"ln unit var {dtype}")
        eps = 0.25
        xv = orc.decode(x)
        var = np.var(xv, axis=1)
        y = orc.layer_norm(x, None, None, eps)
        _close(np.mean(y * y, axis=1), var / (var + f32(eps)), 1e-13,
               what=f"ln var with eps {dtype}")


def pin_ln_constant_rows_give_bias(orc):
    for dtype in ("f32", "bf16"):
        for D in (1, 7, 4097):
            vals = _rows(13, 4, 1, dtype, 0.5, 2.0)
            x = np.repeat(vals, D, axis=1)
            w = _rows(14, 1, D, dtype, 1.0, 0.1)[0]
            b = _rows(15, 1, D, dtype, 0.0, 0.1)[0]
            y = orc.layer_norm(x, w, b, 1e-5)
            want = np.broadcast_to(orc.decode(b), y.shape)
            assert np.array_equal(y, want), f"constant rows {dtype} D={D}"


def pin_scale_invariance(orc):
    x = _rows(16, 8, 300, "bf16")
    xv = orc.decode(x)
    w = _rows(17, 1, 300, "f32", 1.0, 0.1)[0]
    b = _rows(18, 1, 300, "f32", 0.0, 0.1)[0]
    base = xv.astype(np.float32)
    # A power-of-two scale is exact through every step of the definition.
    for c in (4.0, 0.125):
        xs = (base * np.float32(c)).astype(np.float32)
        assert np.array_equal(orc.rms_norm(xs, w, 0.0), orc.rms_norm(base, w, 0.0)), c
        assert np.array_equal(orc.layer_norm(xs, w, b, 0.0),
                              orc.layer_norm(base, w, b, 0.0)), c
    # 3x of a bfloat16 value is exact in binary32; equality up to rounding.
    xs = (base * np.float32(3.0)).astype(np.float32)
    _close(orc.rms_norm(xs, w, 0.0), orc.rms_norm(base, w, 0.0), 1e-14, 1e-15, what="rms 3x")
    _close(orc.layer_norm(xs, w, b, 0.0), orc.layer_norm(base, w, b, 0.0), 1e-13, 1e-14,
           what="ln 3x")


def pin_ln_shift_invariance(orc):
    x = _rows(19, 8, 500, "bf16")
    base = orc.decode(x).astype(np.float32)
    shifted = (base + np.float32(0.5)).astype(np.float32)  # exact for these values
    assert np.array_equal(shifted.astype(np.float64) - 0.5, base.astype(np.float64))
    w = _rows(20, 1, 500, "f32", 1.0, 0.1)[0]
    b = _rows(21, 1, 500, "f32", 0.0, 0.1)[0]
    _close(orc.layer_norm(shifted, w, b, 1e-5), orc.layer_norm(base, w, b, 1e-5), 1e-12,
           1e-13, what="ln shift")


def pin_permutation_equivariance(orc):
    D = 129
    x = _rows(22, 6, D, "f32")
    w = _rows(23, 1, D, "f32", 1.0, 0.1)[0]
    b = _rows(24, 1, D, "f32", 0.0, 0.1)[0]
    perm = np.random.default_rng(25).permutation(D)
    xp = np.ascontiguousarray(x[:, perm])
    _close(orc.rms_norm(xp, w[perm], 1e-6), orc.rms_norm(x, w, 1e-6)[:, perm], 1e-14,
           what="rms perm")
    _close(orc.layer_norm(xp, w[perm], b[perm], 1e-6),
           orc.layer_norm(x, w, b, 1e-6)[:, perm], 1e-13, 1e-14, what="ln perm")


def pin_weight_and_bias_linearity(orc):
    D = 96
    x = _rows(26, 5, D, "f32")
    w = _rows(27, 1, D, "f32", 1.0, 0.5)[0]
    b = _rows(28, 1, D, "f32", 0.0, 0.5)[0]
    plain = orc.rms_norm(x, None, 1e-6)
    _close(orc.rms_norm(x, w, 1e-6), plain * w.astype(np.float64), 1e-15, what="rms w")
    plain_ln = orc.layer_norm(x, None, None, 1e-6)
    _close(orc.layer_norm(x, w, b, 1e-6),
           plain_ln * w.astype(np.float64) + b.astype(np.float64), 1e-14, 1e-15, what="ln w,b")
    ones = np.ones(D, np.float32)
    zeros = np.zeros(D, np.float32)
    assert np.array_equal(orc.layer_norm(x, ones, zeros, 1e-6), plain_ln)


def pin_one_hot_rms(orc):
    D = 64
    x = np.zeros((2, D), np.float32)
    x[0, 5] = 3.0
    x[1, 63] = -0.75
    w = _rows(29, 1, D, "f32", 1.0, 0.1)[0]
    y = orc.rms_norm(x, w, 0.0)
    want = np.zeros((2, D))
    want[0, 5] = math.sqrt(D) * w[5]
    want[1, 63] = -math.sqrt(D) * w[63]
    _close(y, want, 1e-15, what="one-hot rms")


def pin_single_column(orc):
    x = np.array([[1.5], [-2.0], [0.0]], np.float32)
    w = np.array([0.5], np.float32)
    b = np.array([0.25], np.float32)
    eps = 0.25
    want = [1.5 / math.sqrt(2.25 + eps) * 0.5, -2.0 / math.sqrt(4.0 + eps) * 0.5, 0.0]
    _close(orc.rms_norm(x, w, eps)[:, 0], want, 1e-15, what="D=1 rms")
    assert np.array_equal(orc.layer_norm(x, w, b, eps)[:, 0], [0.25, 0.25, 0.25])


def pin_eps_is_binary32(orc):
    """eps is the binary32 value nearest the decimal (it travels as f32 bits):
    with eps dominating, the f32 rounding of 0.1 is visible in the output."""
    x = np.array([[0.25]], np.float32)
    y = orc.rms_norm(x, None, 0.1)[0, 0]
    want_f32 = float(_dec(0.25) / (_dec(0.0625) + _dec(f32(0.1))).sqrt())
    want_f64 = float(_dec(0.25) / (_dec(0.0625) + _dec(0.1)).sqrt())
    assert abs(want_f32 - want_f64) > 1e-10  # the pin can tell the two apart
    _close([y], [want_f32], 1e-15, what="eps as binary32")


# --------------------------------------------------------------------------
# library routines and brute force


def pin_matches_torch_layer_norm(orc):
    g = _golden("kernel_micro_ab_layer_norm_case.json")
    gen = torch.Generator().manual_seed(31)
    shape = tuple(g["shape"])
    D = shape[-1]
    x = (torch.rand(shape, generator=gen) * 2 - 1).float()
    w = (torch.rand(D, generator=gen) + 0.5).float()
    b = (torch.rand(D, generator=gen) * 0.2 - 0.1).float()
    y = orc.layer_norm(x.numpy(), w.numpy(), b.numpy(), g["eps"])
    ref = torch.nn.functional.layer_norm(x.double(), (D,), w.double(), b.double(),
                                         f32(g["eps"])).reshape(-1, D).numpy()
    _close(y, ref, 1e-12, 1e-13, what="torch layer_norm fp64")
    assert float(np.abs(y - ref).max()) < g["page_bound_max_abs_diff"]


def pin_matches_torch_rms_norm(orc):
    for dtype in ("f32", "bf16"):
        x = _rows(32, 64, 1024, dtype, 0.0, 1.0)
        w = _rows(33, 1, 1024, dtype, 1.0, 0.1)[0]
        xv = torch.from_numpy(orc.decode(x))
        wv = torch.from_numpy(orc.decode(w))
        ref = torch.nn.functional.rms_norm(xv, (1024,), wv, f32(1e-6)).numpy()
        _close(orc.rms_norm(x, w, 1e-6), ref, 1e-13, what=f"torch rms_norm {dtype}")


def pin_brute_force_tiny_rows(orc):
    rng = np.random.default_rng(34)
    for D in (1, 2, 3, 4, 5):
        x = _bf16_bits(torch.from_numpy(rng.normal(0.2, 1.5, (6, D)).astype(np.float32)))
        w = _bf16_bits(torch.from_numpy(rng.normal(1.0, 0.2, D).astype(np.float32)))
        b = _bf16_bits(torch.from_numpy(rng.normal(0.0, 0.2, D).astype(np.float32)))
        xv, wv, bv = orc.decode(x), orc.decode(w), orc.decode(b)
        eps = 1e-3
        e = Fraction(f32(eps))
        y_rms = orc.rms_norm(x, w, eps)
        y_ln = orc.layer_norm(x, w, b, eps)
        for r in range(6):
            row = [Fraction(float(v)) for v in xv[r]]
            ms = sum(v * v for v in row) / D
            mu = sum(row) / D
            var = sum((v - mu) ** 2 for v in row) / D
            rden = _dec(ms + e).sqrt()
            lden = _dec(var + e).sqrt()
            want_r = [float(_dec(row[j]) / rden * _dec(wv[j])) for j in range(D)]
            want_l = [float(_dec(row[j] - mu) / lden * _dec(wv[j]) + _dec(bv[j]))
                      for j in range(D)]
            _close(y_rms[r], want_r, 1e-15, 1e-300, what=f"brute rms D={D}")
            _close(y_ln[r], want_l, 1e-14, 1e-15, what=f"brute ln D={D}")


def pin_dual_is_query_then_key(orc):
    q = _rows(35, 12, 128, "bf16")
    k = _rows(36, 5, 64, "bf16", 0.0, 3.0)
    wq = _rows(37, 1, 128, "bf16", 1.0, 0.1)[0]
    wk = _rows(38, 1, 64, "bf16", 1.0, 0.1)[0]
    yq, yk = orc.dual_head_rms_norm(q, k, wq, wk, 1e-6)
    for y, x, w, D in ((yq, q, wq, 128), (yk, k, wk, 64)):
        ref = torch.nn.functional.rms_norm(torch.from_numpy(orc.decode(x)), (D,),
                                           torch.from_numpy(orc.decode(w)), f32(1e-6)).numpy()
        _close(y, ref, 1e-13, what="dual vs torch rms_norm")


def pin_strided_rows(orc):
    D, pad = 100, 13
    wide = _rows(39, 7, D + pad, "f32")
    view = wide[:, :D]
    assert view.strides[0] == (D + pad) * 4
    compact = np.ascontiguousarray(view)
    w = _rows(40, 1, D, "f32", 1.0, 0.1)[0]
    assert np.array_equal(orc.rms_norm(view, w, 1e-6), orc.rms_norm(compact, w, 1e-6))
    assert np.array_equal(orc.layer_norm(view, w, w, 1e-6),
                          orc.layer_norm(compact, w, w, 1e-6))
    # and the rows really are distinct rows of the wide buffer
    _close(orc.rms_norm(view, w, 1e-6)[3],
           orc.rms_norm(compact[3:4], w, 1e-6)[0], 0.0, what="row 3")


def pin_bf16_decoding(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = orc.decode(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    f = np.random.default_rng(41).normal(0, 1e3, 1000).astype(np.float32)
    assert np.array_equal(orc.decode(f), f.astype(np.float64))


def _bits_to_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16)


def pin_add_rms_stored_sum_is_library_cast(orc):
    # bf16: h = bfloat16(float32(x) + float32(r)) by torch's cast (round to
    # nearest even), on random rows and on sums built to land exactly on a
    # bfloat16 midpoint with an even and with an odd kept bit.
    g = np.random.default_rng(71)
    x = torch.from_numpy(g.normal(0, 2, (6, 40)).astype(np.float32)).to(torch.bfloat16)
    r = torch.from_numpy(g.normal(0, 2, (6, 40)).astype(np.float32)).to(torch.bfloat16)
    # 1 + 2^-8 (tie, kept bit even -> rounds down to 1) and 1 + 3 * 2^-8
    # (tie, kept bit odd -> rounds up to 1 + 2^-6): x = 1, r = 2^-8 or 3 * 2^-8
    x[0, :4] = 1.0
    r[0, 0], r[0, 1] = 2.0 ** -8, 3 * 2.0 ** -8
    r[0, 2], r[0, 3] = -(2.0 ** -9), 2.0 ** -9 + 2.0 ** -16
    _, h = orc.add_rms_norm(_bf16_bits(x), _bf16_bits(r), None, 1e-6)
    want = (x.float() + r.float()).to(torch.bfloat16).double().numpy()
    assert np.array_equal(h, want), "stored bf16 sum != library cast"
    assert h[0, 0] == 1.0 and h[0, 1] == 1.0 + 2.0 ** -6, (h[0, 0], h[0, 1])
    # f32: h = float32 addition
    xf = g.normal(0, 3, (5, 33)).astype(np.float32)
    rf = g.normal(0, 3, (5, 33)).astype(np.float32)
    _, hf = orc.add_rms_norm(xf, rf, None, 1e-6)
    assert np.array_equal(hf, (xf + rf).astype(np.float64)), "stored f32 sum != f32 add"


def pin_add_rms_matches_torch(orc):
    for dtype in ("f32", "bf16"):
        x = _rows(72, 7, 96, dtype)
        r = _rows(73, 7, 96, dtype)
        w = _rows(74, 1, 96, dtype, mean=1.0, std=0.1).reshape(-1)
        y, h = orc.add_rms_norm(x, r, w, 1e-5)
        xt = torch.from_numpy(orc.decode(x))
        rt = torch.from_numpy(orc.decode(r))
        ht = (xt.float() + rt.float())
        if dtype == "bf16":
            ht = ht.to(torch.bfloat16)
        ht = ht.double()
        want = torch.nn.functional.rms_norm(ht, (96,), eps=f32(1e-5)) * \
            torch.from_numpy(orc.decode(w))
        _close(y, want.numpy(), 1e-12, 1e-14, f"add_rms vs torch ({dtype})")


def pin_add_rms_zero_residual(orc):
    x = _rows(75, 4, 50, "bf16")
    y, h = orc.add_rms_norm(x, np.zeros_like(x), None, 1e-6)
    xt = torch.from_numpy(orc.decode(x))
    assert np.array_equal(h, xt.numpy()), "x + 0 must store x"
    want = torch.nn.functional.rms_norm(xt, (50,), eps=f32(1e-6))
    _close(y, want.numpy(), 1e-12, 1e-14, "add_rms with r = 0")


def pin_add_rms_strided_residual(orc):
    # the residual's rows are read with the residual's own row stride
    x = _rows(85, 4, 16, "bf16")
    wide = _rows(86, 4, 27, "bf16")
    r = wide[:, 5:21]
    y, h = orc.add_rms_norm(x, r, None, 1e-6)
    xt = torch.from_numpy(orc.decode(x)).float()
    rt = torch.from_numpy(orc.decode(np.ascontiguousarray(r))).float()
    ht = (xt + rt).to(torch.bfloat16).double()
    assert np.array_equal(h, ht.numpy()), "strided residual: stored sum"
    want = torch.nn.functional.rms_norm(ht, (16,), eps=f32(1e-6))
    _close(y, want.numpy(), 1e-12, 1e-14, "add_rms strided residual")


def pin_gated_zero_gate(orc):
    x = _rows(76, 3, 24)
    y = orc.gated_rms_norm(x, np.zeros_like(x), None, 1e-6)
    assert np.all(y == 0.0), "silu(0) = 0 must zero the output"


def pin_gated_closed_form(orc):
    # "Emily.Fast" doctest row [1, 2, 3, 4], weight 1, gate 1 everywhere:
    # y_j = x_j / sqrt(15/2 + eps) * silu(1), silu(1) = 1 / (1 + e^-1).
    x = np.array([[1, 2, 3, 4]], dtype=np.float32)
    z = np.ones_like(x)
    y = orc.gated_rms_norm(x, z, None, 1e-5)
    silu1 = Decimal(1) / (Decimal(1) + (-Decimal(1)).exp())
    den = (Decimal(15) / Decimal(2) + Decimal(f32(1e-5))).sqrt()
    want = [float(Decimal(v) / den * silu1) for v in (1, 2, 3, 4)]
    _close(y[0], want, 1e-14, 0.0, "gated closed form")


def pin_gated_odd_part_is_gate(orc):
    # silu(t) - silu(-t) = t, so y(z) - y(-z) = RMSNorm(x) * w * z.
    x = _rows(77, 5, 64)
    z = _rows(78, 5, 64, std=3.0)
    w = _rows(79, 1, 64, mean=1.0, std=0.1).reshape(-1)
    d = orc.gated_rms_norm(x, z, w, 1e-6) - orc.gated_rms_norm(x, -z, w, 1e-6)
    n = torch.nn.functional.rms_norm(torch.from_numpy(x.astype(np.float64)), (64,),
                                     eps=f32(1e-6)).numpy()
    _close(d, n * w.astype(np.float64) * z.astype(np.float64), 1e-12, 1e-14,
           "gated odd part")


def pin_gated_matches_torch(orc):
    for dtype in ("f32", "bf16"):
        x = _rows(80, 6, 128, dtype)
        z = _rows(81, 6, 128, dtype, std=2.0)
        w = _rows(82, 1, 128, dtype, mean=1.0, std=0.1).reshape(-1)
        y = orc.gated_rms_norm(x, z, w, 1e-6)
        xt, zt = torch.from_numpy(orc.decode(x)), torch.from_numpy(orc.decode(z))
        want = torch.nn.functional.rms_norm(xt, (128,), eps=f32(1e-6)) * \
            torch.from_numpy(orc.decode(w)) * torch.nn.functional.silu(zt)
        _close(y, want.numpy(), 1e-12, 1e-14, f"gated vs torch ({dtype})")


def pin_gated_strided_gate(orc):
    # the gate's rows are read with the gate's own row stride
    x = _rows(83, 4, 16)
    wide = _rows(84, 4, 24, std=2.0)
    got = orc.gated_rms_norm(x, wide[:, 3:19], None, 1e-6)
    want = orc.gated_rms_norm(x, np.ascontiguousarray(wide[:, 3:19]), None, 1e-6)
    assert np.array_equal(got, want)
    xt = torch.from_numpy(x.astype(np.float64))
    zt = torch.from_numpy(np.ascontiguousarray(wide[:, 3:19]).astype(np.float64))
    ref = torch.nn.functional.rms_norm(xt, (16,), eps=f32(1e-6)) * torch.nn.functional.silu(zt)
    _close(got, ref.numpy(), 1e-12, 1e-14, "gated strided gate")


# --------------------------------------------------------------------------
# dual q/k head RMSNorm + RoPE ("Emily.Fast", rope/3 and rope_with_freqs/4)


def _rope_complex(n, pos, dims, traditional, freqs):
    """RoPE as complex multiplication: each plane (a, b) is the complex number
    a + ib times exp(i * pos * f) (numpy's complex exponential)."""
    y = n.copy()
    half = dims // 2
    for i in range(half):
        a, b = (2 * i, 2 * i + 1) if traditional else (i, i + half)
        z = (n[:, a] + 1j * n[:, b]) * np.exp(1j * pos * freqs[i])
        y[:, a], y[:, b] = z.real, z.imag
    return y


def _torch_rms(x, w, eps):
    xt = torch.from_numpy(np.asarray(x, dtype=np.float64))
    n = torch.nn.functional.rms_norm(xt, (xt.shape[-1],), eps=f32(eps)).numpy()
    return n if w is None else n * np.asarray(w, dtype=np.float64)


def pin_rope_is_complex_rotation(orc):
    # 3 tokens x 4 query heads and 2 key heads, head dim 16, partial rotary
    # (dims 12), offset 5, base 10000 (binary32), both plane layouts
    q = _rows(90, 12, 16)
    k = _rows(91, 6, 16)
    wq = _rows(92, 1, 16, mean=1.0, std=0.1).reshape(-1)
    wk = _rows(93, 1, 16, mean=1.0, std=0.1).reshape(-1)
    freqs = [f32(10000.0) ** (-2.0 * i / 12) for i in range(6)]
    for trad in (False, True):
        yq, yk = orc.dual_head_rms_norm_rope(q, k, wq, wk, 1e-6, 4, 2, 5, 12, traditional=trad)
        for y, x, w, heads in ((yq, q, wq, 4), (yk, k, wk, 2)):
            n = _torch_rms(x, w, 1e-6)
            pos = (5 + np.arange(x.shape[0]) // heads).astype(np.float64)
            want = _rope_complex(n, pos, 12, trad, freqs)
            _close(y, want, 1e-13, 1e-14, f"rope complex (traditional={trad})")


def pin_rope_page_freqs_example(orc):
    # "Emily.Fast", rope_with_freqs/4 example: x = iota {1, 1, 4, 8} (4
    # positions of one 8-wide head), offset 0, freqs [1, 0.1, 0.01, 0.001]
    x = np.arange(32, dtype=np.float32).reshape(4, 8)
    freqs = np.array([1.0, 0.1, 0.01, 0.001], dtype=np.float32)
    yq, _ = orc.dual_head_rms_norm_rope(x, x, None, None, 1e-6, 1, 1, 0, 8, inv_freq=freqs)
    n = _torch_rms(x, None, 1e-6)
    want = _rope_complex(n, np.arange(4, dtype=np.float64), 8, False,
                         [float(f) for f in freqs])
    _close(yq, want, 1e-13, 1e-14, "rope page freqs example")
    # with base 10000 and dims 8 the inverse frequencies are 1, 0.1, 0.01, 0.001
    yb, _ = orc.dual_head_rms_norm_rope(x, x, None, None, 1e-6, 1, 1, 0, 8)
    _close(yb, yq, 1e-7, 1e-9, "base 1e4 vs its frequency table")


def pin_rope_preserves_plane_norms_and_tail(orc):
    q = _rows(94, 8, 24)
    yq, _ = orc.dual_head_rms_norm_rope(q, q, None, None, 1e-6, 2, 2, 1000, 16)
    n = _torch_rms(q, None, 1e-6)
    for i in range(8):
        _close(yq[:, i] ** 2 + yq[:, i + 8] ** 2, n[:, i] ** 2 + n[:, i + 8] ** 2, 1e-13,
               1e-15, "plane norm")
    _close(yq[:, 16:], n[:, 16:], 1e-14, 1e-15, "columns past dims pass through")


def pin_rope_position_zero_is_plain_norm(orc):
    q = _rows(95, 6, 32, "bf16")
    wq = _rows(96, 1, 32, "bf16", mean=1.0, std=0.1).reshape(-1)
    yq, _ = orc.dual_head_rms_norm_rope(q, q, wq, wq, 1e-6, 6, 6, 0, 32)
    n = _torch_rms(orc.decode(q), orc.decode(wq), 1e-6)
    _close(yq, n, 1e-14, 1e-15, "token 0 at offset 0 is not rotated")
    y0, _ = orc.dual_head_rms_norm_rope(q, q, wq, wq, 1e-6, 1, 1, 77, 32, scale=0.0)
    _close(y0, n, 1e-14, 1e-15, "scale 0 does not rotate")


def pin_rope_relative_position(orc):
    # q . k after RoPE depends only on the positions' difference: shifting
    # the offset leaves every query/key dot product of a token unchanged
    q = _rows(97, 3, 16)
    k = _rows(98, 3, 16)
    dots = []
    for off in (0, 37, 4096):
        yq, yk = orc.dual_head_rms_norm_rope(q, k, None, None, 1e-6, 1, 1, off, 16)
        dots.append(yq @ yk.T)
    _close(dots[1], dots[0], 1e-11, 1e-12, "relative position (37)")
    _close(dots[2], dots[0], 1e-10, 1e-11, "relative position (4096)")


def pin_rope_layouts_are_a_column_permutation(orc):
    # interleaving the columns turns split-half planes into traditional ones
    d = 16
    perm = np.empty(d, dtype=np.int64)
    perm[0::2], perm[1::2] = np.arange(d // 2), np.arange(d // 2) + d // 2
    q = _rows(99, 5, d)
    ys, _ = orc.dual_head_rms_norm_rope(q, q, None, None, 1e-6, 1, 1, 3, d)
    yt, _ = orc.dual_head_rms_norm_rope(np.ascontiguousarray(q[:, perm]), q, None, None, 1e-6,
                                        1, 1, 3, d, traditional=True)
    _close(yt, ys[:, perm], 1e-13, 1e-15, "traditional = permuted split-half")


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
