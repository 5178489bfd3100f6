"""Parity at the full workload sizes, in the launch configuration bench.py
times (the default plan, seeded device inputs as in bench.py). The oracle
checks sampled rows one by one: the first and last rows, the constant rows
and random rows. Properties that hold at any size are checked over every
row: finite outputs, and LayerNorm constant rows returning exactly the bias.
"""
import numpy as np
import pytest
import torch

import oracle
import transformer_row_normalization_b200 as rn
from transformer_row_normalization_b200 import workloads as wl
from tolerance import check

pytestmark = pytest.mark.gpu


def sample_rows(rows, seed, extra=()):
    g = np.random.default_rng(seed)
    idx = {0, 1, rows - 2, rows - 1, *extra}
    idx.update(int(i) for i in g.choice(rows, size=96, replace=False))
    return torch.tensor(sorted(i for i in idx if 0 <= i < rows), dtype=torch.long)


@pytest.fixture(autouse=True)
def free_memory():
    yield
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", [n for n in wl.LARGE_SUITE if wl.WORKLOADS[n].op != "dual"])
def test_full_size_single(name):
    w = wl.WORKLOADS[name]
    a = wl.make_inputs(w, device="cuda")
    x = a["x"].reshape(-1, w.dim)
    plan = rn.plan(rn.RN_OP_LN if w.op == "ln" else rn.RN_OP_RMS, x, weight=a["w"],
                   bias=a.get("b"))
    assert plan["staged"] == 0  # the kernel bench.py times
    if w.op == "ln":
        y = rn.layer_norm(a["x"], a["w"], a["b"], w.eps).reshape(-1, w.dim)
    else:
        y = rn.rms_norm(a["x"], a["w"], w.eps).reshape(-1, w.dim)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y).all())
    extra = ()
    if w.op == "ln":
        const = torch.arange(0, w.rows, wl.CONSTANT_ROW_PERIOD, device="cuda")
        assert torch.equal(y[const], a["b"].expand(const.numel(), -1)), "constant rows != bias"
        extra = (64, 128, w.rows - 64)
    idx = sample_rows(w.rows, w.seed, extra)
    xs = x[idx.cuda()].cpu()
    ys = y[idx.cuda()]
    if w.op == "ln":
        ref = oracle.layer_norm(xs, a["w"].cpu(), a["b"].cpu(), w.eps)
        check(ys, ref, w.dtype, bias=a["b"], what=name)
    else:
        ref = oracle.rms_norm(xs, a["w"].cpu(), w.eps)
        check(ys, ref, w.dtype, what=name)


def test_full_size_dual_prefill():
    w = wl.WORKLOADS["dual_bf16_prefill"]
    a = wl.make_inputs(w, device="cuda")
    yq, yk = rn.dual_head_rms_norm(a["q"], a["k"], a["wq"], a["wk"], w.eps)
    torch.cuda.synchronize()
    q, k = a["q"].reshape(-1, 128), a["k"].reshape(-1, 128)
    yq, yk = yq.reshape(-1, 128), yk.reshape(-1, 128)
    assert bool(torch.isfinite(yq).all()) and bool(torch.isfinite(yk).all())
    iq = sample_rows(q.shape[0], 3).cuda()
    ik = sample_rows(k.shape[0], 4).cuda()
    rq, rk = oracle.dual_head_rms_norm(q[iq].cpu(), k[ik].cpu(), a["wq"].cpu(), a["wk"].cpu(),
                                       w.eps)
    check(yq[iq], rq, w.dtype, what="prefill q")
    check(yk[ik], rk, w.dtype, what="prefill k")
    # the one launch equals two single calls, bit for bit, at full size
    assert torch.equal(yq, rn.rms_norm(q, a["wq"], w.eps))
    assert torch.equal(yk, rn.rms_norm(k, a["wk"], w.eps))
