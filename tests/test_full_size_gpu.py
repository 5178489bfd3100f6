"""Parity at the full workload sizes, in the launch configuration bench.py
times (the default plan, seeded device inputs as in bench.py). Every row of
every output is compared element by element with the fp64 oracle (in row
chunks on the host cores; see fullsize.py). LayerNorm's constant rows must
also return exactly the bias, and the dual launch must equal two single
calls bit for bit.
"""
import pytest
import torch

import oracle
import transformer_row_normalization_b200 as rn
from fullsize import as_bf16, each_chunk, host
from tolerance import check
from transformer_row_normalization_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def free_memory():
    yield
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", [n for n in wl.LARGE_SUITE if wl.WORKLOADS[n].op != "dual"])
def test_full_size_single(name):
    w = wl.WORKLOADS[name]
    a = wl.make_inputs(w, device="cuda")
    x = a["x"].reshape(-1, w.dim)
    # the default plan: the kernel bench.py times
    plan = rn.plan(rn.RN_OP_LN if w.op == "ln" else rn.RN_OP_RMS, x, weight=a["w"],
                   bias=a.get("b"))
    # rings by default: warp rings for rows one warp's lanes share (768,
    # 1000), block rings for blocks of 512+ threads (16384)
    assert plan["staged"] == (1 if w.dim in (768, 1000, 16384) else 0), plan
    if w.op == "ln":
        y = rn.layer_norm(a["x"], a["w"], a["b"], w.eps).reshape(-1, w.dim)
    else:
        y = rn.rms_norm(a["x"], a["w"], w.eps).reshape(-1, w.dim)
    torch.cuda.synchronize()
    if w.op == "ln":
        const = torch.arange(0, w.rows, wl.CONSTANT_ROW_PERIOD, device="cuda")
        assert torch.equal(y[const], a["b"].expand(const.numel(), -1)), "constant rows != bias"
    hx, hy = host(x), as_bf16(host(y))
    hw = host(a["w"])
    hb = host(a["b"]) if w.op == "ln" else None
    del y, x, a
    torch.cuda.empty_cache()

    def part(r0, r1):
        if w.op == "ln":
            ref = oracle.layer_norm(hx[r0:r1], hw, hb, w.eps)
            check(hy[r0:r1], ref, w.dtype, bias=as_bf16(hb), what=f"{name} rows {r0}:{r1}")
        else:
            ref = oracle.rms_norm(hx[r0:r1], hw, w.eps)
            check(hy[r0:r1], ref, w.dtype, what=f"{name} rows {r0}:{r1}")

    assert each_chunk(w.rows, w.dim, part) == w.rows


def test_full_size_dual_prefill():
    w = wl.WORKLOADS["dual_bf16_prefill"]
    a = wl.make_inputs(w, device="cuda")
    yq, yk = rn.dual_head_rms_norm(a["q"], a["k"], a["wq"], a["wk"], w.eps)
    torch.cuda.synchronize()
    q, k = a["q"].reshape(-1, 128), a["k"].reshape(-1, 128)
    yq, yk = yq.reshape(-1, 128), yk.reshape(-1, 128)
    # the one launch equals two single calls, bit for bit, at full size
    assert torch.equal(yq, rn.rms_norm(q, a["wq"], w.eps))
    assert torch.equal(yk, rn.rms_norm(k, a["wk"], w.eps))
    hq, hk, hyq, hyk = host(q), host(k), as_bf16(host(yq)), as_bf16(host(yk))
    hwq, hwk = host(a["wq"]), host(a["wk"])

    def part_q(r0, r1):
        ref, _ = oracle.dual_head_rms_norm(hq[r0:r1], hk[:1], hwq, hwk, w.eps)
        check(hyq[r0:r1], ref, w.dtype, what=f"prefill q rows {r0}:{r1}")

    def part_k(r0, r1):
        _, ref = oracle.dual_head_rms_norm(hq[:1], hk[r0:r1], hwq, hwk, w.eps)
        check(hyk[r0:r1], ref, w.dtype, what=f"prefill k rows {r0}:{r1}")

    assert each_chunk(hq.shape[0], 128, part_q) == 8192 * 32
    assert each_chunk(hk.shape[0], 128, part_k) == 8192 * 8
