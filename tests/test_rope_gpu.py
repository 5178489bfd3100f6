"""Parity of the dual q/k head RMSNorm + RoPE ("Emily.Fast", rope/3 and
rope_with_freqs/4, after the dual head norm of "norm_fusion.rs") with the fp64
oracle, through the C ABI: plane layouts, partial rotary, offsets, decode,
frequency tables, misaligned views, every token at full size; and its bits against the
unrotated dual head norm where the rotation is the identity."""
import numpy as np
import pytest
import torch

import oracle
import transformer_row_normalization_b200 as rn
from transformer_row_normalization_b200 import workloads as wl
from fullsize import each_chunk
from tolerance import check, guarded_empty

pytestmark = pytest.mark.gpu


def host(t):
    return t.detach().cpu()


def inputs(tokens, hq, hk, d, dtype, seed, dk=None):
    dk = d if dk is None else dk
    q = wl.random_rows(tokens * hq, d, dtype, seed=seed).cuda()
    k = wl.random_rows(tokens * hk, dk, dtype, seed=seed + 1).cuda()
    wq = wl.random_vector(d, dtype, seed=seed + 2).cuda()
    wk = wl.random_vector(dk, dtype, seed=seed + 3).cuda()
    return q, k, wq, wk


def run(q, k, wq, wk, table, offset, dims, hq, hk, trad):
    yq, _, gq = guarded_empty(tuple(q.shape), q.dtype)
    yk, _, gk = guarded_empty(tuple(k.shape), k.dtype)
    rn.dual_head_rms_norm_rope(q, k, wq, wk, 1e-6, table, offset, dims, heads_q=hq, heads_k=hk,
                               traditional=trad, out_q=yq, out_k=yk)
    torch.cuda.synchronize()
    gq(), gk()
    return yq, yk


def check_both(q, k, wq, wk, yq, yk, offset, dims, hq, hk, trad, what, **rope_kw):
    rq, rk = oracle.dual_head_rms_norm_rope(host(q), host(k), host(wq), host(wk), 1e-6, hq, hk,
                                            offset, dims, traditional=trad, **rope_kw)
    check(yq, rq, q.dtype, what=f"{what} q", rope=(dims, trad))
    check(yk, rk, k.dtype, what=f"{what} k", rope=(dims, trad))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("trad", [False, True], ids=["split", "interleaved"])
@pytest.mark.parametrize("tokens,offset", [(1, 0), (1, 4095), (3, 5), (64, 0), (64, 3000)])
def test_prefill_and_decode_heads(dtype, trad, tokens, offset):
    q, k, wq, wk = inputs(tokens, 32, 8, 128, dtype, seed=10 + tokens)
    table = rn.rope_table(128, 8192, device="cuda")
    yq, yk = run(q, k, wq, wk, table, offset, 128, 32, 8, trad)
    check_both(q, k, wq, wk, yq, yk, offset, 128, 32, 8, trad, f"T={tokens} off={offset}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("d,dims", [(128, 64), (64, 64), (80, 32), (256, 256), (1024, 96),
                                    (8, 8), (6, 4), (100, 100)])
def test_head_dims_and_partial_rotary(dtype, d, dims):
    q, k, wq, wk = inputs(9, 4, 2, d, dtype, seed=d + dims)
    table = rn.rope_table(dims, 64, base=500000.0, device="cuda")
    for trad in (False, True):
        yq, yk = run(q, k, wq, wk, table, 7, dims, 4, 2, trad)
        check_both(q, k, wq, wk, yq, yk, 7, dims, 4, 2, trad, f"D={d} dims={dims}",
                   base=500000.0)


def test_unequal_head_dims_and_frequency_table():
    # rope_with_freqs/4: a caller's inverse-frequency table (here a linear
    # scaling of the base schedule), q and k of different widths
    dims = 64
    freqs = (10000.0 ** (-np.arange(0, dims, 2) / dims) / 4.0).astype(np.float32)
    q, k, wq, wk = inputs(17, 6, 2, 128, torch.bfloat16, seed=77, dk=64)
    table = rn.rope_table(dims, 4096, inv_freq=freqs, scale=0.5, device="cuda")
    yq, yk = run(q, k, wq, wk, table, 1000, dims, 6, 2, False)
    check_both(q, k, wq, wk, yq, yk, 1000, dims, 6, 2, False, "freqs", inv_freq=freqs,
               scale=0.5)


def test_misaligned_head_rows():
    # q rows start one element into wider rows: edge elements and the
    # realigned weight cache take part in the rotation
    b = wl.random_rows(5 * 8, 131, torch.bfloat16, seed=91).cuda()
    q = b[:, 1:129]
    _, k, wq, wk = inputs(5, 8, 2, 128, torch.bfloat16, seed=92)
    table = rn.rope_table(128, 16, device="cuda")
    for trad in (False, True):
        yq, yk = run(q, k, wq, wk, table, 2, 128, 8, 2, trad)
        check_both(q, k, wq, wk, yq, yk, 2, 128, 8, 2, trad, "misaligned q")


def test_identity_rotation_matches_the_dual_head_norm():
    # dims 0 rotates nothing, and token 0 at position 0 rotates by angle 0:
    # both must give the bits of the plain dual head norm
    q, k, wq, wk = inputs(12, 4, 2, 128, torch.bfloat16, seed=33)
    pq, pk = rn.dual_head_rms_norm(q, k, wq, wk, 1e-6)
    empty = torch.empty((16, 0), dtype=torch.float32, device="cuda")
    yq, yk = rn.dual_head_rms_norm_rope(q, k, wq, wk, 1e-6, empty, 0, 0, heads_q=4, heads_k=2)
    assert torch.equal(yq, pq) and torch.equal(yk, pk)
    table = rn.rope_table(128, 16, device="cuda")
    yq, yk = rn.dual_head_rms_norm_rope(q, k, wq, wk, 1e-6, table, 0, 128, heads_q=4, heads_k=2)
    assert torch.equal(yq[:4], pq[:4]) and torch.equal(yk[:2], pk[:2])


def test_full_size_prefill():
    """Every token of the 8192-token prefill (all its 32 query and 8 key
    heads) against the oracle, in chunks of whole tokens at their positions."""
    w = wl.WORKLOADS["dual_rope_bf16_prefill"]
    a = wl.make_inputs(w, device="cuda")
    table = rn.rope_table(128, 8192, base=w.meta["rope_base"], device="cuda")
    yq, yk = rn.dual_head_rms_norm_rope(a["q"], a["k"], a["wq"], a["wk"], w.eps, table, 0, 128)
    torch.cuda.synchronize()
    q, k = a["q"].reshape(-1, 128), a["k"].reshape(-1, 128)
    hq, hk, hwq, hwk = host(q), host(k), host(a["wq"]), host(a["wk"])
    hyq, hyk = host(yq.reshape(-1, 128)), host(yk.reshape(-1, 128))

    def part(t0, t1):
        rq, rk = oracle.dual_head_rms_norm_rope(hq[t0 * 32:t1 * 32], hk[t0 * 8:t1 * 8], hwq, hwk,
                                                w.eps, 32, 8, t0, 128)
        check(hyq[t0 * 32:t1 * 32], rq, w.dtype, what=f"tokens {t0}:{t1} q", rope=(128, False))
        check(hyk[t0 * 8:t1 * 8], rk, w.dtype, what=f"tokens {t0}:{t1} k", rope=(128, False))

    # a token is 40 head rows of 128 columns
    assert each_chunk(8192, 40 * 128, part) == 8192


def test_bitwise_repeatable_across_grids():
    q, k, wq, wk = inputs(300, 8, 2, 128, torch.bfloat16, seed=55)
    table = rn.rope_table(128, 512, device="cuda")
    base = rn.dual_head_rms_norm_rope(q, k, wq, wk, 1e-6, table, 9, 128, heads_q=8, heads_k=2)
    try:
        for grid in (1, 7, 148, 444):
            rn.set_grid_override(grid)
            y = rn.dual_head_rms_norm_rope(q, k, wq, wk, 1e-6, table, 9, 128, heads_q=8,
                                           heads_k=2)
            assert torch.equal(y[0], base[0]) and torch.equal(y[1], base[1]), grid
    finally:
        rn.set_grid_override(0)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("trad", [False, True], ids=["split", "interleaved"])
@pytest.mark.parametrize("tokens,hq,hk,offset", [(1, 32, 8, 0), (3, 32, 8, 7), (301, 32, 8, 100),
                                                 (64, 8, 2, 5), (17, 16, 4, 0)])
def test_ring_and_register_rope_agree_bitwise(dtype, trad, tokens, hq, hk, offset):
    """The bulk-copy rings (table row staged with tiles of whole lane-group
    rounds inside one token where the head counts allow it, else read from
    global memory) give the register kernels' bits."""
    q, k, wq, wk = inputs(tokens, hq, hk, 128, dtype, seed=tokens + hq)
    table = rn.rope_table(128, offset + tokens + 1, device="cuda")
    res = {}
    try:
        for path in (1, 2):
            rn.set_path_override(path)
            res[path] = rn.dual_head_rms_norm_rope(q, k, wq, wk, 1e-6, table, offset, 128,
                                                   heads_q=hq, heads_k=hk, traditional=trad)
    finally:
        rn.set_path_override(0)
    assert torch.equal(res[1][0], res[2][0]) and torch.equal(res[1][1], res[2][1])
    assert rn.device_error_count(reset=True) == 0
