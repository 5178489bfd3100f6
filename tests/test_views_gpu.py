"""Head rows in blocks: the query and key heads sliced out of a packed QKV
buffer ("kernel_micro_ab.rs", section 2: the packed QKV op writes the head
buffers), normalized in place or into fresh outputs, with the rest of the
buffer untouched. Parity with the fp64 oracle on contiguous copies, and bits
equal to the same call on contiguous copies."""
import pytest
import torch

import oracle
import transformer_row_normalization_b200 as rn
from transformer_row_normalization_b200 import workloads as wl
from tolerance import check

pytestmark = pytest.mark.gpu


def packed_qkv(tokens, hq, hk, d, dtype, seed, pad=0):
    """[tokens, (hq + 2 hk) * d + pad] buffer and its q, k, v head views."""
    width = (hq + 2 * hk) * d + pad
    buf = wl.random_rows(tokens, width, dtype, seed=seed).cuda()
    q = buf[:, :hq * d].view(tokens, hq, d)
    k = buf[:, hq * d:(hq + hk) * d].view(tokens, hk, d)
    v = buf[:, (hq + hk) * d:(hq + 2 * hk) * d].view(tokens, hk, d)
    return buf, q, k, v


def host_rows(t):
    return t.detach().cpu().contiguous().reshape(-1, t.shape[-1])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("tokens,hq,hk,d", [(7, 32, 8, 128), (1, 16, 4, 64), (33, 4, 2, 100),
                                            (5, 8, 8, 256)])
def test_dual_head_norm_on_a_packed_buffer(dtype, tokens, hq, hk, d):
    buf, q, k, v = packed_qkv(tokens, hq, hk, d, dtype, seed=tokens + d)
    if tokens > 1:  # one token folds into a single row stride
        assert rn.view_layout(q.shape, q.stride())[3] == hq  # really blocks of rows
    wq = wl.random_vector(d, dtype, seed=1).cuda()
    wk = wl.random_vector(d, dtype, seed=2).cuda()
    ref_q, ref_k = oracle.dual_head_rms_norm(host_rows(q), host_rows(k), wq.cpu(), wk.cpu(), 1e-6)
    # into fresh outputs, and equal to the call on contiguous copies
    yq, yk = rn.dual_head_rms_norm(q, k, wq, wk, 1e-6)
    cq, ck = rn.dual_head_rms_norm(q.contiguous(), k.contiguous(), wq, wk, 1e-6)
    torch.cuda.synchronize()
    check(yq.reshape(-1, d), ref_q, dtype, what="q")
    check(yk.reshape(-1, d), ref_k, dtype, what="k")
    assert torch.equal(yq, cq) and torch.equal(yk, ck)
    # in place: q and k overwritten inside the buffer, v untouched
    v_before = v.clone()
    rn.dual_head_rms_norm(q, k, wq, wk, 1e-6, out_q=q, out_k=k)
    torch.cuda.synchronize()
    assert torch.equal(q, cq) and torch.equal(k, ck) and torch.equal(v, v_before)


def test_rope_on_a_packed_buffer_in_place():
    dtype, tokens, hq, hk, d = torch.bfloat16, 9, 32, 8, 128
    buf, q, k, v = packed_qkv(tokens, hq, hk, d, dtype, seed=5)
    wq = wl.random_vector(d, dtype, seed=3).cuda()
    wk = wl.random_vector(d, dtype, seed=4).cuda()
    table = rn.rope_table(d, 64, device="cuda")
    ref_q, ref_k = oracle.dual_head_rms_norm_rope(host_rows(q), host_rows(k), wq.cpu(), wk.cpu(),
                                                  1e-6, hq, hk, 11, d)
    cq, ck = rn.dual_head_rms_norm_rope(q.contiguous(), k.contiguous(), wq, wk, 1e-6, table, 11, d)
    v_before = v.clone()
    rn.dual_head_rms_norm_rope(q, k, wq, wk, 1e-6, table, 11, d, out_q=q, out_k=k)
    torch.cuda.synchronize()
    check(q.reshape(-1, d), ref_q, dtype, what="q", rope=(d, False))
    check(k.reshape(-1, d), ref_k, dtype, what="k", rope=(d, False))
    assert torch.equal(q, cq) and torch.equal(k, ck) and torch.equal(v, v_before)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("d,pad", [(128, 0), (128, 3), (1000, 1), (4096, 0), (4097, 5)])
def test_single_ops_on_head_slices(dtype, d, pad):
    # blocks whose start phase moves from token to token (pad) and widths on
    # both kernel families
    buf, q, k, _ = packed_qkv(6, 4, 2, d, dtype, seed=d + pad, pad=pad)
    w = wl.random_vector(d, dtype, seed=7).cuda()
    b = wl.random_vector(d, dtype, seed=8, mean=0.0, std=0.1).cuda()
    y = rn.rms_norm(q, w, 1e-6)
    check(y.reshape(-1, d), oracle.rms_norm(host_rows(q), w.cpu(), 1e-6), dtype, what="rms")
    y = rn.layer_norm(q, w, b, 1e-5)
    check(y.reshape(-1, d), oracle.layer_norm(host_rows(q), w.cpu(), b.cpu(), 1e-5), dtype,
          bias=b, what="ln")
    # outputs with their own block layout: a second packed buffer
    out_buf, oq, _, _ = packed_qkv(6, 4, 2, d, dtype, seed=99, pad=pad)
    rest = out_buf[:, 4 * d:].clone()
    rn.layer_norm(q, w, b, 1e-5, out=oq)
    torch.cuda.synchronize()
    assert torch.equal(oq, y) and torch.equal(out_buf[:, 4 * d:], rest)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_fused_ops_on_head_slices(dtype):
    d = 128
    buf, q, k, v = packed_qkv(10, 8, 4, d, dtype, seed=21)
    rbuf, rq, _, _ = packed_qkv(10, 8, 4, d, dtype, seed=22)
    w = wl.random_vector(d, dtype, seed=23).cuda()
    y, h = rn.add_rms_norm(q, rq, w, 1e-6)
    ref_y, ref_h = oracle.add_rms_norm(host_rows(q), host_rows(rq), w.cpu(), 1e-6)
    check(y.reshape(-1, d), ref_y, dtype, what="add y")
    assert torch.equal(h.reshape(-1, d).double().cpu(), torch.from_numpy(ref_h))
    # the stored sum written back over the residual slice (in-place stream)
    rest = rbuf[:, 8 * d:].clone()
    rn.add_rms_norm(q, rq, w, 1e-6, out_h=rq)
    torch.cuda.synchronize()
    assert torch.equal(rq, h) and torch.equal(rbuf[:, 8 * d:], rest)
    g = rn.gated_rms_norm(q, k.repeat_interleave(2, dim=1), w, 1e-6)
    ref = oracle.gated_rms_norm(host_rows(q), host_rows(k.repeat_interleave(2, dim=1)), w.cpu(),
                                1e-6)
    check(g.reshape(-1, d), ref, dtype, what="gated", scaled=True)
