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
