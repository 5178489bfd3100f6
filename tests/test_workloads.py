"""The seeded workload recipes (CPU): shapes, dtypes, determinism and the
structural features each recipe promises (outliers, constant rows)."""
import torch

from transformer_row_normalization_b200 import workloads as wl


def test_registry_covers_every_config():
    names = set(wl.WORKLOADS)
    assert set(wl.LARGE_SUITE) <= names and set(wl.SMALL_SUITE) <= names
    assert {f"ln_bf16_65536x{d}" for d in (768, 1000, 4097, 8192, 16384)} <= names


def test_algorithmic_bytes():
    w = wl.WORKLOADS["rms_bf16_16x4096x4096"]
    assert w.algorithmic_bytes() == 2 * 65536 * 4096 * 2 + 4096 * 2 == 1_073_750_016
    w = wl.WORKLOADS["ln_bf16_65536x4097"]
    assert w.algorithmic_bytes() == 1_074_020_356
    w = wl.WORKLOADS["dual_bf16_prefill"]
    assert w.total_rows == 262144 + 65536
    assert w.algorithmic_bytes() == 167_772_672
    assert wl.WORKLOADS["dual_bf16_decode"].algorithmic_bytes() == 20_992
    assert wl.WORKLOADS["rms_f32_4x128x1024"].algorithmic_bytes() == 4_198_400
    assert wl.WORKLOADS["ln_f32_1x1024x768"].algorithmic_bytes() == 6_297_600


def test_small_inputs_are_deterministic_and_shaped():
    for name in wl.SMALL_SUITE:
        w = wl.WORKLOADS[name]
        a = wl.make_inputs(w)
        b = wl.make_inputs(w)
        for k in a:
            assert a[k].dtype == w.dtype
            assert torch.equal(a[k], b[k])
        x = a["q"] if w.op == "dual" else a["x"]
        assert tuple(x.shape) == w.shape


def test_uniform_ranges():
    a = wl.make_inputs(wl.WORKLOADS["ln_f32_1x1024x768"])
    assert a["x"].min() >= -1 and a["x"].max() <= 1
    assert a["w"].min() >= 0.5 and a["w"].max() <= 1.5
    assert a["b"].abs().max() <= 0.1


def test_outlier_and_constant_row_recipes_small_copy():
    # The same recipes at a reduced row count keep their structure.
    w = wl.Workload("ln_bf16_65536x1000", "ln", torch.bfloat16, (256, 1000), 1e-5, 52)
    a = wl.make_inputs(w)
    x = a["x"].float()
    const = x[:: wl.CONSTANT_ROW_PERIOD]
    assert torch.all(const == const[:, :1])
    assert x[1].unique().numel() > 100
    w = wl.Workload("rms_bf16_16x4096x4096", "rms", torch.bfloat16, (4, 64, 4096), 1e-5, 4)
    x = wl.make_inputs(w)["x"].float()
    frac = (x.abs() > 6).float().mean().item()
    assert 0.004 < frac < 0.02
