"""Seeded synthetic workloads for row normalization.

This module holds the input recipes shared by the tests and the benchmark:
shapes, value distributions, seeds. It contains none of the normalization
arithmetic. Values are drawn in float32 with a seeded ``torch.Generator`` on
the requested device (CPU: Mersenne Twister; CUDA: Philox) and rounded to
bfloat16 with round-to-nearest-even where the workload is bfloat16. Parity
checks always hand the oracle the exact bytes that the GPU reads, so the two
generators never need to agree with each other.

Workloads (shapes follow the pages' examples):
  rms_f32_4x128x1024      RMSNorm f32; the batch=4, seq=128, hidden=1024
                          block of "Fused transformer kernels on Emily",
                          Part 1, Correctness; values U(-1,1), w U(0.5,1.5).
  ln_f32_1x1024x768       LayerNorm f32; the (1, 1024, 768) tower shape of
                          "kernel_micro_ab.rs", section 1 (LayerNorm); x
                          U(-1,1), w U(0.5,1.5), b U(-0.1,0.1), eps 1e-6.
  dual_bf16_prefill       q [8192, 32, 128], k [8192, 8, 128] N(0,1),
                          wq, wk N(1, 0.1) -- the query/key head norms of
                          "norm_fusion.rs" at a prefill token count.
  dual_bf16_decode        the same heads at one token (decode).
  rms_bf16_16x4096x4096   RMSNorm bf16, N(0,1) with 1 % of entries x50.
  ln_bf16_65536x{D}       LayerNorm bf16, N(0.5, 2), every 64th row constant.

Fused extensions (the elementwise fusions of "norm_fusion.rs", module doc
comment), at the shapes of the rows they fuse with:
  add_rms_bf16_16x4096x4096   residual add + RMSNorm at the hidden-state shape
                              above: x, residual N(0,1), w N(1, 0.1).
  gated_rms_bf16_8192x32x128  gated output RMSNorm over 128-wide heads at the
                              prefill token count: x, z N(0,1), w N(1, 0.1).
  add_rms_f32_4x128x1024,     the same two ops at the small f32 shape of the
  gated_rms_f32_4x128x1024    Part 1 Correctness cell (x, r/z U(-1,1)).
  dual_rope_bf16_prefill      the dual q/k head norm followed by RoPE
                              ("Emily.Fast", rope/3): the prefill heads above,
                              positions 0..8191, base 10000, all 128 columns
                              rotated, split-half planes.
  ln_bf16_8192x65536,         rows wider than the register kernels hold
  rms_bf16_8192x65536         (streamed): the LayerNorm width sweep's recipe
                              (N(0.5, 2), every 64th row constant) and the
                              RMSNorm recipe (N(0,1)), 1 GB each way.
"""
from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import torch

LN_WIDTHS = (768, 1000, 4097, 8192, 16384)
CONSTANT_ROW_PERIOD = 64


@dataclass(frozen=True)
class Workload:
    name: str
    op: str                      # "rms", "ln", "dual", "dual_rope", "add_rms", "gated_rms"
    dtype: torch.dtype
    shape: Tuple[int, ...]       # x (or q) shape; last axis is the row
    eps: float
    seed: int
    k_shape: Optional[Tuple[int, ...]] = None
    meta: Dict[str, float] = field(default_factory=dict)

    @property
    def dim(self) -> int:
        return self.shape[-1]

    @property
    def rows(self) -> int:
        n = 1
        for s in self.shape[:-1]:
            n *= s
        return n

    @property
    def k_rows(self) -> int:
        if self.k_shape is None:
            return 0
        n = 1
        for s in self.k_shape[:-1]:
            n *= s
        return n

    @property
    def total_rows(self) -> int:
        return self.rows + self.k_rows

    @property
    def element_size(self) -> int:
        return torch.empty((), dtype=self.dtype).element_size()

    def algorithmic_bytes(self) -> int:
        """Read x + write y + read each per-column vector once."""
        s = self.element_size
        if self.op in ("dual", "dual_rope"):
            kd = self.k_shape[-1]
            b = (2 * self.rows * self.dim * s + self.dim * s
                 + 2 * self.k_rows * kd * s + kd * s)
            if self.op == "dual_rope":  # the cos/sin rows of the positions used
                b += self.shape[0] * self.meta["rope_dims"] * 4
            return b
        if self.op == "add_rms":   # read x, r; write y, h
            return 4 * self.rows * self.dim * s + self.dim * s
        if self.op == "gated_rms":  # read x, z; write y
            return 3 * self.rows * self.dim * s + self.dim * s
        vectors = 2 if self.op == "ln" else 1
        return 2 * self.rows * self.dim * s + vectors * self.dim * s


WORKLOADS: Dict[str, Workload] = {}


def _register(w: Workload) -> Workload:
    WORKLOADS[w.name] = w
    return w


_register(Workload("rms_f32_4x128x1024", "rms", torch.float32, (4, 128, 1024), 1e-6, 1))
_register(Workload("ln_f32_1x1024x768", "ln", torch.float32, (1, 1024, 768), 1e-6, 2))
_register(Workload("dual_bf16_prefill", "dual", torch.bfloat16, (8192, 32, 128), 1e-6, 3,
                   k_shape=(8192, 8, 128)))
_register(Workload("dual_bf16_decode", "dual", torch.bfloat16, (1, 32, 128), 1e-6, 30,
                   k_shape=(1, 8, 128)))
_register(Workload("rms_bf16_16x4096x4096", "rms", torch.bfloat16, (16, 4096, 4096), 1e-5, 4))
for _k, _d in enumerate(LN_WIDTHS):
    _register(Workload(f"ln_bf16_65536x{_d}", "ln", torch.bfloat16, (65536, _d), 1e-5, 50 + _k))

_register(Workload("add_rms_bf16_16x4096x4096", "add_rms", torch.bfloat16, (16, 4096, 4096),
                   1e-5, 60))
_register(Workload("gated_rms_bf16_8192x32x128", "gated_rms", torch.bfloat16, (8192, 32, 128),
                   1e-6, 61))
_register(Workload("dual_rope_bf16_prefill", "dual_rope", torch.bfloat16, (8192, 32, 128), 1e-6,
                   64, k_shape=(8192, 8, 128), meta={"rope_dims": 128, "rope_base": 10000.0}))
_register(Workload("add_rms_f32_4x128x1024", "add_rms", torch.float32, (4, 128, 1024), 1e-6, 62))
_register(Workload("gated_rms_f32_4x128x1024", "gated_rms", torch.float32, (4, 128, 1024),
                   1e-6, 63))

# The large bf16 workloads: one pass over each is one benchmark step.
LARGE_SUITE = ("dual_bf16_prefill", "rms_bf16_16x4096x4096") + tuple(
    f"ln_bf16_65536x{d}" for d in LN_WIDTHS)
SMALL_SUITE = ("rms_f32_4x128x1024", "ln_f32_1x1024x768", "dual_bf16_decode")
# The fused extensions, measured beside (not inside) the benchmark step.
_register(Workload("ln_bf16_8192x65536", "ln", torch.bfloat16, (8192, 65536), 1e-5, 65))
_register(Workload("rms_bf16_8192x65536", "rms", torch.bfloat16, (8192, 65536), 1e-5, 66))
FUSED_SUITE = ("add_rms_bf16_16x4096x4096", "gated_rms_bf16_8192x32x128",
               "dual_rope_bf16_prefill", "ln_bf16_8192x65536", "rms_bf16_8192x65536")


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _uniform(shape, lo, hi, g, device):
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo


def _normal(shape, mean, std, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std + mean


def make_inputs(w: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    """Draw the workload's tensors on ``device`` (a fixed draw order per
    workload: x, then the per-column vectors, then masks/constants)."""
    device = torch.device(device)
    g = _gen(device, w.seed)
    out: Dict[str, torch.Tensor] = {}
    if w.name in ("rms_f32_4x128x1024",):
        out["x"] = _uniform(w.shape, -1.0, 1.0, g, device)
        out["w"] = _uniform((w.dim,), 0.5, 1.5, g, device)
    elif w.name == "ln_f32_1x1024x768":
        out["x"] = _uniform(w.shape, -1.0, 1.0, g, device)
        out["w"] = _uniform((w.dim,), 0.5, 1.5, g, device)
        out["b"] = _uniform((w.dim,), -0.1, 0.1, g, device)
    elif w.op in ("dual", "dual_rope"):
        out["q"] = _normal(w.shape, 0.0, 1.0, g, device)
        out["k"] = _normal(w.k_shape, 0.0, 1.0, g, device)
        out["wq"] = _normal((w.dim,), 1.0, 0.1, g, device)
        out["wk"] = _normal((w.k_shape[-1],), 1.0, 0.1, g, device)
    elif w.name == "rms_bf16_16x4096x4096":
        x = _normal(w.shape, 0.0, 1.0, g, device)
        out["w"] = _normal((w.dim,), 1.0, 0.1, g, device)
        outliers = torch.rand(w.shape, generator=g, device=device) < 0.01
        out["x"] = torch.where(outliers, x * 50.0, x)
    elif w.name.startswith("ln_bf16_65536x") or w.name == "ln_bf16_8192x65536":
        x = _normal(w.shape, 0.5, 2.0, g, device)
        out["w"] = _normal((w.dim,), 1.0, 0.1, g, device)
        out["b"] = _normal((w.dim,), 0.0, 0.1, g, device)
        const_rows = torch.arange(0, w.rows, CONSTANT_ROW_PERIOD, device=device)
        values = _normal((const_rows.numel(), 1), 0.5, 2.0, g, device)
        x[const_rows] = values.expand(-1, w.dim)
        out["x"] = x
    elif w.name == "rms_bf16_8192x65536":
        out["x"] = _normal(w.shape, 0.0, 1.0, g, device)
        out["w"] = _normal((w.dim,), 1.0, 0.1, g, device)
    elif w.op in ("add_rms", "gated_rms") and w.dtype == torch.float32:
        second = "r" if w.op == "add_rms" else "z"
        out["x"] = _uniform(w.shape, -1.0, 1.0, g, device)
        out[second] = _uniform(w.shape, -1.0, 1.0, g, device)
        out["w"] = _uniform((w.dim,), 0.5, 1.5, g, device)
    elif w.op in ("add_rms", "gated_rms"):
        second = "r" if w.op == "add_rms" else "z"
        out["x"] = _normal(w.shape, 0.0, 1.0, g, device)
        out[second] = _normal(w.shape, 0.0, 1.0, g, device)
        out["w"] = _normal((w.dim,), 1.0, 0.1, g, device)
    else:
        raise KeyError(w.name)
    return {k: v.to(w.dtype) for k, v in out.items()}


def random_rows(rows, dim, dtype, seed, device="cpu", mean=0.0, std=1.0):
    """Generic N(mean, std) rows for edge-case tests, rounded to ``dtype``."""
    g = _gen(torch.device(device), seed)
    return _normal((rows, dim), mean, std, g, device).to(dtype)


def random_vector(dim, dtype, seed, device="cpu", mean=1.0, std=0.1):
    g = _gen(torch.device(device), seed)
    return _normal((dim,), mean, std, g, device).to(dtype)
