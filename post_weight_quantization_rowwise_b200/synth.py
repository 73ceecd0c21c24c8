"""Seeded synthetic inputs for the weighted-quantization path.

This module only draws random numbers: it holds none of the quantizer's
arithmetic, and both the CUDA path and the CPU oracle take their inputs from
it.  Every draw uses a ``torch.Generator`` seeded explicitly, on the device
the caller names; the same (seed, device) always gives the same bytes.

Recipes (no model weights or calibration text exist here; these stand in for
the tensors the pages discuss):

* weight matrix: N(0, sigma) entries, optionally rounded to bf16 (the values a bf16
  checkpoint holds), then a Bernoulli(outlier_frac) mask whose entries are replaced
  by binary32 ``outlier_scale * t(3)`` values (Student t with 3 degrees of freedom,
  built as z / sqrt(chi2_3 / 3) from four standard normals);
* imatrix row: qw = exp(N(0, 1)) per column (log-normal), optionally with a
  random ``boost_frac`` of the columns multiplied by ``boost``;
* activations: N(0, 1) with a Bernoulli(spike_frac) mask set to
  +-U(lo, hi), the sign a fair coin (values beyond the fp16 range).
"""
from __future__ import annotations

import dataclasses

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _student_t3(n: int, g: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(4, n, generator=g, device=device, dtype=torch.float32)
    chi2 = (z[1:] * z[1:]).sum(0)
    return z[0] / torch.sqrt(chi2 / 3.0)


def weight_matrix(rows: int, cols: int, seed: int, sigma: float = 0.02,
                  outlier_frac: float = 1e-3, outlier_scale: float = 0.2,
                  bf16: bool = False, device="cpu") -> torch.Tensor:
    """float32 [rows, cols]: N(0, sigma) with t(3) outliers.  With bf16 the N(0, sigma) body is
    rounded to bf16 first and the outliers, added after, stay binary32: fp32 weights taken from
    a bf16 checkpoint, plus outliers."""
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    x.mul_(sigma)
    if bf16:
        x = x.to(torch.bfloat16).to(torch.float32)
    if outlier_frac > 0 and rows * cols > 0:
        mask = torch.rand(rows, cols, generator=g, device=device) < outlier_frac
        k = int(mask.sum().item())
        if k:
            x[mask] = outlier_scale * _student_t3(k, g, device)
    return x


def imatrix(cols: int, seed: int, boost_frac: float = 0.0, boost: float = 100.0,
            device="cpu") -> torch.Tensor:
    """float32 [cols]: log-normal column importances, optionally boosted."""
    g = _gen(seed, device)
    qw = torch.exp(torch.randn(cols, generator=g, device=device, dtype=torch.float32))
    if boost_frac > 0 and cols > 0:
        nb = int(round(boost_frac * cols))
        idx = torch.randperm(cols, generator=g, device=device)[:nb]
        qw[idx] *= boost
    return qw


def activations(tokens: int, dim: int, seed: int, spike_frac: float = 1e-4,
                lo: float = 6e4, hi: float = 2e5, device="cpu") -> torch.Tensor:
    """float32 [tokens, dim]: N(0, 1) with +-U(lo, hi) spikes beyond the fp16 range."""
    g = _gen(seed, device)
    a = torch.randn(tokens, dim, generator=g, device=device, dtype=torch.float32)
    if spike_frac > 0 and tokens * dim > 0:
        mask = torch.rand(tokens, dim, generator=g, device=device) < spike_frac
        k = int(mask.sum().item())
        if k:
            mag = lo + (hi - lo) * torch.rand(k, generator=g, device=device)
            sign = torch.where(torch.rand(k, generator=g, device=device) < 0.5, -1.0, 1.0)
            a[mask] = (mag * sign).to(torch.float32)
    return a


# ----------------------------------------------------------------------------
# Workload definitions (shapes and seeds)
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Tensor2D:
    name: str
    rows: int
    cols: int
    seed: int
    sigma: float = 0.02
    bf16: bool = False
    boost_frac: float = 0.0

    @property
    def numel(self) -> int:
        return self.rows * self.cols

    def weights(self, device="cpu") -> torch.Tensor:
        return weight_matrix(self.rows, self.cols, self.seed, sigma=self.sigma, bf16=self.bf16,
                             device=device)

    def qw(self, device="cpu") -> torch.Tensor:
        return imatrix(self.cols, self.seed + 500_000, boost_frac=self.boost_frac, device=device)


def single_matrix_1024x4096() -> Tensor2D:
    """One fp32 weight matrix 1024 x 4096, seed 0 (the small Q4_0 case)."""
    return Tensor2D("w1024x4096", 1024, 4096, 0)


LLAMA2_7B_TENSORS = (  # name, rows (output features), cols (n_per_row)
    ("attn_q", 4096, 4096), ("attn_k", 4096, 4096), ("attn_v", 4096, 4096),
    ("attn_o", 4096, 4096), ("ffn_gate", 11008, 4096), ("ffn_up", 11008, 4096),
    ("ffn_down", 4096, 11008),
)


def llama2_7b_layer_set(layers: int = 32) -> list[Tensor2D]:
    """Llama-2-7B-shaped weights: per layer q/k/v/o 4096x4096, gate/up 11008x4096,
    down 4096x11008; fp32 from bf16 N(0, 0.02), plus 0.1% binary32 0.2*t(3) outliers;
    seed = 3000 + 10*layer + tensor index."""
    out = []
    for layer in range(layers):
        for t, (name, r, c) in enumerate(LLAMA2_7B_TENSORS):
            out.append(Tensor2D(f"blk.{layer}.{name}", r, c, 3000 + 10 * layer + t, bf16=True))
    return out


def moe_experts(experts: int = 256) -> list[Tensor2D]:
    """DeepSeek-shaped experts: gate/up 2048x7168, down 7168x2048, N(0, 0.015) plus
    outliers; per-expert log-normal qw with 5% of the columns boosted x100."""
    out = []
    for e in range(experts):
        for t, (name, r, c) in enumerate((("gate", 2048, 7168), ("up", 2048, 7168),
                                          ("down", 7168, 2048))):
            out.append(Tensor2D(f"exp.{e}.{name}", r, c, 4_000_000 + 10 * e + t, sigma=0.015,
                                boost_frac=0.05))
    return out


def scaling_sweep() -> list[Tensor2D]:
    """Single tensors 4096^2, 8192^2, 16384^2, 16384x53248."""
    shapes = ((4096, 4096), (8192, 8192), (16384, 16384), (16384, 53248))
    return [Tensor2D(f"sweep{r}x{c}", r, c, 5000 + i) for i, (r, c) in enumerate(shapes)]


def activation_batch_4096x7168(device="cpu") -> torch.Tensor:
    """Q8_K_128 input: 4096 tokens x 7168, seed 2."""
    return activations(4096, 7168, 2, device=device)
