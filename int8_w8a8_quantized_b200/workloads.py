"""Seeded synthetic inputs for the W8A8 scaled-FP8 Linear.

This module only draws random numbers: it holds none of the quantization or
GEMM arithmetic, so both the CUDA path and the CPU oracle can consume its
tensors.  The pages use no public dataset (their end-to-end runs need model
weights); these recipes stand in for diffusion-transformer activations and
weights, shaped like the image- and video-DiT Linears the pages quantize.

Recipes (all bf16 after the draw; ``std`` is the normal's standard deviation):

* activations ``x``: N(0, 1), or Student-t with integer ``nu`` degrees of
  freedom built as z / sqrt(chi2_nu / nu) (chi2_nu a sum of nu squared
  normals), times ``amplitude``; optionally ``outlier_cols`` columns chosen
  without replacement and multiplied by ``outlier_mult``; optionally
  ``zero_rows`` rows set to zero;
* weights ``w``: N(0, std) with std 0.02 (image DiT) or 0.015 (video DiT);
* bias: N(0, 0.01).

Column/row choices come from the same seeded generator.  Generation happens
on the device that is asked for (a CUDA generator for the large shapes), so
the same seed gives different but equally valid draws on CPU and GPU; a test
always hands the very same tensor to both sides.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def activations(M: int, K: int, *, seed: int, device="cpu", nu: int | None = None,
                amplitude: float = 1.0, outlier_cols: int = 0, outlier_mult: float = 1.0,
                zero_rows: int = 0) -> torch.Tensor:
    """bf16 [M, K] activation matrix following the recipe in the module doc."""
    g = _gen(seed, device)
    if nu is None:
        x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    else:
        z = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
        chi2 = torch.zeros(M, K, device=device, dtype=torch.float32)
        for _ in range(int(nu)):
            e = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
            chi2.addcmul_(e, e)
            del e
        x = z.div_(chi2.div_(float(nu)).sqrt_())
        del chi2
    if amplitude != 1.0:
        x.mul_(float(amplitude))
    if outlier_cols > 0 and K > 0:
        cols = torch.randperm(K, generator=g, device=device)[:outlier_cols]
        x[:, cols] *= float(outlier_mult)
    if zero_rows > 0 and M > 0:
        rows = torch.randperm(M, generator=g, device=device)[:zero_rows]
        x[rows, :] = 0.0
    return x.to(torch.bfloat16)


def weights(N: int, K: int, *, seed: int, std: float, device="cpu") -> torch.Tensor:
    """bf16 [N, K] weight (nn.Linear layout: out x in), N(0, std)."""
    g = _gen(seed, device)
    return (torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def bias(N: int, *, seed: int, std: float = 0.01, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return (torch.randn(N, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


@dataclass(frozen=True)
class Linear:
    """One Linear of a block: its name, the activation it reads, K -> N."""
    name: str
    x: str
    K: int
    N: int


@dataclass(frozen=True)
class XRecipe:
    nu: int | None = None
    amplitude: float = 1.0
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0


@dataclass(frozen=True)
class Workload:
    """A set of Linears over M tokens, with the activation/weight recipes."""
    name: str
    M: int
    linears: tuple
    x_recipe: XRecipe
    w_std: float
    act_qmax: tuple = (448.0,)
    has_bias: bool = True
    seed: int = 0
    notes: str = ""
    extra: dict = field(default_factory=dict)

    def x_shapes(self) -> dict:
        """Distinct activation inputs and their K."""
        out = {}
        for lin in self.linears:
            out.setdefault(lin.x, lin.K)
        return out

    def flops(self) -> int:
        return sum(2 * self.M * lin.N * lin.K for lin in self.linears) * len(self.act_qmax)

    def make_x(self, xname: str, device="cpu") -> torch.Tensor:
        K = self.x_shapes()[xname]
        r = self.x_recipe
        idx = sorted(self.x_shapes()).index(xname)
        return activations(self.M, K, seed=self.seed * 1000 + 10 + idx, device=device,
                           nu=r.nu, amplitude=r.amplitude,
                           outlier_cols=int(round(r.outlier_frac * K)),
                           outlier_mult=r.outlier_mult)

    def make_w(self, lin: Linear, device="cpu") -> torch.Tensor:
        idx = [l.name for l in self.linears].index(lin.name)
        return weights(lin.N, lin.K, seed=self.seed * 1000 + 100 + idx, std=self.w_std, device=device)

    def make_bias(self, lin: Linear, device="cpu"):
        if not self.has_bias:
            return None
        idx = [l.name for l in self.linears].index(lin.name)
        return bias(lin.N, seed=self.seed * 1000 + 200 + idx, device=device)


def _dit_block(K: int, F: int):
    """Q, K, V read one normed input; O reads the attention output; FFN up
    reads the second normed input; FFN down reads the activated FFN hidden."""
    return (
        Linear("q", "x_attn", K, K),
        Linear("k", "x_attn", K, K),
        Linear("v", "x_attn", K, K),
        Linear("o", "x_o", K, K),
        Linear("ffn_up", "x_ffn", K, F),
        Linear("ffn_down", "x_ffn_h", F, K),
    )


# Tiny W8A8 Linear: X [64, 256] N(0,1) with 4 outlier columns x20,
# W [128, 256] N(0, 0.02), qmax 448, bias N(0, 0.01), seed 0.
TINY = Workload("tiny_w8a8_linear", 64, (Linear("lin", "x", 256, 128),),
                XRecipe(outlier_frac=4 / 256, outlier_mult=20.0), w_std=0.02, seed=0)

# Image-DiT block Linears: 83 x 83 latent grid = 6889 tokens, hidden 3072,
# FFN 12288; X N(0,1) with 1 % outlier columns x20, W N(0, 0.02).
IMAGE_DIT = Workload("image_dit_block", 6889, _dit_block(3072, 12288),
                     XRecipe(outlier_frac=0.01, outlier_mult=20.0), w_std=0.02, seed=2)

# Video-DiT block Linears: 21 x 45 x 80 latent grid = 75600 tokens, hidden
# 5120, FFN 13824; X heavy tailed (Student-t nu = 4), W N(0, 0.015).
VIDEO_DIT = Workload("video_dit_block", 75600, _dit_block(5120, 13824),
                     XRecipe(nu=4), w_std=0.015, seed=3)

# Reduced-qmax FFN-out: M = 32760, K = 13824 -> N = 5120, activation qmax 7
# and 14, X = 4 * Student-t(nu = 3), FP8 W (qmax 448) N(0, 0.015), bias.
REDUCED_QMAX = Workload("reduced_qmax_ffn_out", 32760, (Linear("ffn_down", "x_ffn_h", 13824, 5120),),
                        XRecipe(nu=3, amplitude=4.0), w_std=0.015, act_qmax=(7.0, 14.0), seed=4)

WORKLOADS = {w.name: w for w in (TINY, IMAGE_DIT, VIDEO_DIT, REDUCED_QMAX)}


def quantizer_input(device="cpu", M: int = 8192, K: int = 3072, seed: int = 1) -> torch.Tensor:
    """Activation-quantizer workload: X [8192, 3072] N(0,1), 1 % of the
    columns (31) x50, plus 16 all-zero rows."""
    return activations(M, K, seed=seed, device=device, outlier_cols=int(round(0.01 * K)),
                       outlier_mult=50.0, zero_rows=16)
