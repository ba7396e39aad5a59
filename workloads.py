"""Seeded synthetic inputs for the Muon / Dimuon step.

This module only draws random numbers and lays out shapes; it holds none of
the optimizer's arithmetic.  Both the tests (which hand the same arrays to the
CUDA library and to the CPU oracle) and the benchmark use it.

Recipes (all host-side numpy, float64 draws, then cast by the caller):

* toy LoRA factor, 4x16 fp32 ("Dimuon: LoRA 에 맞춰 다시 짠 Muon", section
  "16 columns with input size 0.1 to 10"): Z ~ N(0,1) from default_rng(0),
  s_j = logspace(-1, 1, 16), G = Z * s_j^2 column-wise; the same G feeds both
  steps.
* one 1024x1024 matrix: G ~ N(0,1), seed 1.
* GPT-2-small hidden matrices (12 layers x {Q, K, V, attn-out 768x768,
  MLP-up 768x3072, MLP-down 3072x768}): G = N(0,1) * col_scale_j with
  col_scale ~ LogNormal(0, 1), and 3 distinct outlier input columns per
  matrix multiplied by 50; seed 2.
* large batch: 8 x 4096x4096, 4 x 4096x14336, 4 x 14336x4096, G ~ N(0,1),
  seed 3.
* LoRA batch: 224 projections of width 4096, each with A (r x 4096) and
  B (4096 x r).  Per projection s_j ~ log-uniform(0.1, 10) over the 4096
  input channels with 6 outlier channels x100; gradient columns of A (rows of
  B) are scaled by s_j^2 and drawn fresh N(0,1) each step; for 16 chosen rows
  of each B the gradient is zero for steps 1-5 and scaled by 1e-3 from step 6.
  Seed 4.
* 1-D parameters ("From PCG to Muon", section 6 "Muon Reshaping"): 64
  vectors of 262,267 variables (2^18 + 123, so the last row is ragged),
  each laid out row-major at width 1, 2, 8, 32 or 128 with the cells past the
  end zero; gradients N(0,1) on the variables and zero in the padding, seed 5.
* weights: W ~ N(0, 0.02^2) from default_rng(seed + 1000).
"""
from __future__ import annotations

import numpy as np

GPT2_LAYERS = 12
GPT2_WIDTH = 768
VECTOR_LENGTH = (1 << 18) + 123
VECTOR_COUNT = 64


def toy_lora_factor():
    """The 4x16 toy gradient and the per-column input sizes s_j."""
    rng = np.random.default_rng(0)
    Z = rng.standard_normal((4, 16))
    s = np.logspace(-1, 1, 16)
    return Z * (s ** 2)[None, :], s


def weights_like(shapes, seed):
    rng = np.random.default_rng(seed + 1000)
    return [0.02 * rng.standard_normal(shp) for shp in shapes]


def gaussian_grads(shapes, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal(shp) for shp in shapes]


def single_square_shapes(n=1024):
    return [(n, n)]


def gpt2_small_shapes(layers=GPT2_LAYERS, d=GPT2_WIDTH):
    shapes = []
    for _ in range(layers):
        shapes += [(d, d)] * 4 + [(d, 4 * d), (4 * d, d)]
    return shapes


def gpt2_small_grads(seed=2, layers=GPT2_LAYERS, d=GPT2_WIDTH,
                     n_outliers=3, outlier_gain=50.0):
    """Gradients with log-normal per-input-column scales and outlier columns."""
    rng = np.random.default_rng(seed)
    out = []
    for shp in gpt2_small_shapes(layers, d):
        rows, cols = shp
        col_scale = rng.lognormal(0.0, 1.0, cols)
        idx = rng.choice(cols, n_outliers, replace=False)
        col_scale[idx] *= outlier_gain
        out.append(rng.standard_normal(shp) * col_scale[None, :])
    return out


def large_batch_shapes():
    return [(4096, 4096)] * 8 + [(4096, 14336)] * 4 + [(14336, 4096)] * 4


def lora_shapes(r, projections=224, width=4096):
    """Interleaved [A_0, B_0, A_1, B_1, ...] factor shapes."""
    shapes = []
    for _ in range(projections):
        shapes += [(r, width), (width, r)]
    return shapes


class LoraGradStream:
    """Per-step gradients for the LoRA batch (fresh N(0,1) every step)."""

    def __init__(self, r, projections=224, width=4096, seed=4,
                 n_outliers=6, outlier_gain=100.0, dead_rows=16):
        self.r, self.projections, self.width = r, projections, width
        rng = np.random.default_rng(seed)
        self.scales = []
        self.dead = []
        for _ in range(projections):
            s = np.exp(rng.uniform(np.log(0.1), np.log(10.0), width))
            s[rng.choice(width, n_outliers, replace=False)] *= outlier_gain
            self.scales.append(s)
            self.dead.append(rng.choice(width, dead_rows, replace=False))
        self.rng = np.random.default_rng(seed + 1)

    def step(self, t):
        """Gradients for step t (1-based), in lora_shapes order."""
        grads = []
        for p in range(self.projections):
            s2 = self.scales[p] ** 2
            gA = self.rng.standard_normal((self.r, self.width)) * s2[None, :]
            gB = self.rng.standard_normal((self.width, self.r)) * s2[:, None]
            gB[self.dead[p], :] *= 0.0 if t <= 5 else 1e-3
            grads += [gA, gB]
        return grads


CONFIGS = {
    "toy": "toy LoRA factor 4x16 fp32, two steps",
    "square1024": "one 1024x1024 bf16 matrix",
    "gpt2_small": "GPT-2-small hidden matrices (72), Moonshot scale, wd 0.1",
    "large_batch": "8x4096^2 + 4x4096x14336 + 4x14336x4096 bf16",
    "lora": "224 LoRA projections (A r x 4096, B 4096 x r), Dimuon, 20 steps",
}


def vector_shapes(width, count=VECTOR_COUNT, length=VECTOR_LENGTH):
    """count vectors of `length` variables, each in a ceil(length / width) x
    width matrix (row-major, zero-padded)."""
    return [(-(-length // width), width)] * count


def vector_grads(width, count=VECTOR_COUNT, length=VECTOR_LENGTH, seed=5):
    """N(0,1) gradients on the variables, zero in the padding cells, laid out
    as vector_shapes(width)."""
    rng = np.random.default_rng(seed)
    rows = -(-length // width)
    out = []
    for _ in range(count):
        g = np.zeros(rows * width)
        g[:length] = rng.standard_normal(length)
        out.append(g.reshape(rows, width))
    return out
