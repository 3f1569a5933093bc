"""Seeded synthetic inputs for the quantizer workloads.

This module draws random numbers only.  It holds none of the quantizer's
arithmetic and is shared by the tests, the smoke check and the benchmark so
that the CUDA library and the CPU oracle see the same bytes.  There are no
trained weights or calibration datasets here: the weight matrices stand in
for the Llama/Qwen linear layers the pages quantize, with the shapes and the
heavy-tailed value distributions stated below.

Workloads (rows = output features, cols = input features; blocks run along a
row, so a row is contiguous in memory):

* ``small_outliers``  128 x 256 fp32, N(0, 0.02^2), two planted outliers per
  row at +-10 sigma (two distinct random columns, random sign); seed 0.
* ``q_proj_4096``     4096 x 4096 bf16, Student-t(4) * 0.02, each output row
  scaled by a lognormal(0, 0.5) multiplier; seed 2.
* ``mlp_11008``       11008 x 4096 bf16, Student-t(4) * 0.02; the WMSE
  importance is diag(X^T X) of activations X (2048 x 4096 bf16, N(0,1), 41 =
  round(1% of 4096) random columns scaled by 50), summed in fp64 and rounded
  once to fp32; seed 3.
* ``up_proj_28672``   28672 x 8192 bf16, Student-t(3) * 0.015, with one
  random-sign mask per 32-column group from splitmix64; seed 4.
* ``llama3_8b``       224 tensors of a Llama-3-8B-shaped model (32 layers x
  q,k,v,o,gate,up,down; hidden 4096, kv 1024, intermediate 14336),
  Student-t(4) * 0.02 in bf16; seed 5.

Student-t(nu) for integer nu is drawn as z / sqrt(chi2_nu / nu) with chi2_nu
the sum of nu squared standard normals, in fp32, then rounded to bf16 (round
to nearest even).
"""
from __future__ import annotations

import numpy as np
import torch

LLAMA3_8B_LAYERS = 32
LLAMA3_8B_HIDDEN = 4096
LLAMA3_8B_KV = 1024
LLAMA3_8B_INTER = 14336


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def student_t(shape, nu: int, scale: float, gen: torch.Generator, device="cpu") -> torch.Tensor:
    """Student-t(nu) * scale in fp32 (integer nu)."""
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(int(nu)):
        u = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        chi2.add_(u * u)
    return z / torch.sqrt(chi2 / float(nu)) * float(scale)


def small_outliers(rows=128, cols=256, seed=0, std=0.02, mult=10.0, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    w = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32) * std
    # two distinct random columns per row, random sign, magnitude mult * std
    perm = torch.argsort(torch.rand((rows, cols), generator=g, device=device), dim=1)[:, :2]
    sign = torch.where(torch.rand((rows, 2), generator=g, device=device) < 0.5, -1.0, 1.0)
    w.scatter_(1, perm, sign.to(torch.float32) * (mult * std))
    return w


def q_proj(rows=4096, cols=4096, seed=2, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    w = student_t((rows, cols), 4, 0.02, g, device)
    mult = torch.exp(0.5 * torch.randn((rows, 1), generator=g, device=device, dtype=torch.float32))
    return (w * mult).to(torch.bfloat16)


def t_weight(rows, cols, nu=4, scale=0.02, seed=3, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return student_t((rows, cols), nu, scale, g, device).to(torch.bfloat16)


def importance_diag_xtx(cols=4096, tokens=2048, frac_hot=0.01, hot_scale=50.0, seed=3,
                        device="cpu") -> torch.Tensor:
    """diag(X^T X) of synthetic activations X (tokens x cols, bf16 N(0,1), a few hot columns)."""
    g = _gen(seed + 1000, device)
    x = torch.randn((tokens, cols), generator=g, device=device, dtype=torch.float32)
    n_hot = int(round(frac_hot * cols))
    hot = torch.randperm(cols, generator=g, device=device)[:n_hot]
    x[:, hot] *= hot_scale
    xb = x.to(torch.bfloat16).to(torch.float64)
    return (xb * xb).sum(dim=0).to(torch.float32)


def splitmix64(seed: int, n: int) -> np.ndarray:
    """The first n outputs of splitmix64 started at ``seed`` (uint64)."""
    with np.errstate(over="ignore"):
        state = np.uint64(seed) + np.arange(1, n + 1, dtype=np.uint64) * np.uint64(0x9E3779B97F4A7C15)
        z = state
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def sign_masks(cols: int, seed: int = 4) -> np.ndarray:
    """One 32-bit random-sign mask per 32-column group (bit j set: negate column 32g+j)."""
    return (splitmix64(seed, cols // 32) & np.uint64(0xFFFFFFFF)).astype(np.uint32)


def llama3_8b_shapes(layers=LLAMA3_8B_LAYERS, hidden=LLAMA3_8B_HIDDEN, kv=LLAMA3_8B_KV,
                     inter=LLAMA3_8B_INTER):
    """(name, rows, cols) of every linear weight: rows = out features, cols = in features."""
    out = []
    for layer in range(layers):
        for name, r, c in (("q", hidden, hidden), ("k", kv, hidden), ("v", kv, hidden),
                           ("o", hidden, hidden), ("gate", inter, hidden), ("up", inter, hidden),
                           ("down", hidden, inter)):
            out.append((f"layers.{layer}.{name}", r, c))
    return out


def llama3_8b_tensor(index: int, rows: int, cols: int, seed=5, device="cpu") -> torch.Tensor:
    return t_weight(rows, cols, nu=4, scale=0.02, seed=seed * 100003 + index, device=device)
