"""Seeded synthetic inputs for the Huffman weight-decoding path.

This module only draws numbers: fp32 weight tensors shaped like the models the
EntroLLM and LazyWeights pages evaluate (smolLM-1.7B, phi3-mini-4k, mistral-7B)
and bf16 activation vectors.  It holds none of the method's arithmetic (no
quantization, no coding, no decoding) and imports neither the oracle nor the
CUDA library, so both sides of every parity test can draw from it.

The pages measure on real checkpoints and language datasets; none of those is
available here, so these seeded tensors stand in for them.  Value laws:

* ``t4(scale)``: Student-t with 4 degrees of freedom times ``scale``.
* ``t4std(sigma)``: Student-t(4) rescaled to standard deviation ``sigma``
  (the t(4) law has variance 2, so ``sigma * t / sqrt(2)``).
* ``laplace(b)``: Laplace(0, b); "Laplace with std s" means b = s / sqrt(2).
* ``shifted``: ``w - min(w)`` (a non-negative tensor).
* ``uniform``: U(-1, 1).
* ``skew``: 0 with probability 0.9, else +-0.02 * (1 + |t(4)|): the non-zero
  draws stay clear of the zero code, so the most frequent code has p = 0.9.

Small single tensors (the 1024x1024 and 4096x4096 cases) come from NumPy's
``default_rng([config_seed, tensor_index])``; model-sized tensors come from
torch's Philox generator on the requested device, seeded with
``config_seed * 2**32 + tensor_index``, so that billions of weights can be drawn
in seconds on the GPU.  Activations x ~ N(0, 1) are drawn with NumPy
``default_rng([config_seed, 2_000_000 + K])`` and rounded to bf16.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator, List, Optional, Tuple

import numpy as np
import torch

QUANT_AUTO = 0
QUANT_UNSIGNED = 1
QUANT_ASYM = 2

FORMAT_SINGLE = 1      # one bitstream per chunk
FORMAT_LANES = 2       # 32 word-interleaved lane bitstreams per chunk
FORMAT_ROWS = 3        # row tiles: lane l of a chunk is row l of a 32- or 64-row tile
FORMAT_ROWS_CO = 4     # row tiles, each lane's words in consumption order (no lane padding)


@dataclasses.dataclass(frozen=True)
class TensorSpec:
    name: str
    rows: int           # N (output features)
    cols: int           # K (input features)
    law: str            # see module docstring
    param: float        # scale / sigma / b of the law
    shifted: bool = False
    index: int = 0      # tensor index within its workload (seed component)

    @property
    def n(self) -> int:
        return self.rows * self.cols


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    bits: int
    quant_mode: int
    max_len: int
    fmt: int
    chunk_rule: str     # "fixed:<C>" or "rows" (whole rows, about 8192 symbols)
    tensors: Tuple[TensorSpec, ...]
    description: str
    lanes: int = 32     # interleaved lanes per chunk of the lanes format

    def chunk_symbols(self, cols: int) -> int:
        if self.chunk_rule.startswith("fixed:"):
            return int(self.chunk_rule.split(":")[1])
        return max(1, 8192 // cols) * cols

    @property
    def n(self) -> int:
        return sum(t.n for t in self.tensors)


def _smollm_1p7b(seed: int) -> Tuple[TensorSpec, ...]:
    layers, d, f, vocab = 24, 2048, 8192, 49152
    shapes = []
    for layer in range(layers):
        for nm, r, c in (("q", d, d), ("k", d, d), ("v", d, d), ("o", d, d),
                         ("gate", f, d), ("up", f, d), ("down", d, f)):
            shapes.append((f"layers.{layer}.{nm}", r, c))
    shapes.append(("embed", vocab, d))
    return _t4_mixed(seed, shapes)


def _phi3_mini(seed: int) -> Tuple[TensorSpec, ...]:
    layers, d, f = 32, 3072, 8192
    shapes = []
    for layer in range(layers):
        for nm, r, c in (("qkv", 3 * d, d), ("o", d, d), ("gate_up", 2 * f, d), ("down", d, f)):
            shapes.append((f"layers.{layer}.{nm}", r, c))
    return _t4_mixed(seed, shapes)


def _t4_mixed(seed: int, shapes) -> Tuple[TensorSpec, ...]:
    """Per-tensor sigma ~ U(0.01, 0.04) and a seeded 10% of tensors shifted non-negative."""
    meta = np.random.default_rng([seed, 1_000_000])
    count = len(shapes)
    sigmas = meta.uniform(0.01, 0.04, size=count)
    shifted = set(int(i) for i in meta.choice(count, size=int(round(0.1 * count)), replace=False))
    return tuple(TensorSpec(nm, r, c, "t4std", float(sigmas[i]), i in shifted, i)
                 for i, (nm, r, c) in enumerate(shapes))


def _mistral_7b() -> Tuple[TensorSpec, ...]:
    layers, d, kv, f = 32, 4096, 1024, 14336
    b = 0.02 / math.sqrt(2.0)
    out, i = [], 0
    for layer in range(layers):
        for nm, r, c in (("q", d, d), ("k", kv, d), ("v", kv, d), ("o", d, d),
                         ("gate", f, d), ("up", f, d), ("down", d, f)):
            out.append(TensorSpec(f"layers.{layer}.{nm}", r, c, "laplace", b, False, i))
            i += 1
    return tuple(out)


WORKLOADS = {
    "t4_1024x1024_u8": Workload(
        "t4_1024x1024_u8", 0, 8, QUANT_ASYM, 16, FORMAT_SINGLE, "fixed:4096",
        (TensorSpec("w", 1024, 1024, "t4", 0.02),),
        "single 1024x1024 tensor, 0.02*t(4), asymmetric 8-bit, max code length 16, "
        "single-stream 4096-symbol chunks"),
    "laplace_4096x4096_u4": Workload(
        "laplace_4096x4096_u4", 1, 4, QUANT_ASYM, 12, FORMAT_LANES, "fixed:8192",
        (TensorSpec("w", 4096, 4096, "laplace", 0.015),),
        "single 4096x4096 tensor, Laplace(0, 0.015), asymmetric 4-bit, max code length 12, "
        "32 word-interleaved lanes per 8192-symbol chunk"),
    "smollm_1p7b_u8": Workload(
        "smollm_1p7b_u8", 2, 8, QUANT_AUTO, 16, FORMAT_ROWS, "fixed:4096",
        _smollm_1p7b(2),
        "SmolLM-1.7B-shaped (24 layers + 49152x2048 embedding), t(4) with per-tensor std "
        "U(0.01, 0.04), 10% shifted non-negative, mixed unsigned/asymmetric 8-bit"),
    "mistral_7b_u4": Workload(
        "mistral_7b_u4", 3, 4, QUANT_ASYM, 12, FORMAT_ROWS, "fixed:8192",
        _mistral_7b(),
        "Mistral-7B-shaped (32 layers), Laplace with std 0.02, asymmetric 4-bit, "
        "row tiles of 32 rows x 256 columns, fused GEMV at batch 1", 32),
    "phi3_mini_u8": Workload(
        "phi3_mini_u8", 4, 8, QUANT_AUTO, 16, FORMAT_ROWS, "fixed:4096",
        _phi3_mini(4),
        "Phi-3-mini-shaped (32 layers), t(4) with per-tensor std U(0.01, 0.04), 10% shifted, "
        "mixed unsigned/asymmetric 8-bit, row tiles of 32 rows x 128 columns, fused GEMV at batch 1/4/16"),
    "stress_8192_u8": Workload(
        "stress_8192_u8", 4, 8, QUANT_ASYM, 16, FORMAT_ROWS, "fixed:4096",
        (TensorSpec("near_uniform", 8192, 8192, "uniform", 1.0, False, 1000),
         TensorSpec("skew", 8192, 8192, "skew", 0.02, False, 1001)),
        "two 8192x8192 stress tensors: near-uniform codes and p(mode)=0.9 skew"),
}


def _torch_seed(seed: int, index: int) -> int:
    return (seed << 32) + index


def _draw_torch(spec: TensorSpec, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(_torch_seed(seed, spec.index))
    shape = (spec.rows, spec.cols)
    if spec.law in ("t4", "t4std", "skew"):
        z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        u1 = 1.0 - torch.rand(shape, generator=g, device=device, dtype=torch.float32)
        u2 = 1.0 - torch.rand(shape, generator=g, device=device, dtype=torch.float32)
        chi2_4 = -2.0 * torch.log(u1 * u2)          # chi-square, 4 degrees of freedom
        t = z * torch.rsqrt(chi2_4 * 0.25)
        if spec.law == "t4":
            w = spec.param * t
        elif spec.law == "t4std":
            w = (spec.param / math.sqrt(2.0)) * t
        else:
            keep = torch.rand(shape, generator=g, device=device) >= 0.9
            mag = spec.param * (1.0 + t.abs())
            w = torch.where(keep, torch.sign(t) * mag, torch.zeros_like(t))
    elif spec.law == "laplace":
        u = torch.rand(shape, generator=g, device=device, dtype=torch.float32).clamp_min(1e-7) - 0.5
        w = -spec.param * torch.sign(u) * torch.log1p(-2.0 * u.abs())
    elif spec.law == "uniform":
        w = torch.rand(shape, generator=g, device=device, dtype=torch.float32) * 2.0 - 1.0
    else:
        raise ValueError(spec.law)
    w = w.to(torch.float32)
    if spec.shifted:
        w = w - w.min()
    return w.contiguous()


def _draw_numpy(spec: TensorSpec, seed: int) -> np.ndarray:
    rng = np.random.default_rng([seed, spec.index])
    shape = (spec.rows, spec.cols)
    if spec.law == "t4":
        w = spec.param * rng.standard_t(4, size=shape)
    elif spec.law == "laplace":
        w = rng.laplace(0.0, spec.param, size=shape)
    else:
        raise ValueError(f"numpy path has no law {spec.law}")
    w = w.astype(np.float32)
    if spec.shifted:
        w = w - w.min()
    return np.ascontiguousarray(w)


def weights(workload: Workload, spec: TensorSpec, device="cpu") -> torch.Tensor:
    """The fp32 [rows, cols] weight tensor ``spec`` of ``workload`` on ``device``.

    Single-tensor workloads are drawn with NumPy (device-independent values); model-sized
    ones with torch's generator on ``device`` (values depend on the device type).
    """
    if len(workload.tensors) == 1 and spec.law in ("t4", "laplace"):
        return torch.from_numpy(_draw_numpy(spec, workload.seed)).to(device)
    return _draw_torch(spec, workload.seed, device)


def iter_weights(workload: Workload, device="cpu") -> Iterator[Tuple[TensorSpec, torch.Tensor]]:
    for spec in workload.tensors:
        yield spec, weights(workload, spec, device)


def activations(seed: int, batch: int, cols: int) -> torch.Tensor:
    """x ~ N(0, 1) of shape [batch, cols], rounded to bf16 (CPU tensor)."""
    rng = np.random.default_rng([seed, 2_000_000 + cols])
    x = rng.standard_normal((batch, cols)).astype(np.float32)
    return torch.from_numpy(x).to(torch.bfloat16)


def small_tensor(kind: str, rows: int, cols: int, seed: int) -> np.ndarray:
    """Small seeded fp32 tensors for edge-case tests (CPU, NumPy)."""
    rng = np.random.default_rng([seed, 3_000_000 + rows * 131 + cols])
    shape = (rows, cols)
    if kind == "t4":
        w = 0.02 * rng.standard_t(4, size=shape)
    elif kind == "laplace":
        w = rng.laplace(0.0, 0.015, size=shape)
    elif kind == "uniform":
        w = rng.uniform(-1.0, 1.0, size=shape)
    elif kind == "shifted":
        w = 0.02 * rng.standard_t(4, size=shape)
        w = w - w.min()
    elif kind == "positive":
        w = 0.5 + 0.01 * rng.standard_t(4, size=shape)
        w = np.abs(w)
    elif kind == "skew":
        t = 0.02 * rng.standard_t(4, size=shape)
        w = np.where(rng.random(shape) >= 0.9, t, 0.0)
    elif kind == "constant":
        w = np.full(shape, -0.375)
    elif kind == "zeros":
        w = np.zeros(shape)
    elif kind == "two_values":
        w = np.where(rng.random(shape) < 0.3, 1.0, -1.0)
    else:
        raise ValueError(kind)
    return np.ascontiguousarray(w.astype(np.float32))


def names() -> List[str]:
    return list(WORKLOADS)


def get(name: str) -> Workload:
    return WORKLOADS[name]


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a CPU bf16 tensor (no arithmetic)."""
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def describe(name: Optional[str] = None) -> str:
    if name is None:
        return "\n".join(f"{k}: {w.description}" for k, w in WORKLOADS.items())
    return WORKLOADS[name].description
