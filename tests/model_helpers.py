"""Encode and upload a whole model-shaped workload (test and benchmark plumbing).

Weights are drawn on the GPU (seeded torch Philox, see workloads.py), copied to
the host one tensor at a time and encoded by libentro on all host cores; the
fp32 model is never held in memory as a whole.  A regenerated tensor is
bit-identical, so parity checks redraw the tensors they sample.
"""
from __future__ import annotations

import time
from typing import List

import torch

import workloads


def encode_workload(entro, W: workloads.Workload, device="cuda", limit=None):
    """Returns (device tensors, per-tensor blob info, seconds spent encoding)."""
    dts, infos = [], []
    t_enc = 0.0
    specs = W.tensors if limit is None else W.tensors[:limit]
    for spec in specs:
        w = workloads.weights(W, spec, device=device).cpu().numpy()
        t0 = time.perf_counter()
        blob = entro.Blob.encode(w, bits=W.bits, quant_mode=W.quant_mode, max_len=W.max_len, fmt=W.fmt,
                                 chunk_symbols=W.chunk_symbols(spec.cols), lanes=W.lanes)
        t_enc += time.perf_counter() - t0
        del w
        dts.append(entro.upload(blob, device=device))
        infos.append(blob.info())
        del blob
    return dts, infos, t_enc


def sample_indices(n: int, k: int = 4) -> List[int]:
    """A spread of tensor indices: first, last and evenly spaced ones."""
    if n <= k:
        return list(range(n))
    step = (n - 1) / (k - 1)
    return sorted(set(int(round(i * step)) for i in range(k)))
