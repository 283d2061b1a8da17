"""The entropy-reducing effect of tensor-level quantization (EntroLLM, arXiv
2505.02380v4: abstract; technical summary, "Methodologie" item 1): one scale
(and zero point) per tensor keeps the integer codes as peaked as the weights,
while block-based quantization stretches every small block over the whole code
range and flattens the histogram.  Checked on the seeded stand-ins for the pages'
tensors: the code entropy and the length-limited Huffman bits/weight of the
tensor-level codes (the oracle's quantizer, unsigned/asymmetric by lower entropy)
against block-wise asymmetric min/max quantization with blocks of 64 and 128
weights along a row (the comparator, written out below).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

# (workload, tensor name, rows kept) -- a row slice keeps the test short
CASES = [
    ("t4_1024x1024_u8", None, 1024),
    ("laplace_4096x4096_u4", None, 512),
    ("smollm_1p7b_u8", "layers.0.q", 512),
    ("smollm_1p7b_u8", "layers.0.gate", 256),
    ("mistral_7b_u4", "layers.0.q", 512),
    ("phi3_mini_u8", "layers.0.o", 512),
]


def block_codes(w: np.ndarray, bits: int, block: int) -> np.ndarray:
    """Asymmetric min/max quantization per block of `block` consecutive weights of a row."""
    top = (1 << bits) - 1
    rows, cols = w.shape
    assert cols % block == 0
    b = w.astype(np.float64).reshape(rows, cols // block, block)
    lo = b.min(axis=2, keepdims=True)
    hi = b.max(axis=2, keepdims=True)
    scale = (hi - lo) / top
    scale = np.where(scale > 0, scale, 1.0)
    zero = np.rint(-lo / scale)
    q = np.clip(np.rint(b / scale) + zero, 0, top)
    return q.astype(np.uint8).reshape(-1)


def stats(codes: np.ndarray, bits: int, max_len: int):
    hist = oracle.histogram(codes, 1 << bits)
    H = oracle.entropy(hist)
    lengths = oracle.code_lengths(hist, max_len).astype(np.float64)
    return H, float((hist * lengths).sum() / hist.sum())


def measure(name, tensor, rows):
    W = workloads.get(name)
    spec = W.tensors[0] if tensor is None else next(s for s in W.tensors if s.name == tensor)
    w = workloads.weights(W, spec, device="cpu").numpy()[:rows]
    q, _, _, _ = oracle.quantize(w, W.bits, oracle.MODE_AUTO)
    out = {"tensor": stats(q, W.bits, W.max_len)}
    for block in (64, 128):
        out[f"block{block}"] = stats(block_codes(w, W.bits, block), W.bits, W.max_len)
    return W, spec, out


def test_block_quantizer_reduces_to_tensor_level_on_one_block():
    """With one block per row, the comparator is per-row asymmetric quantization: on a row
    whose min is 0 and max 1 its codes equal the tensor-level asymmetric codes of that row."""
    w = np.linspace(0.0, 1.0, 64, dtype=np.float32).reshape(1, 64)
    q_block = block_codes(w, 8, 64)
    q_tensor, _, _, _ = oracle.quantize(w, 8, oracle.MODE_ASYM)
    assert np.array_equal(q_block, q_tensor)
    assert q_block[0] == 0 and q_block[-1] == 255


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-{c[1]}" for c in CASES])
def test_tensor_level_codes_have_lower_entropy(case):
    W, spec, out = measure(*case)
    H_t, L_t = out["tensor"]
    for block in (64, 128):
        H_b, L_b = out[f"block{block}"]
        assert H_t < H_b - 0.25, (spec.name, block, H_t, H_b)
        assert L_t < L_b, (spec.name, block, L_t, L_b)
    # smaller blocks stretch the codes further
    assert out["block64"][0] > out["block128"][0]
