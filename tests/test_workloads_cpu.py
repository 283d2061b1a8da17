"""The seeded synthetic workloads on CPU: model shapes and symbol totals, the
per-tensor value laws, and the two 8192x8192 stress tensors' defining
properties (near-uniform 8-bit codes; p(mode) = 0.9 with a Huffman code whose
unlimited length exceeds the 16-bit limit, so the limit binds)."""
import heapq
import math

import numpy as np
import pytest

import oracle
import workloads


def _huffman_max_length(hist):
    """Longest code of an unlimited Huffman code (Huffman 1952), by a heap of subtree depths."""
    items = [(int(h), i, 0) for i, h in enumerate(hist) if h > 0]
    heapq.heapify(items)
    tick = len(hist)
    while len(items) > 1:
        w1, _, d1 = heapq.heappop(items)
        w2, _, d2 = heapq.heappop(items)
        heapq.heappush(items, (w1 + w2, tick, max(d1, d2) + 1))
        tick += 1
    return items[0][2]


def _entropy(hist):
    p = hist[hist > 0] / hist.sum()
    return float(-(p * np.log2(p)).sum())


@pytest.mark.parametrize("name, count, symbols", [
    ("smollm_1p7b_u8", 169, 24 * 67_108_864 + 100_663_296),
    ("mistral_7b_u4", 224, 32 * 218_103_808),
    ("phi3_mini_u8", 128, 32 * 113_246_208),
])
def test_model_shapes_and_totals(name, count, symbols):
    W = workloads.get(name)
    assert len(W.tensors) == count
    assert sum(t.rows * t.cols for t in W.tensors) == symbols
    assert [t.index for t in W.tensors] == list(range(count))


def test_smollm_layout_and_mixed_laws():
    W = workloads.get("smollm_1p7b_u8")
    shapes = [(t.rows, t.cols) for t in W.tensors]
    assert shapes.count((2048, 2048)) == 4 * 24
    assert shapes.count((8192, 2048)) == 2 * 24 and shapes.count((2048, 8192)) == 24
    assert shapes.count((49152, 2048)) == 1
    for name in ("smollm_1p7b_u8", "phi3_mini_u8"):
        ts = workloads.get(name).tensors
        sig = np.array([t.param for t in ts])
        assert all(t.law == "t4std" for t in ts)
        assert sig.min() >= 0.01 and sig.max() <= 0.04
        assert sum(t.shifted for t in ts) == round(0.1 * len(ts))


def test_value_laws_on_drawn_tensors():
    # Mistral-shaped k projection: Laplace with std 0.02 (b = 0.02 / sqrt 2)
    W = workloads.get("mistral_7b_u4")
    w = workloads.weights(W, W.tensors[1]).numpy().astype(np.float64)
    assert w.shape == (1024, 4096)
    assert abs(w.std() / 0.02 - 1.0) < 0.01 and abs(w.mean()) < 2e-4
    # SmolLM-shaped q projection: sigma * t(4) / sqrt 2.  t(4) has no finite fourth moment, so
    # the check uses the interquartile range.  The t(4) CDF in closed form is
    # F(t) = 1/2 + (3/4) u (1 - u^2 / 3) with u = t / sqrt(4 + t^2); its upper quartile solves F = 3/4.
    W = workloads.get("smollm_1p7b_u8")
    spec = next(t for t in W.tensors if not t.shifted)
    w = workloads.weights(W, spec).numpy().astype(np.float64)
    u = _solve_quartile_u()
    t75 = 2.0 * u / math.sqrt(1.0 - u * u)
    assert abs(t75 - 0.74070) < 1e-4          # the tabulated upper quartile of t(4)
    q1, q3 = np.quantile(w, [0.25, 0.75])
    assert abs((q3 - q1) / (2.0 * t75 * spec.param / math.sqrt(2.0)) - 1.0) < 0.01
    # a shifted tensor is non-negative with minimum 0
    shifted = next(t for t in W.tensors if t.shifted and t.rows * t.cols <= 1 << 24)
    ws = workloads.weights(W, shifted).numpy()
    assert float(ws.min()) == 0.0


def _solve_quartile_u():
    """u in (0, 1) with (3/4) u (1 - u^2 / 3) = 1/4 (bisection; the left side increases on (0, 1))."""
    lo, hi = 0.0, 1.0
    for _ in range(80):
        mid = 0.5 * (lo + hi)
        if 0.75 * mid * (1.0 - mid * mid / 3.0) < 0.25:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_stress_tensors_properties():
    W = workloads.get("stress_8192_u8")
    uniform, skew = W.tensors
    assert (uniform.rows, uniform.cols) == (skew.rows, skew.cols) == (8192, 8192)
    # near-uniform: asymmetric 8-bit codes of U(-1, 1), entropy ~7.99 bits
    q, _, _, _ = oracle.quantize(workloads.weights(W, uniform).numpy(), 8, oracle.MODE_ASYM)
    hist = np.bincount(q, minlength=256)
    assert 7.98 < _entropy(hist) <= 8.0
    assert int(oracle.code_lengths(hist, 16).max()) <= 9
    # skew: each weight is 0 with probability 0.9, so p(mode) is 0.9 up to sampling noise (within
    # four standard errors); the unlimited Huffman code is longer than 16 bits, so the limit binds
    q, _, _, _ = oracle.quantize(workloads.weights(W, skew).numpy(), 8, oracle.MODE_ASYM)
    hist = np.bincount(q, minlength=256)
    p_mode = hist.max() / hist.sum()
    assert abs(p_mode - 0.9) <= 4.0 * math.sqrt(0.9 * 0.1 / hist.sum())
    assert _huffman_max_length(hist) > 16
    assert int(oracle.code_lengths(hist, 16).max()) == 16
