"""Full-size parity on the model-shaped workloads, in the launch configuration the
grouped kernels use (one launch over every tensor).

Whole-model outputs are too large for the oracle to recompute in full; sampled
tensors are checked completely (codes via bf16 bit patterns, every GEMV row),
and properties that hold at any size (status word, finiteness) are checked
everywhere.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from model_helpers import encode_workload, sample_indices

pytestmark = pytest.mark.gpu

GEMV_TOL = 2e-3


@pytest.fixture(scope="module")
def entro():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import huffman_decode_canonical_b200 as m
    return m


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)


def _oracle_weights(W, spec):
    w = workloads.weights(W, spec, device="cuda").cpu().numpy()
    q, s, z, scheme = oracle.quantize(w, W.bits, W.quant_mode)
    return q, s, z, scheme


def test_smollm_whole_model_decode_to_bf16(entro):
    """SmolLM-1.7B shapes, mixed unsigned/asymmetric 8-bit: one grouped launch decodes all 169 tensors."""
    W = workloads.get("smollm_1p7b_u8")
    dts, infos, _ = encode_workload(entro, W)
    outs = [torch.empty((d.rows, d.cols), dtype=torch.bfloat16, device="cuda") for d in dts]
    g = entro.Group(dts, entro.GROUP_BF16, outs=outs)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.launch(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    shifted = [i for i, s in enumerate(W.tensors) if s.shifted]
    picks = sorted(set(sample_indices(len(W.tensors), 4) + shifted[:2]))
    for i in picks:
        spec = W.tensors[i]
        q, s, z, scheme = _oracle_weights(W, spec)
        assert infos[i]["scheme"] == scheme and infos[i]["scale"] == s and infos[i]["zero"] == z, spec.name
        assert np.array_equal(_bits(outs[i]), oracle.dequant_bf16(q, s, z)), spec.name


def test_mistral_decode_step_gemv(entro):
    """Mistral-7B shapes, asymmetric 4-bit, row-aligned chunks: the 224 GEMVs of one decode step in one launch."""
    W = workloads.get("mistral_7b_u4")
    dts, infos, _ = encode_workload(entro, W)
    xs = [workloads.activations(W.seed, 1, d.cols).cuda() for d in dts]
    ys = [torch.full((1, d.rows), float("nan"), device="cuda") for d in dts]
    g = entro.Group(dts, entro.GROUP_GEMV, xs=xs, ys=ys, batch=1)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.launch(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert all(torch.isfinite(y).all() for y in ys)
    for i in sample_indices(len(W.tensors), 5):
        spec = W.tensors[i]
        q, s, z, _ = _oracle_weights(W, spec)
        wb = oracle.dequant_bf16(q, s, z).reshape(spec.rows, spec.cols)
        y_ref, mag = oracle.gemv(wb, workloads.bf16_bits(xs[i].cpu()))
        err = np.abs(ys[i].cpu().numpy().astype(np.float64) - y_ref) / np.where(mag > 0, mag, 1.0)
        assert float(err.max()) <= GEMV_TOL, (spec.name, float(err.max()))


@pytest.mark.parametrize("batch", [1, 4, 16])
def test_phi3_gemv_batches(entro, batch):
    """Phi-3-mini shapes, mixed 8-bit, fused GEMV at batch 1, 4 and 16 over the first 8 layers."""
    W = workloads.get("phi3_mini_u8")
    dts, infos, _ = encode_workload(entro, W, limit=32)
    xs = [workloads.activations(W.seed + batch, batch, d.cols).cuda() for d in dts]
    ys = [torch.full((batch, d.rows), float("nan"), device="cuda") for d in dts]
    g = entro.Group(dts, entro.GROUP_GEMV, xs=xs, ys=ys, batch=batch)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.launch(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for i in sample_indices(len(dts), 4):
        spec = W.tensors[i]
        q, s, z, _ = _oracle_weights(W, spec)
        wb = oracle.dequant_bf16(q, s, z).reshape(spec.rows, spec.cols)
        rows = slice(0, min(spec.rows, 512))
        y_ref, mag = oracle.gemv(wb[rows], workloads.bf16_bits(xs[i].cpu()))
        got = ys[i][:, rows].cpu().numpy().astype(np.float64)
        err = np.abs(got - y_ref) / np.where(mag > 0, mag, 1.0)
        assert float(err.max()) <= GEMV_TOL, (spec.name, batch, float(err.max()))


def test_stress_tensors(entro):
    """8192x8192 near-uniform codes (entropy ~7.99 bits) and p(mode)=0.9 skew (the 16-bit limit binds)."""
    W = workloads.get("stress_8192_u8")
    dts, infos, _ = encode_workload(entro, W)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i, spec in enumerate(W.tensors):
        q, s, z, _ = _oracle_weights(W, spec)
        hist = np.bincount(q, minlength=256)
        if spec.law == "skew":
            assert abs(hist.max() / hist.sum() - 0.9) < 5e-4            # p(mode) = 0.9 by construction
            assert int(infos[i]["lengths"].max()) == 16            # the limit binds
        else:
            p = hist[hist > 0] / hist.sum()
            assert float(-(p * np.log2(p)).sum()) > 7.9
        out = dts[i].decode_dequant_bf16(status=st)
        codes = dts[i].decode_codes(status=st)
        x = workloads.activations(7, 1, spec.cols).cuda()
        y = dts[i].decode_gemv(x, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        wb = oracle.dequant_bf16(q, s, z)
        assert np.array_equal(_bits(out), wb)
        assert np.array_equal(codes.cpu().numpy()[: q.size], q)
        rows = slice(0, 256)
        y_ref, mag = oracle.gemv(wb.reshape(spec.rows, spec.cols)[rows], workloads.bf16_bits(x.cpu()))
        err = np.abs(y[:, rows].cpu().numpy().astype(np.float64) - y_ref) / np.where(mag > 0, mag, 1.0)
        assert float(err.max()) <= GEMV_TOL
