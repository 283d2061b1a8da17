"""Full-size parity on the model-shaped workloads, every tensor of every model.

* Codes and bf16 weights: the GPU's decode of every tensor is compared bit for bit
  with the oracle's quantization (codes) and dequantization (bf16) of the same
  seeded tensor.  SmolLM-shaped: the whole model in one grouped bf16 launch (the
  benchmark's launch); Mistral- and Phi-3-shaped: codes and bf16 of every tensor.
* Fused GEMV: one grouped launch over every tensor of the model (the benchmark's
  decode step), at each batch size of the configuration; sampled rows of every
  tensor (first, last and evenly spaced) against the oracle's fp64 product of the
  oracle's bf16 weights, within 2e-3 of sum |w x|.

The oracle's work for a tensor (quantize, dequantize, compare) runs on worker
threads while the GPU decodes the next tensor.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import workloads
from model_helpers import encode_workload

pytestmark = pytest.mark.gpu

GEMV_TOL = 2e-3
SAMPLE_ROWS = 16


@pytest.fixture(scope="module")
def entro():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import huffman_decode_canonical_b200 as m
    return m


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)


def _pack4(q):
    return (q[0::2] | (q[1::2] << 4)).astype(np.uint8)


def _sample_rows(rows):
    return np.unique(np.linspace(0, rows - 1, min(rows, SAMPLE_ROWS)).round().astype(np.int64))


def _check_tensor(W, spec, w, info, got_bf, got_codes):
    q, s, z, scheme = oracle.quantize(w, W.bits, W.quant_mode)
    assert (info["scheme"], info["scale"], info["zero"]) == (scheme, s, z), spec.name
    ref = oracle.dequant_bf16(q, s, z)
    assert np.array_equal(got_bf, ref), spec.name
    if got_codes is not None:
        assert np.array_equal(got_codes, q if W.bits == 8 else _pack4(q)), spec.name
    rows = _sample_rows(spec.rows)
    return rows, ref.reshape(spec.rows, spec.cols)[rows]


def _decode_and_check(entro, W, dts, infos, codes=True, bf16_group=False):
    """Decode every tensor on the GPU and check it against the oracle; returns the sampled
    rows of every tensor for the GEMV checks."""
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = None
    if bf16_group:
        outs = [torch.empty((d.rows, d.cols), dtype=torch.bfloat16, device="cuda") for d in dts]
        entro.Group(dts, entro.GROUP_BF16, outs=outs).launch(status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
    samples = [None] * len(dts)
    pending = []
    with ThreadPoolExecutor(8) as pool:
        for i, (spec, dt) in enumerate(zip(W.tensors, dts)):
            w = workloads.weights(W, spec, device="cuda").cpu().numpy()
            if outs is not None:
                got_bf = _bits(outs[i])
                outs[i] = None
            else:
                got_bf = _bits(dt.decode_dequant_bf16(status=st))
            got_codes = dt.decode_codes(status=st).cpu().numpy()[: dt.codes_nbytes()] if codes else None
            torch.cuda.synchronize()
            assert int(st.item()) == 0, spec.name
            pending.append((i, pool.submit(_check_tensor, W, spec, w, infos[i], got_bf, got_codes)))
            del w, got_bf, got_codes
            while len(pending) > 8:
                j, f = pending.pop(0)
                samples[j] = f.result()
        for j, f in pending:
            samples[j] = f.result()
    return samples


def _gemv_check(entro, W, dts, samples, batch):
    """One grouped launch over every tensor (the benchmark's step); sampled rows of every
    tensor against the oracle.  Tensors with the same column count share activations."""
    xs = {K: workloads.activations(W.seed + batch, batch, K).cuda() for K in set(d.cols for d in dts)}
    ys = [torch.full((batch, d.rows), float("nan"), device="cuda") for d in dts]
    g = entro.Group(dts, entro.GROUP_GEMV, xs=[xs[d.cols] for d in dts], ys=ys, batch=batch)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.launch(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    xbits = {K: workloads.bf16_bits(x.cpu()) for K, x in xs.items()}
    worst = 0.0
    for spec, d, y, (rows, wb) in zip(W.tensors, dts, ys, samples):
        assert torch.isfinite(y).all(), spec.name
        y_ref, mag = oracle.gemv(wb, xbits[d.cols])
        got = y[:, torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
        err = float((np.abs(got - y_ref) / np.where(mag > 0, mag, 1.0)).max())
        assert err <= GEMV_TOL, (spec.name, batch, err)
        worst = max(worst, err)
    return worst


def test_smollm_whole_model_decode_to_bf16(entro):
    """SmolLM-1.7B shapes, mixed unsigned/asymmetric 8-bit: one grouped launch decodes all
    169 tensors to bf16; every tensor bit-exact."""
    W = workloads.get("smollm_1p7b_u8")
    dts, infos, _ = encode_workload(entro, W)
    _decode_and_check(entro, W, dts, infos, codes=False, bf16_group=True)


def test_mistral_every_tensor_and_decode_step(entro):
    """Mistral-7B shapes, asymmetric 4-bit: codes and bf16 of all 224 tensors bit-exact, and the
    decode step's fused GEMV (one launch over every tensor) at batch 1, 4 and 16."""
    W = workloads.get("mistral_7b_u4")
    dts, infos, _ = encode_workload(entro, W)
    samples = _decode_and_check(entro, W, dts, infos)
    for batch in (1, 4, 16):
        _gemv_check(entro, W, dts, samples, batch)


def test_phi3_every_tensor_and_gemv_batches(entro):
    """Phi-3-mini shapes, mixed 8-bit: codes and bf16 of all 128 tensors bit-exact, and the fused
    GEMV over every tensor at batch 1, 4 and 16."""
    W = workloads.get("phi3_mini_u8")
    dts, infos, _ = encode_workload(entro, W)
    samples = _decode_and_check(entro, W, dts, infos)
    for batch in (1, 4, 16):
        _gemv_check(entro, W, dts, samples, batch)


def test_stress_tensors(entro):
    """8192x8192 near-uniform codes (entropy ~7.99 bits) and p(mode)=0.9 skew (the 16-bit limit
    binds): codes and bf16 bit-exact, GEMV on sampled rows."""
    W = workloads.get("stress_8192_u8")
    dts, infos, _ = encode_workload(entro, W)
    for i, spec in enumerate(W.tensors):
        q, s, z, _ = oracle.quantize(workloads.weights(W, spec, device="cuda").cpu().numpy(), W.bits, W.quant_mode)
        hist = np.bincount(q, minlength=256)
        if spec.law == "skew":
            assert abs(hist.max() / hist.sum() - 0.9) < 5e-4            # p(mode) = 0.9 by construction
            assert int(infos[i]["lengths"].max()) == 16            # the limit binds
        else:
            p = hist[hist > 0] / hist.sum()
            assert float(-(p * np.log2(p)).sum()) > 7.9
    samples = _decode_and_check(entro, W, dts, infos)
    _gemv_check(entro, W, dts, samples, 1)
