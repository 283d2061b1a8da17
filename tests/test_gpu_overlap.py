"""Launch overlap (programmatic dependent launch) changes no result.

With overlap on, a decode kernel may start while the kernel before it on the
stream is finishing; it reads only the tensor's device image until that kernel
has completed.  Checked here: back-to-back decodes of several tensors and
formats give the same bits as with overlap off, and a GEMV whose activations
are written by a torch kernel launched just before it sees those activations.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def entro():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import huffman_decode_canonical_b200 as m
    prev = m.set_overlap(False)
    yield m
    m.set_overlap(prev)


def _tensors(entro):
    specs = [("laplace", 4, 4096, 512, 8192, entro.FORMAT_LANES), ("t4", 8, 96, 3072, 6144, entro.FORMAT_LANES),
             ("t4", 8, 64, 1024, 4096, entro.FORMAT_SINGLE), ("skew", 8, 256, 512, 8192, entro.FORMAT_LANES)]
    out = []
    for i, (kind, bits, rows, cols, chunk, fmt) in enumerate(specs):
        w = workloads.small_tensor(kind, rows, cols, seed=40 + i)
        blob = entro.Blob.encode(w, bits=bits, quant_mode=entro.QUANT_ASYM, chunk_symbols=chunk, fmt=fmt)
        out.append((entro.upload(blob), fmt, w, bits))
    return out


def _run(entro, tensors, st):
    res = []
    for dt, fmt, _, _ in tensors:
        res.append(dt.decode_codes(status=st))
        res.append(dt.decode_dequant_bf16(status=st))
        if fmt == entro.FORMAT_LANES:
            for batch in (1, 4):
                xb = workloads.activations(7, batch, dt.cols).cuda()
                x = (xb.float() * 0.5).to(torch.bfloat16)  # written by a torch kernel just before the GEMV
                res.append(dt.decode_gemv(x, status=st))
    return res


def test_overlap_gives_identical_results(entro):
    tensors = _tensors(entro)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    entro.set_overlap(False)
    ref = [r.clone() for r in _run(entro, tensors, st)]
    torch.cuda.synchronize()
    entro.set_overlap(True)
    try:
        for _ in range(3):
            got = _run(entro, tensors, st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            for a, b in zip(ref, got):
                assert torch.equal(a, b)
    finally:
        entro.set_overlap(False)


def test_overlap_gemv_reads_activations_written_just_before(entro):
    """y(-x) must be exactly -y(x): the second GEMV's x is negated in place by a torch
    kernel launched right before it."""
    w = workloads.small_tensor("laplace", 512, 4096, seed=5)
    q, s, z, _ = oracle.quantize(w, 4, oracle.MODE_ASYM)
    dt = entro.upload(entro.Blob.encode(w, bits=4, quant_mode=entro.QUANT_ASYM, chunk_symbols=8192))
    x = workloads.activations(3, 2, 4096).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    entro.set_overlap(True)
    try:
        y1 = dt.decode_gemv(x, status=st).clone()
        x.mul_(-1)
        y2 = dt.decode_gemv(x, status=st)
        torch.cuda.synchronize()
    finally:
        entro.set_overlap(False)
    assert int(st.item()) == 0
    assert torch.equal(y2, -y1)
    wb = oracle.dequant_bf16(q, s, z).reshape(512, 4096)
    y_ref, mag = oracle.gemv(wb, workloads.bf16_bits(x.cpu()))
    err = np.abs(y2.cpu().numpy().astype(np.float64) - y_ref) / np.where(mag > 0, mag, 1.0)
    assert float(err.max()) <= 2e-3
