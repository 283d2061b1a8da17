"""The grouped fused GEMV that allocates nothing (its work table lives in a fixed
array inside the library), for callers that may not allocate device memory.

Runs last (file name) so that a failure here does not hide the other tests.  It
must pass in a fresh process -- where its first call sets the table's device
address up -- and after every other test.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

GEMV_TOL = 2e-3   # the GEMV tolerance of the parity tests, relative to sum_k |w_k x_k|


def test_static_group_gemv_matches_group_launch():
    """Five tensors of different shapes: the fixed-table GEMV within the tolerance of the
    oracle's fp64 product and bit-identical to the grouped launch, on two calls in a row;
    more tensors than the table holds -> E_LIMIT."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import huffman_decode_canonical_b200 as entro

    import oracle
    shapes = [(64, 256), (48, 1024), (16, 3072), (8, 8192), (96, 512)]
    batch = 3
    dts, xs, ys_ref, ys_new, refs = [], [], [], [], []
    for i, (r, c) in enumerate(shapes):
        w = workloads.small_tensor("laplace", r, c, seed=40 + i)
        dt = entro.upload(entro.Blob.encode(w, bits=4, quant_mode=entro.QUANT_ASYM,
                                            chunk_symbols=max(1, 8192 // c) * c))
        x = workloads.activations(i, batch, c)
        q, s, z, _ = oracle.quantize(w, 4, oracle.MODE_ASYM)
        refs.append(oracle.gemv(oracle.dequant_bf16(q, s, z).reshape(r, c), workloads.bf16_bits(x)))
        x = x.cuda()
        dts.append(dt)
        xs.append(x)
        ys_ref.append(torch.empty((batch, r), dtype=torch.float32, device="cuda"))
        ys_new.append(torch.full((batch, r), float("nan"), dtype=torch.float32, device="cuda"))
    ref = entro.Group(dts, entro.GROUP_GEMV, xs=xs, ys=ys_ref, batch=batch)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref.launch(status=st)
    for call in range(2):                         # two calls in a row reuse the one table
        for y in ys_new:
            y.fill_(float("nan"))
        entro.decode_gemv_group_static(dts, xs, ys_new, batch=batch, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for a, b, (y_ref, m) in zip(ys_new, ys_ref, refs):
            err = np.abs(a.cpu().numpy().astype(np.float64) - y_ref) / np.where(m > 0, m, 1.0)
            assert np.isfinite(err).all() and float(err.max()) <= GEMV_TOL, (call, float(err.max()))
            assert torch.equal(a, b)                  # the same kernel on the same table contents
    too_many = [dts[0]] * (entro.STATIC_GROUP_MAX + 1)
    with pytest.raises(entro.EntroError) as e:
        entro.decode_gemv_group_static(too_many, [xs[0]] * len(too_many), [ys_new[0]] * len(too_many),
                                       batch=batch)
    assert e.value.code == entro.E_LIMIT


@pytest.mark.parametrize("fmt", ["lanes", "rows", "rows_co"])
def test_static_group_gemv_many_tensors_against_oracle(fmt):
    """70 small tensors: the fixed table is filled in three host-to-device copies of up to
    32 entries, so the later copies' offsets and running chunk and symbol counts are used.
    Checked against the oracle's fp64 product and against the grouped launch, twice."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import oracle
    import huffman_decode_canonical_b200 as entro

    f = {"rows": entro.FORMAT_ROWS, "rows_co": entro.FORMAT_ROWS_CO, "lanes": entro.FORMAT_LANES}[fmt]
    batch = 2
    dts, xs, refs = [], [], []
    for i in range(70):
        r, c = 8 + 8 * (i % 5), 256 * (1 + i % 3)
        w = workloads.small_tensor("laplace", r, c, seed=200 + i)
        q, s, z, _ = oracle.quantize(w, 4, oracle.MODE_ASYM)
        dt = entro.upload(entro.Blob.encode(w, bits=4, quant_mode=entro.QUANT_ASYM, fmt=f,
                                            chunk_symbols=8192 if fmt != "lanes" else max(1, 8192 // c) * c))
        x = workloads.activations(300 + i, batch, c)
        refs.append(oracle.gemv(oracle.dequant_bf16(q, s, z).reshape(r, c), workloads.bf16_bits(x)))
        dts.append(dt)
        xs.append(x.cuda())
    ys_group = [torch.empty((batch, d.rows), dtype=torch.float32, device="cuda") for d in dts]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    entro.Group(dts, entro.GROUP_GEMV, xs=xs, ys=ys_group, batch=batch).launch(status=st)
    for call in range(2):
        ys = [torch.full((batch, d.rows), float("nan"), dtype=torch.float32, device="cuda") for d in dts]
        entro.decode_gemv_group_static(dts, xs, ys, batch=batch, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for y, yg, (y_ref, mag) in zip(ys, ys_group, refs):
            err = np.abs(y.cpu().numpy().astype(np.float64) - y_ref) / np.where(mag > 0, mag, 1.0)
            assert np.isfinite(err).all() and float(err.max()) <= GEMV_TOL, (call, float(err.max()))
            assert torch.equal(y, yg)                 # the same kernel on the same table contents
