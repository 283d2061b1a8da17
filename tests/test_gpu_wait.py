"""The bounded waits: a kernel whose copy barrier never completes gives up, reports
ENTRO_E_TIMEOUT in the status word and returns, and the context stays usable.

The stall is made on the host: the library's test hook makes every launch declare
more bytes on its decode-table barrier than the copy delivers (a wait that nothing
satisfies).  No GPU fault, trap or endless loop is involved; each wait gives up
after about a second.
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
    return m


@pytest.mark.parametrize("fmt", ["lanes", "rows", "single"])
def test_stalled_table_copy_times_out_and_context_survives(entro, fmt):
    w = workloads.small_tensor("laplace", 64, 1024, seed=9)
    f = {"lanes": entro.FORMAT_LANES, "rows": entro.FORMAT_ROWS, "single": entro.FORMAT_SINGLE}[fmt]
    dt = entro.upload(entro.Blob.encode(w, bits=4, quant_mode=entro.QUANT_ASYM, fmt=f,
                                        chunk_symbols=8192 if fmt != "single" else 4096))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    prev = entro.test_stall_tables(16)
    try:
        dt.decode_dequant_bf16(status=st)
        torch.cuda.synchronize()
    finally:
        entro.test_stall_tables(prev)
    assert int(st.item()) == entro.E_TIMEOUT
    # the same decode without the stall is whole and bit-exact
    q, s, z, _ = oracle.quantize(w, 4, oracle.MODE_ASYM)
    st.zero_()
    bf = dt.decode_dequant_bf16(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(bf.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1),
                          oracle.dequant_bf16(q, s, z))
