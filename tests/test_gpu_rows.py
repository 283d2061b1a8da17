"""GPU parity of the row-tile format (a tile of 32 or 64 rows per chunk, lane = row):
codes and bf16 weights bit for bit against the CPU oracle, the fused GEMV on the
tensor cores within 2e-3 of the oracle's fp64 product, for every batch size 1-16.

Expected values come from the oracle only (quantize -> codes, dequantize -> bf16
bit patterns, fp64 GEMV).  Shapes cover ragged row groups (rows not a multiple of
the tile height), ragged column tiles, tiles narrower than a 4-run MMA group, both
tile heights, 4- and 8-bit codes, codes longer than the 12-bit table (limits 16 and
20) and a binding limit below it (9), and a one-symbol alphabet.  The 32-lane cases
run again in consumption order (format 4), whose layout is checked against the
oracle's bytes before the decode.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

GEMV_TOL = 2e-3


@pytest.fixture(scope="module")
def entro():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import huffman_decode_canonical_b200 as m
    return m


def _pack4(q):
    q = q.astype(np.uint8)
    return (q[0::2] | (q[1::2] << 4)).astype(np.uint8)


def _mode(m):
    return {0: oracle.MODE_AUTO, 1: oracle.MODE_UNSIGNED, 2: oracle.MODE_ASYM}[m]


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


CASES = [
    # kind, bits, mode, max_len, chunk, lanes, rows, cols
    ("laplace", 4, 2, 12, 8192, 32, 100, 1000),     # ragged rows and last column tile (232 wide)
    ("laplace", 4, 2, 12, 8192, 32, 256, 4096),
    ("t4", 8, 0, 16, 4096, 32, 70, 3072),           # mixed quantization, slow path
    ("skew", 8, 2, 16, 512, 32, 33, 24),            # binding limit; 16-column tiles, 24 columns
    ("skew", 8, 2, 20, 2048, 32, 64, 200),          # codes longer than 16 bits: refill per lookup
    ("skew", 8, 2, 9, 1024, 32, 40, 96),            # limit below the table width
    ("uniform", 8, 2, 16, 8192, 32, 48, 512),       # ~8 bits per code
    ("constant", 8, 0, 16, 256, 32, 5, 80),         # one-symbol alphabet
    ("positive", 4, 1, 12, 1024, 32, 30, 72),       # unsigned
    ("two_values", 4, 2, 12, 256, 32, 1, 8),        # one row, one run
    ("laplace", 4, 2, 12, 16384, 64, 130, 520),     # 64-row tiles
    ("t4", 8, 0, 16, 4096, 64, 100, 1024),
    ("skew", 8, 2, 20, 1024, 64, 65, 64),
]


def _ids(c):
    return f"{c[0]}-b{c[1]}-m{c[2]}-L{c[3]}-c{c[4]}-l{c[5]}-{c[6]}x{c[7]}"


def _encode(entro, case, consumption=False):
    kind, bits, mode, lmax, chunk, lanes, rows, cols = case
    w = workloads.small_tensor(kind, rows, cols, seed=rows * 7 + cols)
    q, s, z, _ = oracle.quantize(w, bits, _mode(mode))
    fmt = entro.FORMAT_ROWS_CO if consumption else entro.FORMAT_ROWS
    blob = entro.Blob.encode(w, bits=bits, quant_mode=mode, max_len=lmax, fmt=fmt, chunk_symbols=chunk, lanes=lanes)
    if consumption:   # the stored layout is the oracle's, byte for byte
        assert blob.to_bytes() == oracle.encode(w, bits, _mode(mode), lmax, oracle.FMT_ROWS_CO, chunk, lanes=lanes)
    return entro.upload(blob), q, s, z


# consumption order (format 4): the 32-lane cases
CO_CASES = [c for c in CASES if c[5] == 32]


@pytest.mark.parametrize("consumption", [False, True], ids=["padded", "consumption"])
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_rows_decode_codes_and_bf16(entro, case, consumption):
    bits = case[1]
    if consumption and case[5] != 32:
        pytest.skip("consumption order: 32-lane tiles")
    dt, q, s, z = _encode(entro, case, consumption)
    st = _status()
    codes = dt.decode_codes(status=st)
    bf = dt.decode_dequant_bf16(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    expect = q if bits == 8 else _pack4(q)
    assert np.array_equal(codes.cpu().numpy()[: dt.codes_nbytes()], expect)
    got_bf = bf.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(got_bf, oracle.dequant_bf16(q, s, z))


def _gemv_err(dt, q, s, z, batch, seed):
    x = workloads.activations(seed, batch, dt.cols)
    st = _status()
    y = dt.decode_gemv(x.cuda(), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    wb = oracle.dequant_bf16(q, s, z).reshape(dt.rows, dt.cols)
    y_ref, mag = oracle.gemv(wb, workloads.bf16_bits(x))
    err = np.abs(y.cpu().numpy().astype(np.float64) - y_ref) / np.where(mag > 0, mag, 1.0)
    return float(err.max()), y


@pytest.mark.parametrize("batch", [1, 2, 5, 8, 9, 16])
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_rows_gemv(entro, case, batch):
    dt, q, s, z = _encode(entro, case)
    err, y = _gemv_err(dt, q, s, z, batch, seed=batch)
    assert err <= GEMV_TOL, err
    # fixed summation order: a second call gives the same bits
    err2, y2 = _gemv_err(dt, q, s, z, batch, seed=batch)
    assert torch.equal(y, y2)


@pytest.mark.parametrize("batch", [1, 5, 16])
@pytest.mark.parametrize("case", CO_CASES, ids=[_ids(c) for c in CO_CASES])
def test_rows_consumption_order_gemv(entro, case, batch):
    """The same products from the consumption-order layout: within the tolerance of the
    oracle, and bit for bit the padded layout's (the same codes, the same summation)."""
    dt, q, s, z = _encode(entro, case, consumption=True)
    err, y = _gemv_err(dt, q, s, z, batch, seed=batch)
    assert err <= GEMV_TOL, err
    dt2, _, _, _ = _encode(entro, case)
    _, y2 = _gemv_err(dt2, q, s, z, batch, seed=batch)
    assert torch.equal(y, y2)


def test_rows_consumption_order_needs_32_lanes(entro):
    w = workloads.small_tensor("laplace", 130, 520, seed=1)
    dt = entro.upload(entro.Blob.encode(w, bits=4, fmt=entro.FORMAT_ROWS_CO, chunk_symbols=16384, lanes=64))
    with pytest.raises(entro.EntroError) as e:
        dt.decode_codes(status=_status())
    assert e.value.code == entro.E_INVAL


def test_rows_consumption_order_corrupt(entro):
    """A lane's word count raised far past its words (it runs out of codes with words
    still to take) is reported; a count one too high (its extra word shifts the later
    lanes' words) and random payload bits end with a status, never a hang."""
    w = workloads.small_tensor("laplace", 64, 1024, seed=3)
    blob = entro.Blob.encode(w, bits=4, fmt=entro.FORMAT_ROWS_CO, chunk_symbols=8192)
    for extra, allowed in ((40, (entro.E_CORRUPT, entro.E_OVERRUN)), (1, (0, entro.E_CORRUPT, entro.E_OVERRUN))):
        dt = entro.upload(blob)
        off = _payload_offset(dt)
        dt.mem[off + 5] += extra                      # chunk 0, lane 5's count
        torch.cuda.synchronize()
        st = _status()
        dt.decode_codes(status=st)
        torch.cuda.synchronize()
        assert int(st.item()) in allowed
    dt = entro.upload(blob)
    off = _payload_offset(dt)
    gen = torch.Generator(device="cuda").manual_seed(1)
    dt.mem[off: off + dt.info["payload_bytes"]] = torch.randint(
        0, 256, (dt.info["payload_bytes"],), dtype=torch.uint8, device="cuda", generator=gen)
    torch.cuda.synchronize()
    st = _status()
    dt.decode_dequant_bf16(status=st)
    dt.decode_gemv(workloads.activations(0, 1, 1024).cuda(), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) in (0, entro.E_OVERRUN, entro.E_CORRUPT)


@pytest.mark.parametrize("consumption", [False, True], ids=["padded", "consumption"])
def test_rows_group_gemv_and_bf16(entro, consumption):
    """One grouped launch over tensors of different shapes (row groups split across CTAs)."""
    shapes = [(96, 512), (1000, 256), (33, 3072), (512, 1024)]
    fmt = entro.FORMAT_ROWS_CO if consumption else entro.FORMAT_ROWS
    dts, qs = [], []
    for i, (r, c) in enumerate(shapes):
        w = workloads.small_tensor("laplace", r, c, seed=100 + i)
        q, s, z, _ = oracle.quantize(w, 4, oracle.MODE_ASYM)
        blob = entro.Blob.encode(w, bits=4, quant_mode=entro.QUANT_ASYM, fmt=fmt, chunk_symbols=8192)
        dts.append(entro.upload(blob))
        qs.append((q, s, z))
    for batch in (1, 4, 16):
        xs = [workloads.activations(7, batch, d.cols).cuda() for d in dts]
        ys = [torch.full((batch, d.rows), float("nan"), device="cuda") for d in dts]
        g = entro.Group(dts, entro.GROUP_GEMV, xs=xs, ys=ys, batch=batch)
        st = _status()
        g.launch(status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for d, (q, s, z), x, y in zip(dts, qs, xs, ys):
            wb = oracle.dequant_bf16(q, s, z).reshape(d.rows, d.cols)
            y_ref, mag = oracle.gemv(wb, workloads.bf16_bits(x.cpu()))
            err = np.abs(y.cpu().numpy().astype(np.float64) - y_ref) / np.where(mag > 0, mag, 1.0)
            assert float(err.max()) <= GEMV_TOL
    outs = [torch.empty((d.rows, d.cols), dtype=torch.bfloat16, device="cuda") for d in dts]
    g = entro.Group(dts, entro.GROUP_BF16, outs=outs)
    st = _status()
    g.launch(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for o, (q, s, z) in zip(outs, qs):
        assert np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1),
                              oracle.dequant_bf16(q, s, z))


def test_rows_group_rejects_mixed_formats(entro):
    w = workloads.small_tensor("laplace", 64, 512, seed=3)
    a = entro.upload(entro.Blob.encode(w, bits=4, fmt=entro.FORMAT_ROWS, chunk_symbols=8192))
    b = entro.upload(entro.Blob.encode(w, bits=4, fmt=entro.FORMAT_LANES, chunk_symbols=8192))
    xs = [workloads.activations(0, 1, 512).cuda()] * 2
    ys = [torch.empty((1, 64), device="cuda") for _ in range(2)]
    with pytest.raises(entro.EntroError) as e:
        entro.Group([a, b], entro.GROUP_GEMV, xs=xs, ys=ys, batch=1)
    assert e.value.code == entro.E_INVAL


def test_rows_empty_tensor(entro):
    blob = entro.Blob.encode(np.zeros((0, 64), np.float32), bits=4, fmt=entro.FORMAT_ROWS, chunk_symbols=8192)
    dt = entro.upload(blob)
    st = _status()
    dt.decode_codes(status=st)
    dt.decode_dequant_bf16(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def _payload_offset(dt):
    info = dt.info
    return dt.mem.numel() - ((info["payload_bytes"] + 4 * 64 + 255) // 256) * 256


def test_rows_corrupt_payload_sets_status_without_hanging(entro):
    # one-symbol alphabet: the code is '0', so all-ones words are no code at all
    w = np.full((64, 256), 0.25, np.float32)
    dt = entro.upload(entro.Blob.encode(w, bits=8, fmt=entro.FORMAT_ROWS, chunk_symbols=4096))
    off = _payload_offset(dt)
    dt.mem[off: off + dt.info["payload_bytes"]] = 0xFF
    torch.cuda.synchronize()
    for call in (lambda st: dt.decode_codes(status=st),
                 lambda st: dt.decode_gemv(workloads.activations(0, 1, 256).cuda(), status=st)):
        st = _status()
        call(st)
        torch.cuda.synchronize()
        assert int(st.item()) == entro.E_CORRUPT
    # random payload bits in a complete code: every pattern decodes, lanes may run past their words
    w = workloads.small_tensor("laplace", 64, 1024, seed=3)
    dt = entro.upload(entro.Blob.encode(w, bits=4, fmt=entro.FORMAT_ROWS, chunk_symbols=8192))
    off = _payload_offset(dt)
    gen = torch.Generator(device="cuda").manual_seed(0)
    dt.mem[off: off + dt.info["payload_bytes"]] = torch.randint(
        0, 256, (dt.info["payload_bytes"],), dtype=torch.uint8, device="cuda", generator=gen)
    torch.cuda.synchronize()
    st = _status()
    dt.decode_dequant_bf16(status=st)
    dt.decode_gemv(workloads.activations(0, 1, 1024).cuda(), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) in (0, entro.E_OVERRUN, entro.E_CORRUPT)
