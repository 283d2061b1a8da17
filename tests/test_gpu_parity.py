"""GPU parity: the sm_100a kernels, called through the C ABI, against the CPU oracle.

Expected values come from the oracle only (quantize -> codes, dequantize ->
bf16 bit patterns, fp64 GEMV).  Codes and bf16 weights must match bit for bit;
the fp32-accumulated GEMV must stay within 2e-3 of the fp64 oracle, measured
as max |y_gpu - y_ref| / sum_k |w_k x_k| per output.
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
    if q.size % 2:
        q = np.concatenate([q, np.zeros(1, np.uint8)])
    return (q[0::2] | (q[1::2] << 4)).astype(np.uint8)


def _status(dev="cuda"):
    return torch.zeros(1, dtype=torch.int32, device=dev)


def _oracle_mode(m):
    return {0: oracle.MODE_AUTO, 1: oracle.MODE_UNSIGNED, 2: oracle.MODE_ASYM}[m]


def check_decode(entro, w, bits, mode, max_len, fmt, chunk, lanes=32):
    """Decode codes and bf16 on the GPU; compare with the oracle bit for bit."""
    q, s, z, scheme = oracle.quantize(w, bits, _oracle_mode(mode))
    blob = entro.Blob.encode(w, bits=bits, quant_mode=mode, max_len=max_len, fmt=fmt, chunk_symbols=chunk,
                             lanes=lanes)
    dt = entro.upload(blob)
    st = _status()
    codes = dt.decode_codes(status=st)
    bf = dt.decode_dequant_bf16(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = codes.cpu().numpy()[: dt.codes_nbytes()]
    expect = q if bits == 8 else _pack4(q)
    assert np.array_equal(got, expect)
    ref_bf = oracle.dequant_bf16(q, s, z)
    got_bf = bf.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(got_bf, ref_bf)
    return dt, q, s, z


def gemv_error(y_gpu, y_ref, mag):
    denom = np.where(mag > 0, mag, 1.0)
    return float(np.max(np.abs(y_gpu.astype(np.float64) - y_ref) / denom))


def check_gemv(entro, dt, q, s, z, batch, seed=0):
    K, N = dt.cols, dt.rows
    x = workloads.activations(seed, batch, K)
    st = _status()
    y = dt.decode_gemv(x.cuda(), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    wb = oracle.dequant_bf16(q, s, z).reshape(N, K)
    y_ref, mag = oracle.gemv(wb, workloads.bf16_bits(x))
    err = gemv_error(y.cpu().numpy(), y_ref, mag)
    assert err <= GEMV_TOL, err
    return err


SMALL = [
    # kind, bits, mode, max_len, fmt, chunk, rows, cols
    ("t4", 8, 2, 16, 2, 8192, 64, 128),
    ("t4", 8, 2, 16, 2, 1024, 33, 97),        # ragged last chunk, ragged run
    ("laplace", 4, 2, 12, 2, 8192, 129, 64),
    ("laplace", 4, 2, 12, 2, 512, 7, 131),    # odd n: last packed byte half used
    ("laplace", 4, 2, 12, 2, 16384, 300, 200),
    ("t4", 8, 0, 16, 2, 2048, 100, 100),
    ("shifted", 8, 0, 16, 2, 256, 3, 300),
    ("positive", 4, 1, 12, 2, 1024, 30, 70),
    ("skew", 8, 2, 16, 2, 4096, 200, 100),    # limit binds, slow path
    ("skew", 8, 2, 20, 2, 1024, 64, 100),     # limit above 16: refill per symbol
    ("skew", 8, 2, 9, 2, 1024, 64, 100),      # limit below the table width
    ("uniform", 8, 2, 16, 2, 2048, 40, 64),
    ("constant", 8, 0, 16, 2, 256, 5, 77),    # one-symbol alphabet
    ("two_values", 4, 2, 12, 2, 256, 1, 1),
    ("t4", 8, 2, 16, 1, 4096, 64, 64),        # single stream
    ("t4", 8, 2, 16, 1, 1000, 33, 65),
    ("laplace", 4, 2, 12, 1, 4096, 100, 100),
    ("skew", 8, 2, 16, 1, 512, 50, 50),
    ("zeros", 4, 0, 12, 1, 50, 3, 33),
    ("t4", 8, 2, 16, 1, 16384, 64, 512),      # single stream, chunks at the CTA-per-chunk limit
    ("t4", 8, 2, 16, 1, 20000, 50, 500),      # single stream above it (warp per chunk), ragged
    ("skew", 8, 2, 20, 1, 2048, 64, 100),     # single stream, codes longer than 16 bits
    ("uniform", 8, 2, 16, 1, 4096, 32, 256),  # single stream, ~8 bits per code
    ("laplace", 4, 2, 12, 1, 1024, 33, 97),   # single stream 4-bit, odd n
    ("laplace", 4, 2, 12, 2, -8192, 129, 64),  # 64 lanes (negative chunk marks them)
    ("laplace", 4, 2, 12, 2, -1024, 7, 333),   # 64 lanes, ragged
    ("t4", 8, 0, 16, 2, -2048, 100, 100),
    ("skew", 8, 2, 20, 2, -1024, 64, 100),     # 64 lanes, slow path, refill per symbol
    ("constant", 8, 0, 16, 2, -512, 5, 77),
]


@pytest.mark.parametrize("case", SMALL, ids=[f"{c[0]}-b{c[1]}-m{c[2]}-L{c[3]}-f{c[4]}-c{c[5]}-{c[6]}x{c[7]}"
                                             for c in SMALL])
def test_decode_small_cases(entro, case):
    kind, bits, mode, lmax, fmt, chunk, rows, cols = case
    w = workloads.small_tensor(kind, rows, cols, seed=rows * 7 + cols)
    check_decode(entro, w, bits, mode, lmax, fmt, abs(chunk), lanes=64 if chunk < 0 else 32)


def test_empty_tensor(entro):
    blob = entro.Blob.encode(np.zeros((0, 256), np.float32), bits=8)
    dt = entro.upload(blob)
    st = _status()
    dt.decode_codes(status=st)
    dt.decode_dequant_bf16(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_single_stream_workload(entro):
    """1024x1024 Student-t weights, asymmetric 8-bit, single-stream 4096-symbol chunks."""
    W = workloads.get("t4_1024x1024_u8")
    w = workloads.weights(W, W.tensors[0]).numpy()
    check_decode(entro, w, W.bits, W.quant_mode, W.max_len, W.fmt, W.chunk_symbols(1024))


def test_lanes_workload_and_gemv(entro):
    """4096x4096 Laplace weights, asymmetric 4-bit, 32 lanes per 8192-symbol chunk: codes, bf16, GEMV."""
    W = workloads.get("laplace_4096x4096_u4")
    w = workloads.weights(W, W.tensors[0]).numpy()
    dt, q, s, z = check_decode(entro, w, W.bits, W.quant_mode, W.max_len, W.fmt, W.chunk_symbols(4096))
    check_gemv(entro, dt, q, s, z, batch=1)


@pytest.mark.parametrize("lanes", [32, 64])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("batch", [1, 2, 3, 4, 16])
@pytest.mark.parametrize("shape", [(96, 512), (40, 3072), (24, 14336)])
def test_gemv_shapes_and_batches(entro, bits, batch, shape, lanes):
    rows, cols = shape
    w = workloads.small_tensor("t4" if bits == 8 else "laplace", rows, cols, seed=cols + bits)
    chunk = max(1, 8192 // cols) * cols
    q, s, z, _ = oracle.quantize(w, bits, oracle.MODE_ASYM)
    blob = entro.Blob.encode(w, bits=bits, quant_mode=entro.QUANT_ASYM, chunk_symbols=chunk, lanes=lanes)
    dt = entro.upload(blob)
    check_gemv(entro, dt, q, s, z, batch=batch, seed=batch)


@pytest.mark.parametrize("bits,lanes,batch,shape", [(8, 32, 16, (2405, 8192)), (4, 64, 5, (2406, 3072)),
                                                     (4, 32, 3, (600, 14336))])
def test_gemv_batched_many_warps(entro, bits, lanes, batch, shape):
    """Batched GEMV over enough whole-row chunks for many warps per CTA (16 at K = 8192), so
    chunk groups end part-way through a CTA's warps; two launches give identical results."""
    rows, cols = shape
    w = workloads.small_tensor("t4" if bits == 8 else "laplace", rows, cols, seed=rows + bits)
    chunk = max(1, 8192 // cols) * cols
    q, s, z, _ = oracle.quantize(w, bits, oracle.MODE_ASYM)
    dt = entro.upload(entro.Blob.encode(w, bits=bits, quant_mode=entro.QUANT_ASYM, chunk_symbols=chunk,
                                        lanes=lanes))
    x = workloads.activations(bits + batch, batch, cols)
    st = _status()
    y1 = dt.decode_gemv(x.cuda(), status=st)
    y2 = dt.decode_gemv(x.cuda(), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(y1, y2)
    y_ref, mag = oracle.gemv(oracle.dequant_bf16(q, s, z).reshape(rows, cols), workloads.bf16_bits(x))
    assert gemv_error(y1.cpu().numpy(), y_ref, mag) <= GEMV_TOL


@pytest.mark.parametrize("batch", [4, 16])
def test_gemv_batched_partial_last_chunk(entro, batch):
    """33 rows in chunks of 2 rows: the last chunk is half a chunk (the CUDA-core batched path)."""
    w = workloads.small_tensor("t4", 33, 3072, seed=33)
    q, s, z, _ = oracle.quantize(w, 8, oracle.MODE_ASYM)
    dt = entro.upload(entro.Blob.encode(w, bits=8, quant_mode=entro.QUANT_ASYM, chunk_symbols=6144))
    check_gemv(entro, dt, q, s, z, batch=batch, seed=batch)


def test_gemv_rejects_unsupported_layouts(entro):
    w = workloads.small_tensor("t4", 16, 300, seed=0)
    dt = entro.upload(entro.Blob.encode(w, bits=8, chunk_symbols=4096))
    with pytest.raises(entro.EntroError):
        dt.decode_gemv(torch.zeros((1, 300), dtype=torch.bfloat16, device="cuda"))
    w = workloads.small_tensor("t4", 16, 256, seed=0)
    dt = entro.upload(entro.Blob.encode(w, bits=8, chunk_symbols=768))     # 3 rows per chunk is fine
    dt.decode_gemv(torch.zeros((1, 256), dtype=torch.bfloat16, device="cuda"))
    dt = entro.upload(entro.Blob.encode(w, bits=8, chunk_symbols=512, fmt=entro.FORMAT_SINGLE))
    with pytest.raises(entro.EntroError):
        dt.decode_gemv(torch.zeros((1, 256), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(entro.EntroError):
        dt.decode_gemv(torch.zeros((17, 256), dtype=torch.bfloat16, device="cuda"))


def test_group_gemv_and_bf16(entro):
    shapes = [(64, 256), (32, 512), (128, 1024), (16, 3072), (8, 8192)]
    xs, ys, outs, dts, refs = [], [], [], [], []
    for i, (r, c) in enumerate(shapes):
        w = workloads.small_tensor("laplace", r, c, seed=i)
        q, s, z, _ = oracle.quantize(w, 4, oracle.MODE_ASYM)
        dt = entro.upload(entro.Blob.encode(w, bits=4, quant_mode=entro.QUANT_ASYM,
                                            chunk_symbols=max(1, 8192 // c) * c))
        x = workloads.activations(i, 2, c)
        wb = oracle.dequant_bf16(q, s, z)
        refs.append((oracle.gemv(wb.reshape(r, c), workloads.bf16_bits(x)), wb))
        dts.append(dt)
        xs.append(x.cuda())
        ys.append(torch.full((2, r), float("nan"), device="cuda"))
        outs.append(torch.empty((r, c), dtype=torch.bfloat16, device="cuda"))
    g = entro.Group(dts, entro.GROUP_GEMV, xs=xs, ys=ys, batch=2)
    gb = entro.Group(dts, entro.GROUP_BF16, outs=outs)
    st = _status()
    for _ in range(2):                      # launches are repeatable
        g.launch(status=st)
        gb.launch(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for y, o, ((y_ref, mag), wb) in zip(ys, outs, refs):
        assert gemv_error(y.cpu().numpy(), y_ref, mag) <= GEMV_TOL
        assert np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1), wb)


def test_corrupt_device_data_sets_status_without_hanging(entro):
    # one-symbol alphabet: the code is '0', so all-ones words are no code at all
    w = np.full((64, 256), 0.25, np.float32)
    dt = entro.upload(entro.Blob.encode(w, bits=8, chunk_symbols=4096))
    info = dt.info
    payload_off = dt.mem.numel() - ((info["payload_bytes"] + 4 * 64 + 255) // 256) * 256
    dt.mem[payload_off: payload_off + info["payload_bytes"]] = 0xFF
    torch.cuda.synchronize()  # a device image changes only between decode launches (launch overlap contract)
    st = _status()
    dt.decode_codes(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == entro.E_CORRUPT
    # random payload bits in a complete code: every pattern decodes, lanes run past their words
    w = workloads.small_tensor("laplace", 64, 1024, seed=3)
    dt = entro.upload(entro.Blob.encode(w, bits=4, quant_mode=entro.QUANT_ASYM, chunk_symbols=8192))
    info = dt.info
    payload_off = dt.mem.numel() - ((info["payload_bytes"] + 4 * 64 + 255) // 256) * 256
    gen = torch.Generator(device="cuda").manual_seed(0)
    dt.mem[payload_off: payload_off + info["payload_bytes"]] = torch.randint(
        0, 256, (info["payload_bytes"],), dtype=torch.uint8, device="cuda", generator=gen)
    torch.cuda.synchronize()
    st = _status()
    bf = dt.decode_dequant_bf16(status=st)
    torch.cuda.synchronize()
    code = int(st.item())
    assert code in (0, entro.E_OVERRUN, entro.E_CORRUPT)
    if code == 0:   # decoded without a complaint: then not to the original weights
        q, s, z, _ = oracle.quantize(w, 4, oracle.MODE_ASYM)
        got = bf.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)
        assert not np.array_equal(got, oracle.dequant_bf16(q, s, z))


def test_decode_is_deterministic(entro):
    W = workloads.get("laplace_4096x4096_u4")
    w = workloads.weights(W, W.tensors[0]).numpy()[:1024]
    dt = entro.upload(entro.Blob.encode(w, bits=4, quant_mode=entro.QUANT_ASYM, chunk_symbols=8192))
    x = workloads.activations(1, 1, 4096).cuda()
    y1 = dt.decode_gemv(x).clone()
    y2 = dt.decode_gemv(x)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_launch_configs_do_not_shrink_each_other(entro):
    """A launch needing more shared memory, then one needing less, then the first again."""
    big = workloads.small_tensor("uniform", 64, 4096, seed=1)        # ~8 bits/code: long lanes
    small = workloads.small_tensor("skew", 64, 4096, seed=2)         # short lanes
    dts = [entro.upload(entro.Blob.encode(w, bits=8, quant_mode=entro.QUANT_ASYM, chunk_symbols=8192))
           for w in (big, small)]
    assert dts[0].info["max_chunk_words"] > dts[1].info["max_chunk_words"]
    st = _status()
    outs = [dts[i].decode_dequant_bf16(status=st) for i in (0, 1, 0, 1)]
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(outs[0], outs[2]) and torch.equal(outs[1], outs[3])
