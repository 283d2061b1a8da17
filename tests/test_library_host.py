"""CPU tests of libentro: the C ABI loads and exports every declared symbol, and
the host encoder writes blobs byte-identical to the oracle's (same format, same
quantization, same package-merge tie rule) without sharing any code with it."""
import os
import re

import numpy as np
import pytest

import oracle
import workloads
import huffman_decode_canonical_b200 as entro

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "entro.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"ENTRO_API[^;(]*?\b(entro_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    declared = _declared_symbols()
    assert len(declared) >= 15
    lib = entro.lib()
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(entro.EXPORTS) == declared
    assert entro.version() == 100
    assert entro._strerror(entro.E_CORRUPT).startswith("corrupt")


_MODE = {oracle.MODE_AUTO: entro.QUANT_AUTO, oracle.MODE_UNSIGNED: entro.QUANT_UNSIGNED,
         oracle.MODE_ASYM: entro.QUANT_ASYM}

CASES = [
    ("t4", 8, oracle.MODE_ASYM, 16, 1, 4096, 64, 64),
    ("t4", 8, oracle.MODE_ASYM, 16, 1, 1000, 33, 65),
    ("t4", 8, oracle.MODE_ASYM, 16, 1, 1, 3, 5),
    ("laplace", 4, oracle.MODE_ASYM, 12, 2, 8192, 128, 96),
    ("laplace", 4, oracle.MODE_ASYM, 12, 2, 512, 7, 131),
    ("laplace", 4, oracle.MODE_ASYM, 12, 1, 4096, 128, 96),
    ("t4", 8, oracle.MODE_AUTO, 16, 2, 768, 50, 51),
    ("shifted", 8, oracle.MODE_AUTO, 16, 2, 256, 3, 300),
    ("positive", 8, oracle.MODE_AUTO, 16, 2, 1024, 30, 70),
    ("positive", 4, oracle.MODE_UNSIGNED, 12, 2, 1024, 30, 70),
    ("skew", 8, oracle.MODE_ASYM, 16, 2, 16384, 200, 100),
    ("skew", 8, oracle.MODE_ASYM, 9, 2, 1024, 20, 100),
    ("skew", 8, oracle.MODE_ASYM, 20, 2, 1024, 20, 100),
    ("uniform", 8, oracle.MODE_ASYM, 16, 2, 2048, 40, 64),
    ("constant", 8, oracle.MODE_AUTO, 16, 2, 256, 5, 77),
    ("zeros", 4, oracle.MODE_AUTO, 12, 1, 50, 3, 33),
    ("two_values", 4, oracle.MODE_ASYM, 12, 2, 256, 1, 1),
    ("t4", 4, oracle.MODE_ASYM, 4, 2, 512, 9, 100),
    ("t4", 8, oracle.MODE_ASYM, 16, 2, 256, 0, 16),
    ("laplace", 4, oracle.MODE_ASYM, 12, 2, -1024, 7, 333),     # 64 lanes (negative chunk marks them)
    ("t4", 8, oracle.MODE_AUTO, 16, 2, -6144, 20, 3072),
    ("skew", 8, oracle.MODE_ASYM, 16, 2, -14336, 3, 14336),
    ("laplace", 4, oracle.MODE_ASYM, 12, 3, 8192, 100, 1000),     # row tiles, ragged both ways
    ("t4", 8, oracle.MODE_AUTO, 16, 3, 4096, 70, 3072),
    ("skew", 8, oracle.MODE_ASYM, 16, 3, 512, 33, 24),
    ("laplace", 4, oracle.MODE_ASYM, 12, 3, -1024, 130, 520),    # 64-row tiles
    ("t4", 8, oracle.MODE_ASYM, 16, 3, 256, 0, 16),
    ("laplace", 4, oracle.MODE_ASYM, 12, 4, 8192, 100, 1000),     # row tiles in consumption order
    ("t4", 8, oracle.MODE_AUTO, 16, 4, 4096, 70, 3072),
    ("skew", 8, oracle.MODE_ASYM, 16, 4, 512, 33, 24),
    ("skew", 8, oracle.MODE_ASYM, 20, 4, 2048, 64, 200),          # refill before every lookup
    ("laplace", 4, oracle.MODE_ASYM, 12, 4, -1024, 130, 520),
    ("constant", 8, oracle.MODE_AUTO, 16, 4, 256, 5, 80),
    ("t4", 8, oracle.MODE_ASYM, 16, 4, 256, 0, 16),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-b{c[1]}-m{c[2]}-L{c[3]}-f{c[4]}-c{c[5]}-{c[6]}x{c[7]}"
                                             for c in CASES])
def test_encoder_blob_identical_to_oracle(case):
    kind, bits, mode, lmax, fmt, chunk, rows, cols = case
    lanes = 64 if chunk < 0 else 32
    chunk = abs(chunk)
    w = workloads.small_tensor(kind, max(rows, 1), cols, seed=rows * 7 + cols)[:rows]
    ref = oracle.encode(w, bits, mode, lmax, fmt, chunk, lanes=lanes)
    for threads in (1, 3):
        blob = entro.Blob.encode(w, bits=bits, quant_mode=_MODE[mode], max_len=lmax, fmt=fmt,
                                 chunk_symbols=chunk, threads=threads, lanes=lanes)
        got = blob.to_bytes()
        assert len(got) == len(ref)
        assert got == ref
    info = blob.info()
    prm = oracle.params(ref)
    for k in ("bits", "scheme", "max_len", "format", "rows", "cols", "n", "chunk_symbols", "n_chunks", "lanes"):
        assert info[k] == prm[k], k
    assert info["scale"] == prm["scale"] and info["zero"] == prm["zero"]
    assert (info["lengths"] == prm["lengths"]).all()
    q = oracle.quantize(w, bits, mode)[0]
    hist = np.bincount(q, minlength=256)
    assert info["coded_bits"] == int((hist * prm["lengths"].astype(np.int64)).sum())


@pytest.mark.parametrize("name", ["t4_1024x1024_u8", "laplace_4096x4096_u4"])
def test_encoder_identical_on_single_tensor_workloads(name):
    W = workloads.get(name)
    spec = W.tensors[0]
    w = workloads.weights(W, spec).numpy()
    C = W.chunk_symbols(spec.cols)
    ref = oracle.encode(w, W.bits, W.quant_mode, W.max_len, W.fmt, C)
    got = entro.Blob.encode(w, bits=W.bits, quant_mode=W.quant_mode, max_len=W.max_len, fmt=W.fmt,
                            chunk_symbols=C).to_bytes()
    assert got == ref


@pytest.mark.parametrize("consumption", [False, True], ids=["padded", "consumption"])
@pytest.mark.parametrize("name,index,rows", [("phi3_mini_u8", 1, 512), ("mistral_7b_u4", 6, 96)])
def test_encoder_identical_on_model_shaped_tensor(name, index, rows, consumption):
    """Model-shaped tensors in their workload's row-tile format (and in consumption order): a
    Phi-3-mini-shaped o projection (3072 columns, 32 x 128 tiles) and a Mistral-shaped down
    projection (14336 columns, 32 x 256 tiles, a ragged last row group)."""
    W = workloads.get(name)
    spec = W.tensors[index]
    w = workloads.weights(W, spec).numpy()[:rows]
    C = W.chunk_symbols(spec.cols)
    assert W.fmt == oracle.FMT_ROWS
    fmt = oracle.FMT_ROWS_CO if consumption else W.fmt
    ref = oracle.encode(w, W.bits, W.quant_mode, W.max_len, fmt, C, lanes=W.lanes)
    got = entro.Blob.encode(w, bits=W.bits, quant_mode=W.quant_mode, max_len=W.max_len, fmt=fmt,
                            chunk_symbols=C, lanes=W.lanes).to_bytes()
    assert got == ref


def test_encoder_errors_match_oracle():
    bad = np.array([[0.0, np.nan]], np.float32)
    with pytest.raises(entro.EntroError) as e:
        entro.Blob.encode(bad, bits=8)
    assert e.value.code == entro.E_INVAL
    with pytest.raises(oracle.OracleError):
        oracle.encode(bad, 8, oracle.MODE_ASYM, 16, 2, 256)
    neg = np.array([[-1.0, 1.0]], np.float32)
    with pytest.raises(entro.EntroError):
        entro.Blob.encode(neg, bits=8, quant_mode=entro.QUANT_UNSIGNED)
    many = np.linspace(-1, 1, 4096, dtype=np.float32).reshape(16, 256)   # 256 distinct 8-bit codes
    with pytest.raises(entro.EntroError) as e:
        entro.Blob.encode(many, bits=8, max_len=7)
    assert e.value.code == entro.E_LIMIT
    with pytest.raises(oracle.OracleError):
        oracle.encode(many, 8, oracle.MODE_ASYM, 7, 2, 256)
    for kw in ({"bits": 5}, {"fmt": 5}, {"chunk_symbols": 300}, {"chunk_symbols": 32768}, {"max_len": 25},
               {"lanes": 48}, {"lanes": 64, "chunk_symbols": 768}, {"fmt": 3, "chunk_symbols": 300}):
        with pytest.raises(entro.EntroError):
            entro.Blob.encode(many, **kw)
    # row tiles need whole runs of 8 columns
    odd = workloads.small_tensor("t4", 8, 12, seed=3)
    with pytest.raises(entro.EntroError) as e:
        entro.Blob.encode(odd, bits=8, fmt=entro.FORMAT_ROWS, chunk_symbols=256)
    assert e.value.code == entro.E_INVAL
    with pytest.raises(oracle.OracleError):
        oracle.encode(odd, 8, oracle.MODE_ASYM, 16, oracle.FMT_ROWS, 256)


def test_blob_bytes_roundtrip_and_validation():
    w = workloads.small_tensor("laplace", 40, 512, seed=1)
    blob = entro.Blob.encode(w, bits=4, quant_mode=entro.QUANT_ASYM, chunk_symbols=1024)
    data = blob.to_bytes()
    again = entro.Blob.from_bytes(data)
    assert again.to_bytes() == data
    assert again.info()["max_chunk_words"] == blob.info()["max_chunk_words"]
    # header, lengths, index and size are all checked
    for off, val in ((0, 0), (8, 5), (128 + 3, 13), (384 + 16, 7)):
        bad = bytearray(data)
        bad[off] = val
        with pytest.raises(entro.EntroError) as e:
            entro.Blob.from_bytes(bytes(bad))
        assert e.value.code == entro.E_FORMAT
    with pytest.raises(entro.EntroError):
        entro.Blob.from_bytes(data[:-4])


def test_consumption_order_blob_validation():
    """A consumption-order blob round-trips through bytes; a chunk whose word count is not a
    whole number of 16-byte groups, or smaller than its header and first three rows, is
    refused before anything reaches a device."""
    w = workloads.small_tensor("laplace", 64, 1024, seed=4)
    blob = entro.Blob.encode(w, bits=4, quant_mode=entro.QUANT_ASYM, fmt=entro.FORMAT_ROWS_CO, chunk_symbols=8192)
    data = blob.to_bytes()
    again = entro.Blob.from_bytes(data)
    assert again.to_bytes() == data and again.info()["format"] == entro.FORMAT_ROWS_CO
    info = blob.info()
    # max_chunk_words: the staging rows a chunk needs (its words over 32 lanes, rounded up)
    idx = np.frombuffer(data, np.uint64, 2 * (info["n_chunks"] + 1), 384).reshape(-1, 2)
    sizes = np.diff(idx[:, 0].astype(np.int64))
    assert info["max_chunk_words"] == int(-(-sizes.max() // 32))
    assert (sizes % 4 == 0).all() and (sizes >= 8 + 3 * 32).all()
    for start1 in (int(idx[1, 0]) + 1, 8 + 3 * 32 - 4):   # 1 word off; chunk 0 below header + three rows
        bad = bytearray(data)
        bad[384 + 16: 384 + 24] = np.uint64(start1).tobytes()
        with pytest.raises(entro.EntroError) as e:
            entro.Blob.from_bytes(bytes(bad))
        assert e.value.code == entro.E_FORMAT


def test_device_bytes_layout():
    w = workloads.small_tensor("t4", 64, 256, seed=2)
    blob = entro.Blob.encode(w, bits=8, chunk_symbols=2048)
    info = blob.info()
    nb = blob.device_bytes()
    assert nb % 256 == 0
    assert nb >= info["payload_bytes"] + info["index_bytes"] + 4096 * 4
