"""CPU oracle for the Huffman weight-decoding path -- TEST INFRASTRUCTURE ONLY.

Thin ctypes wrapper over ``entro_oracle.c`` (plain C, bit-by-bit, no lookup
tables).  Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this package; the product library never does, and
this package never imports the product.

Which passage each function follows is stated in ``entro_oracle.c``.  Every
function is pinned by tests against facts that do not come from this code
(Kraft equality, entropy bounds, brute-force optimal codes on tiny alphabets,
hand-worked fixtures under ``tests/golden/``, library routines for the bf16
rounding and the fp64 matrix product).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "entro_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

OK, EINVAL, ELIMIT, EFORMAT, ECORRUPT, ENOMEM = 0, -1, -2, -3, -4, -5
MODE_AUTO, MODE_UNSIGNED, MODE_ASYM = 0, 1, 2
SCHEME_UNSIGNED, SCHEME_ASYM = 0, 1
FMT_SINGLE, FMT_LANES, FMT_ROWS, FMT_ROWS_CO = 1, 2, 3, 4


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} failed with status {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (plain -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i64, u64, i32 = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int
            lib.or_quantize.argtypes = [P, i64, i32, i32, P, P, P, P]
            lib.or_histogram.argtypes = [P, i64, i32, P]
            lib.or_histogram.restype = None
            lib.or_entropy.argtypes = [P, i32]
            lib.or_entropy.restype = ctypes.c_double
            lib.or_code_lengths.argtypes = [P, i32, i32, P]
            lib.or_canonical_codes.argtypes = [P, i32, P]
            lib.or_encode.argtypes = [P, i64, i64, i32, i32, i32, i32, i64, i32, P, u64, P]
            lib.or_decode.argtypes = [P, u64, P]
            lib.or_decode_chunks.argtypes = [P, u64, u64, u64, P]
            lib.or_blob_params.argtypes = [P, u64, P]
            lib.or_dequant_bf16.argtypes = [P, i64, ctypes.c_float, ctypes.c_int32, P]
            lib.or_dequant_bf16.restype = None
            lib.or_gemv.argtypes = [P, i64, i64, P, i32, i64, i64, P, P]
            lib.or_gemv.restype = None
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(code: int, what: str):
    if code != OK:
        raise OracleError(code, what)


def quantize(w: np.ndarray, bits: int, mode: int) -> Tuple[np.ndarray, float, int, int]:
    """Tensor-level quantization -> (codes uint8, scale fp32, zero int, scheme)."""
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(-1)
    q = np.zeros(max(1, w.size), dtype=np.uint8)
    s = np.zeros(1, np.float32)
    z = np.zeros(1, np.int32)
    sch = np.zeros(1, np.int32)
    _check(_load().or_quantize(_ptr(w), w.size, bits, mode, _ptr(q), _ptr(s), _ptr(z), _ptr(sch)),
           "quantize")
    return q[: w.size], float(s[0]), int(z[0]), int(sch[0])


def histogram(q: np.ndarray, nsym: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8).reshape(-1)
    h = np.zeros(nsym, np.int64)
    _load().or_histogram(_ptr(q), q.size, nsym, _ptr(h))
    return h


def entropy(hist: np.ndarray) -> float:
    h = np.ascontiguousarray(hist, dtype=np.int64)
    return float(_load().or_entropy(_ptr(h), h.size))


def code_lengths(hist: np.ndarray, max_len: int) -> np.ndarray:
    """Optimal code lengths under the limit max_len (package-merge)."""
    h = np.ascontiguousarray(hist, dtype=np.int64)
    out = np.zeros(h.size, np.uint8)
    _check(_load().or_code_lengths(_ptr(h), h.size, max_len, _ptr(out)), "code_lengths")
    return out


def canonical_codes(lengths: np.ndarray) -> np.ndarray:
    ln = np.ascontiguousarray(lengths, dtype=np.uint8)
    out = np.zeros(ln.size, np.uint32)
    _check(_load().or_canonical_codes(_ptr(ln), ln.size, _ptr(out)), "canonical_codes")
    return out


def encode(w: np.ndarray, bits: int, mode: int, max_len: int, fmt: int, chunk_symbols: int,
           lanes: int = 32) -> bytes:
    """Whole encoder: fp32 [rows, cols] -> serialized blob bytes (lanes: 32 or 64 for the lanes format)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    if w.ndim != 2:
        raise ValueError("w must be 2-D")
    rows, cols = w.shape
    size = np.zeros(1, np.uint64)
    lib = _load()
    _check(lib.or_encode(_ptr(w), rows, cols, bits, mode, max_len, fmt, chunk_symbols, lanes,
                         None, 0, _ptr(size)), "encode(size)")
    out = np.zeros(int(size[0]), np.uint8)
    _check(lib.or_encode(_ptr(w), rows, cols, bits, mode, max_len, fmt, chunk_symbols, lanes,
                         _ptr(out), out.size, _ptr(size)), "encode")
    return out.tobytes()


def params(blob: bytes) -> Dict[str, float]:
    b = np.frombuffer(blob, np.uint8)
    out = np.zeros(14, np.int64)
    _check(_load().or_blob_params(_ptr(b), b.size, _ptr(out)), "params")
    keys = ["bits", "scheme", "max_len", "format", "rows", "cols", "n", "chunk_symbols",
            "n_chunks", "scale_bits", "zero", "payload_words", "lanes", "run"]
    d = {k: int(v) for k, v in zip(keys, out)}
    d["scale"] = float(np.array([d["scale_bits"]], np.uint32).view(np.float32)[0])
    d["lengths"] = np.frombuffer(blob, np.uint8, 256, 128).copy()
    return d


def decode(blob: bytes) -> np.ndarray:
    """Bit-by-bit canonical decode of a whole blob -> codes uint8[n]."""
    p = params(blob)
    b = np.frombuffer(blob, np.uint8)
    out = np.zeros(max(1, p["n"]), np.uint8)
    _check(_load().or_decode(_ptr(b), b.size, _ptr(out)), "decode")
    return out[: p["n"]]


def decode_chunks(blob: bytes, c0: int, c1: int) -> np.ndarray:
    """Decode chunks [c0, c1) -> their codes (concatenated, each chunk in its own order:
    row-major for the single-stream and lanes layouts, the tile's rows one after the other
    for the row-tile layout)."""
    p = params(blob)
    b = np.frombuffer(blob, np.uint8)
    first, last = _chunk_first(p, c0), _chunk_first(p, c1)
    out = np.zeros(max(1, p["n"] - first), np.uint8)        # room for anything a chunk may claim
    _check(_load().or_decode_chunks(_ptr(b), b.size, c0, c1, _ptr(out)), "decode_chunks")
    return out[: max(0, last - first)]


def _chunk_first(p: Dict, c: int) -> int:
    """Symbols in the chunks before chunk c, from the blob's geometry (chunk order)."""
    if c >= p["n_chunks"]:
        return p["n"]
    if p["format"] not in (FMT_ROWS, FMT_ROWS_CO):
        return min(p["n"], c * p["chunk_symbols"])
    rows, cols, lanes = p["rows"], p["cols"], p["lanes"]
    kc = p["chunk_symbols"] // lanes
    tiles = -(-cols // kc)
    g, j = divmod(c, tiles)
    nrows = min(lanes, rows - g * lanes)
    return g * lanes * cols + nrows * j * kc


def tile(p: Dict, c: int) -> Tuple[int, int, int, int]:
    """Row-tile layout: (first row, first column, rows, columns) of chunk c."""
    lanes, kc = p["lanes"], p["chunk_symbols"] // p["lanes"]
    tiles = -(-p["cols"] // kc)
    g, j = divmod(c, tiles)
    return g * lanes, j * kc, min(lanes, p["rows"] - g * lanes), min(kc, p["cols"] - j * kc)


def dequant_bf16(q: np.ndarray, scale: float, zero: int) -> np.ndarray:
    """w = bf16_rne(float(q - zero) * scale) -> uint16 bit patterns."""
    q = np.ascontiguousarray(q, dtype=np.uint8).reshape(-1)
    out = np.zeros(max(1, q.size), np.uint16)
    _load().or_dequant_bf16(_ptr(q), q.size, ctypes.c_float(scale), zero, _ptr(out))
    return out[: q.size]


def gemv(w_bf16: np.ndarray, x_bf16: np.ndarray, r0: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 y[b, r] = sum_k w[r, k] * x[b, k] for the rows held in ``w_bf16`` (uint16 bits).

    Returns (y, mag) where mag[b, r] = sum_k |w[r, k] * x[b, k]|.
    """
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = w.shape
    batch = x.shape[0]
    assert x.shape[1] == cols
    y = np.zeros((batch, rows), np.float64)
    mag = np.zeros((batch, rows), np.float64)
    _load().or_gemv(_ptr(w), rows, cols, _ptr(x), batch, r0, r0 + rows, _ptr(y), _ptr(mag))
    return y, mag
