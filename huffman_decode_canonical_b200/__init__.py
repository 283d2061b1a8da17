"""Python binding of libentro (argument marshalling only).

Every step of the path -- quantization and Huffman coding on the host, decoding,
dequantization and the fused GEMV on the GPU -- runs inside ``libentro.so``;
this module turns numpy / torch objects into pointers and sizes for the C ABI
declared in ``include/entro.h`` and turns return codes into exceptions.
PyTorch is used for device memory and streams only.  There is no fallback:
importing this package fails when the shared library is missing, and device
calls need a CUDA GPU.

The method is EntroLLM ("EntroLLM: Entropy Encoded Weight Compression for
Efficient Large Language Model Inference on Edge Devices", arXiv
2505.02380v4): mixed tensor-level quantization, Huffman coding of the codes and
parallel decoding of chunks; with the lane-interleaved, decode-on-demand
storage of "LazyWeights: Decode-on-Demand Edge LLMs" (arXiv 2611.17108v1).
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libentro.so")

OK = 0
E_INVAL, E_LIMIT, E_FORMAT, E_CORRUPT, E_OVERRUN, E_NOMEM, E_CUDA, E_TIMEOUT = -1, -2, -3, -4, -5, -6, -7, -8
QUANT_AUTO, QUANT_UNSIGNED, QUANT_ASYM = 0, 1, 2
SCHEME_UNSIGNED, SCHEME_ASYM = 0, 1
FORMAT_SINGLE, FORMAT_LANES, FORMAT_ROWS, FORMAT_ROWS_CO = 1, 2, 3, 4
GROUP_GEMV, GROUP_BF16 = 1, 2


class EntroError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        detail = f" [{_lib.entro_last_cuda_error().decode()}]" if code == E_CUDA else ""
        super().__init__(f"{what}: {_strerror(code)} ({code}){detail}")


class _Opts(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("quant_mode", ctypes.c_int32), ("max_len", ctypes.c_int32),
                ("format", ctypes.c_int32), ("chunk_symbols", ctypes.c_int64), ("threads", ctypes.c_int32),
                ("lanes", ctypes.c_int32)]


class _Info(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("scheme", ctypes.c_int32), ("max_len", ctypes.c_int32),
                ("format", ctypes.c_int32), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("n", ctypes.c_int64), ("chunk_symbols", ctypes.c_int64), ("n_chunks", ctypes.c_int64),
                ("scale", ctypes.c_float), ("zero", ctypes.c_int32), ("payload_bytes", ctypes.c_uint64),
                ("index_bytes", ctypes.c_uint64), ("blob_bytes", ctypes.c_uint64), ("coded_bits", ctypes.c_uint64),
                ("max_chunk_words", ctypes.c_uint32), ("lanes", ctypes.c_uint32),
                ("lengths", ctypes.c_uint8 * 256)]


EXPORTS = ["entro_encode", "entro_blob_from_bytes", "entro_blob_bytes", "entro_blob_info", "entro_blob_free",
           "entro_device_bytes", "entro_upload", "entro_tensor_free", "entro_decode_codes",
           "entro_decode_dequant_bf16", "entro_decode_gemv", "entro_group_table_bytes", "entro_group_prepare",
           "entro_group_launch", "entro_group_free", "entro_strerror", "entro_version", "entro_last_cuda_error",
           "entro_decode_gemv_group_static", "entro_set_overlap", "entro_test_stall_tables"]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python huffman_decode_canonical_b200/build.py` "
                          "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
    PP = ctypes.POINTER(ctypes.c_void_p)
    sig = {
        "entro_encode": ([P, I64, I64, ctypes.POINTER(_Opts), PP], I32),
        "entro_blob_from_bytes": ([P, U64, PP], I32),
        "entro_blob_bytes": ([P, PP, ctypes.POINTER(U64)], I32),
        "entro_blob_info": ([P, ctypes.POINTER(_Info)], I32),
        "entro_blob_free": ([P], None),
        "entro_device_bytes": ([P, ctypes.POINTER(U64)], I32),
        "entro_upload": ([P, P, U64, P, PP], I32),
        "entro_tensor_free": ([P], None),
        "entro_decode_codes": ([P, P, P, P], I32),
        "entro_decode_dequant_bf16": ([P, P, P, P], I32),
        "entro_decode_gemv": ([P, P, I32, P, P, P], I32),
        "entro_group_table_bytes": ([I32], U64),
        "entro_group_prepare": ([P, I32, I32, P, P, P, I32, P, U64, P, PP], I32),
        "entro_group_launch": ([P, P, P], I32),
        "entro_group_free": ([P], None),
        "entro_strerror": ([I32], ctypes.c_char_p),
        "entro_version": ([], I32),
        "entro_last_cuda_error": ([], ctypes.c_char_p),
        "entro_decode_gemv_group_static": ([P, P, P, I32, I32, P, P], I32),
        "entro_set_overlap": ([I32], I32),
        "entro_test_stall_tables": ([ctypes.c_uint32], ctypes.c_uint32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def _strerror(code: int) -> str:
    return _lib.entro_strerror(code).decode()


def _check(code: int, what: str):
    if code != OK:
        raise EntroError(code, what)


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dptr(t: Optional[torch.Tensor]) -> Optional[ctypes.c_void_p]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


# ------------------------------------------------------------------ host side

class Blob:
    """One encoded tensor held on the host (library-owned serialized bytes)."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle

    @classmethod
    def encode(cls, w, bits: int = 8, quant_mode: int = QUANT_AUTO, max_len: int = 0,
               fmt: int = FORMAT_LANES, chunk_symbols: int = 0, threads: int = 0, lanes: int = 0) -> "Blob":
        if isinstance(w, torch.Tensor):
            w = w.detach().to("cpu", torch.float32).numpy()
        w = np.ascontiguousarray(w, dtype=np.float32)
        if w.ndim != 2:
            raise ValueError("w must be 2-D [rows, cols]")
        opts = _Opts(bits, quant_mode, max_len, fmt, chunk_symbols, threads, lanes)
        h = ctypes.c_void_p()
        _check(_lib.entro_encode(w.ctypes.data_as(ctypes.c_void_p) if w.size else None, w.shape[0], w.shape[1],
                                 ctypes.byref(opts), ctypes.byref(h)), "entro_encode")
        return cls(h)

    @classmethod
    def from_bytes(cls, data: bytes) -> "Blob":
        buf = np.frombuffer(data, np.uint8)
        h = ctypes.c_void_p()
        _check(_lib.entro_blob_from_bytes(buf.ctypes.data_as(ctypes.c_void_p), buf.size, ctypes.byref(h)),
               "entro_blob_from_bytes")
        return cls(h)

    def to_bytes(self) -> bytes:
        p = ctypes.c_void_p()
        n = ctypes.c_uint64()
        _check(_lib.entro_blob_bytes(self._h, ctypes.byref(p), ctypes.byref(n)), "entro_blob_bytes")
        return ctypes.string_at(p, n.value)

    def info(self) -> dict:
        i = _Info()
        _check(_lib.entro_blob_info(self._h, ctypes.byref(i)), "entro_blob_info")
        d = {f: getattr(i, f) for f, _ in _Info._fields_ if f != "lengths"}
        d["lengths"] = np.frombuffer(bytes(i.lengths), np.uint8).copy()
        return d

    def device_bytes(self) -> int:
        n = ctypes.c_uint64()
        _check(_lib.entro_device_bytes(self._h, ctypes.byref(n)), "entro_device_bytes")
        return n.value

    def close(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.entro_blob_free(self._h)
            self._h = None

    def __del__(self):
        self.close()


def encode(w, **kw) -> Blob:
    return Blob.encode(w, **kw)


# ------------------------------------------------------------------ device side

class DeviceTensor:
    """A blob's decode image in device memory (a torch uint8 buffer) + its handle."""

    def __init__(self, blob: Blob, device: Optional[torch.device] = None,
                 stream: Optional[torch.cuda.Stream] = None):
        device = torch.device(device if device is not None else "cuda")
        if device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
        info = blob.info()
        self.rows, self.cols, self.n = info["rows"], info["cols"], info["n"]
        self.bits, self.format = info["bits"], info["format"]
        self.chunk_symbols, self.n_chunks = info["chunk_symbols"], info["n_chunks"]
        self.payload_bytes, self.index_bytes = info["payload_bytes"], info["index_bytes"]
        self.info = info
        nbytes = blob.device_bytes()
        with torch.cuda.device(device):
            self.mem = torch.empty(nbytes, dtype=torch.uint8, device=device)
            h = ctypes.c_void_p()
            _check(_lib.entro_upload(blob._h, _dptr(self.mem), nbytes, _stream_ptr(stream), ctypes.byref(h)),
                   "entro_upload")
        self._h = h
        self.device = device

    # output buffers ---------------------------------------------------
    def codes_nbytes(self) -> int:
        return self.n if self.bits == 8 else (self.n + 1) // 2

    def empty_codes(self) -> torch.Tensor:
        return torch.empty(max(self.codes_nbytes(), 1), dtype=torch.uint8, device=self.device)

    def empty_bf16(self) -> torch.Tensor:
        return torch.empty((self.rows, self.cols), dtype=torch.bfloat16, device=self.device)

    # calls ------------------------------------------------------------
    def decode_codes(self, out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        out = self.empty_codes() if out is None else out
        _check(_lib.entro_decode_codes(self._h, _dptr(out), _dptr(status), _stream_ptr(stream)),
               "entro_decode_codes")
        return out

    def decode_dequant_bf16(self, out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                            stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        out = self.empty_bf16() if out is None else out
        _check(_lib.entro_decode_dequant_bf16(self._h, _dptr(out), _dptr(status), _stream_ptr(stream)),
               "entro_decode_dequant_bf16")
        return out

    def decode_gemv(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        if x.dim() == 1:
            x = x.unsqueeze(0)
        batch = x.shape[0]
        if x.dtype != torch.bfloat16 or not x.is_contiguous() or x.shape[1] != self.cols:
            raise ValueError("x must be a contiguous bf16 [batch, cols] tensor")
        y = torch.empty((batch, self.rows), dtype=torch.float32, device=self.device) if y is None else y
        _check(_lib.entro_decode_gemv(self._h, _dptr(x), batch, _dptr(y), _dptr(status), _stream_ptr(stream)),
               "entro_decode_gemv")
        return y

    def close(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.entro_tensor_free(self._h)
            self._h = None

    def __del__(self):
        self.close()


def upload(blob: Blob, device=None, stream=None) -> DeviceTensor:
    return DeviceTensor(blob, device, stream)


class Group:
    """One launch over many tensors (fused GEMV of a decode step, or whole-model bf16 decode)."""

    def __init__(self, tensors: Sequence[DeviceTensor], kind: int, xs: Optional[Sequence[torch.Tensor]] = None,
                 ys: Optional[Sequence[torch.Tensor]] = None, outs: Optional[Sequence[torch.Tensor]] = None,
                 batch: int = 1, stream: Optional[torch.cuda.Stream] = None):
        count = len(tensors)
        self.tensors = list(tensors)
        self.xs, self.ys, self.outs = xs, ys, outs       # keep the buffers alive
        dev = tensors[0].device
        nbytes = int(_lib.entro_group_table_bytes(count))
        self.table = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        arr = ctypes.c_void_p * count
        th = arr(*[t._h for t in tensors])
        xp = arr(*[x.data_ptr() for x in xs]) if xs is not None else None
        yp = arr(*[y.data_ptr() for y in ys]) if ys is not None else None
        op = arr(*[o.data_ptr() for o in outs]) if outs is not None else None
        h = ctypes.c_void_p()
        _check(_lib.entro_group_prepare(th, count, kind, xp, yp, op, batch, _dptr(self.table), nbytes,
                                        _stream_ptr(stream), ctypes.byref(h)), "entro_group_prepare")
        self._h = h

    def launch(self, status: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
        _check(_lib.entro_group_launch(self._h, _dptr(status), _stream_ptr(stream)), "entro_group_launch")

    def close(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.entro_group_free(self._h)
            self._h = None

    def __del__(self):
        self.close()


STATIC_GROUP_MAX = 512


def decode_gemv_group_static(tensors: Sequence[DeviceTensor], xs: Sequence[torch.Tensor],
                             ys: Sequence[torch.Tensor], batch: int = 1, status: Optional[torch.Tensor] = None,
                             stream: Optional[torch.cuda.Stream] = None) -> None:
    """Grouped fused GEMV whose work table lives inside the library (no device allocation)."""
    count = len(tensors)
    if count < 1 or len(xs) != count or len(ys) != count:
        raise ValueError("need one x and one y per tensor")
    for t, x, y in zip(tensors, xs, ys):
        if (x.dtype != torch.bfloat16 or not x.is_contiguous() or x.dim() != 2 or x.shape != (batch, t.cols)
                or x.device != t.device):
            raise ValueError("each x must be a contiguous bf16 [batch, cols] tensor on the tensors' device")
        if (y.dtype != torch.float32 or not y.is_contiguous() or y.dim() != 2 or y.shape != (batch, t.rows)
                or y.device != t.device):
            raise ValueError("each y must be a contiguous fp32 [batch, rows] tensor on the tensors' device")
    arr = ctypes.c_void_p * count
    _check(_lib.entro_decode_gemv_group_static(arr(*[t._h for t in tensors]), arr(*[x.data_ptr() for x in xs]),
                                               arr(*[y.data_ptr() for y in ys]), count, batch, _dptr(status),
                                               _stream_ptr(stream)), "entro_decode_gemv_group_static")


def test_stall_tables(extra_bytes: int) -> int:
    """Test hook for the bounded waits: later launches wait for `extra_bytes` of table copy that
    never arrive, so each gives up after about a second with E_TIMEOUT in the status word.
    0 turns it off.  Returns the previous value."""
    return int(_lib.entro_test_stall_tables(int(extra_bytes)))


def version() -> int:
    return int(_lib.entro_version())


def set_overlap(enable: bool) -> bool:
    """Launch overlap (programmatic dependent launch) for every later decode call in this
    process: a decode may start while the kernel before it on the stream finishes, reading
    only the tensor's device image until that kernel has completed.  Enable only if no
    kernel launched right before a decode call writes that tensor's device image.
    Returns the previous setting."""
    return bool(_lib.entro_set_overlap(1 if enable else 0))


__all__ = ["Blob", "DeviceTensor", "Group", "EntroError", "encode", "upload", "lib", "version", "set_overlap", "EXPORTS",
           "decode_gemv_group_static", "STATIC_GROUP_MAX",
           "test_stall_tables", "QUANT_AUTO", "QUANT_UNSIGNED", "QUANT_ASYM", "FORMAT_SINGLE", "FORMAT_LANES", "FORMAT_ROWS_CO",
           "FORMAT_ROWS", "GROUP_GEMV",
           "GROUP_BF16", "SCHEME_UNSIGNED", "SCHEME_ASYM"]
