"""CPU oracle of the exponent-split KV codec -- TEST INFRASTRUCTURE ONLY.

A plain, slow, single-threaded C implementation (oracle.c) of what the codec
computes, after "SplitZip: Ultra-Fast Lossless KV Compression for Disaggregated
LLM Serving" (project page, Abstract and FAQ), in this library's stream format
v1.  Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA library.

The wrappers below only marshal numpy buffers into the C calls.
"""
import ctypes

import numpy as np

from . import build as _build

BF16 = 0
E5M2 = 1

OK, ERR_ARG, ERR_DTYPE, ERR_SMALL, ERR_CORRUPT = 0, 1, 2, 3, 4
FLAG_RAW_BLOCKS = 1  # header byte 39, bit 0: blocks that would expand are stored raw

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u64p = ctypes.POINTER(ctypes.c_uint64)


def _u8(a: np.ndarray):
    return a.ctypes.data_as(_u8p)


def _raw(x) -> np.ndarray:
    """Flat little-endian byte view of a numpy array (or bytes)."""
    if isinstance(x, (bytes, bytearray)):
        a = np.frombuffer(x, dtype=np.uint8)
    else:
        a = np.asarray(x)
    return np.ascontiguousarray(a).reshape(-1).view(np.uint8)


def elem_size(dtype: int) -> int:
    return 2 if dtype == BF16 else 1


class Oracle:
    """ctypes view of one build of oracle.c (the default build, or a test's variant)."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        L.orc_compressed_size.argtypes = [ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64]
        L.orc_compressed_size.restype = ctypes.c_uint64
        L.orc_histogram.argtypes = [ctypes.c_int, _u8p, ctypes.c_uint64, _u64p]
        L.orc_histogram.restype = ctypes.c_int
        L.orc_codebook.argtypes = [ctypes.c_int, _u64p, _u8p]
        L.orc_codebook.restype = ctypes.c_int
        L.orc_encode.argtypes = [ctypes.c_int, _u8p, ctypes.c_uint64, _u8p, ctypes.c_uint64]
        L.orc_encode.restype = ctypes.c_int64
        L.orc_encode_codebook.argtypes = [ctypes.c_int, _u8p, ctypes.c_uint64, _u8p, _u8p, ctypes.c_uint64]
        L.orc_encode_codebook.restype = ctypes.c_int64
        L.orc_encode_ex.argtypes = [ctypes.c_int, _u8p, ctypes.c_uint64, _u8p, ctypes.c_uint,
                                    _u8p, ctypes.c_uint64]
        L.orc_encode_ex.restype = ctypes.c_int64
        L.orc_decode.argtypes = [_u8p, ctypes.c_uint64, _u8p, ctypes.c_uint64]
        L.orc_decode.restype = ctypes.c_int
        self.lib = L
        self.path = path

    def compressed_size(self, dtype: int, n: int, E: int) -> int:
        return int(self.lib.orc_compressed_size(dtype, n, E))

    def histogram(self, dtype: int, x) -> np.ndarray:
        raw = _raw(x)
        n = raw.size // elem_size(dtype)
        h = np.zeros(256, dtype=np.uint64)
        rc = self.lib.orc_histogram(dtype, _u8(raw), n, h.ctypes.data_as(_u64p))
        if rc:
            raise ValueError("orc_histogram failed: %d" % rc)
        return h

    def codebook(self, dtype: int, hist) -> np.ndarray:
        h = np.ascontiguousarray(np.asarray(hist, dtype=np.uint64))
        if h.size < 256:
            h = np.concatenate([h, np.zeros(256 - h.size, dtype=np.uint64)])
        cb = np.zeros(15, dtype=np.uint8)
        rc = self.lib.orc_codebook(dtype, h.ctypes.data_as(_u64p), _u8(cb))
        if rc:
            raise ValueError("orc_codebook failed: %d" % rc)
        return cb

    def encode_ex_status(self, dtype: int, x, cb=None, raw_blocks=False, cap=None):
        """Encode with the tensor's own codebook (cb None) or a given one, with or
        without raw blocks; return (bytes written or -error, stream as uint8)."""
        raw = _raw(x)
        n = raw.size // elem_size(dtype)
        cbp = None
        if cb is not None:
            cbv = np.ascontiguousarray(np.asarray(cb, dtype=np.uint8).reshape(-1))
            if cbv.size != 15:
                raise ValueError("a codebook has 15 entries")
            cbp = _u8(cbv)
        if cap is None:
            cap = self.compressed_size(dtype, n, n)
        # poisoned, so that a stream byte the encoder forgets to write shows up
        out = np.full(max(cap, 1), 0xA5, dtype=np.uint8)
        flags = FLAG_RAW_BLOCKS if raw_blocks else 0
        r = int(self.lib.orc_encode_ex(dtype, _u8(raw), n, cbp, flags, _u8(out), cap))
        return r, (out[:r].copy() if r >= 0 else out[:0])

    def encode_ex(self, dtype: int, x, cb=None, raw_blocks=False) -> np.ndarray:
        r, out = self.encode_ex_status(dtype, x, cb, raw_blocks)
        if r < 0:
            raise ValueError("orc_encode_ex failed: %d" % -r)
        return out

    def encode_status(self, dtype: int, x, cap=None, raw_blocks=False):
        """Encode; return (bytes written or -error, stream as uint8)."""
        if raw_blocks:
            return self.encode_ex_status(dtype, x, None, True, cap)
        raw = _raw(x)
        n = raw.size // elem_size(dtype)
        if cap is None:
            cap = self.compressed_size(dtype, n, n)
        out = np.full(max(cap, 1), 0xA5, dtype=np.uint8)
        r = int(self.lib.orc_encode(dtype, _u8(raw), n, _u8(out), cap))
        return r, (out[:r].copy() if r >= 0 else out[:0])

    def encode(self, dtype: int, x, raw_blocks=False) -> np.ndarray:
        """Encode raw elements (numpy array or bytes); return the stream as uint8."""
        r, out = self.encode_status(dtype, x, raw_blocks=raw_blocks)
        if r < 0:
            raise ValueError("orc_encode failed: %d" % -r)
        return out

    def encode_codebook_status(self, dtype: int, x, cb, cap=None, raw_blocks=False):
        """Encode with the given 15-entry codebook; return (bytes written or -error, stream)."""
        if raw_blocks:
            return self.encode_ex_status(dtype, x, cb, True, cap)
        raw = _raw(x)
        n = raw.size // elem_size(dtype)
        cbv = np.ascontiguousarray(np.asarray(cb, dtype=np.uint8).reshape(-1))
        if cbv.size != 15:
            raise ValueError("a codebook has 15 entries")
        if cap is None:
            cap = self.compressed_size(dtype, n, n)
        out = np.full(max(cap, 1), 0xA5, dtype=np.uint8)
        r = int(self.lib.orc_encode_codebook(dtype, _u8(raw), n, _u8(cbv), _u8(out), cap))
        return r, (out[:r].copy() if r >= 0 else out[:0])

    def encode_codebook(self, dtype: int, x, cb, raw_blocks=False) -> np.ndarray:
        """Encode raw elements with a given codebook (codebook reuse); return the stream."""
        r, out = self.encode_codebook_status(dtype, x, cb, raw_blocks=raw_blocks)
        if r < 0:
            raise ValueError("orc_encode_codebook failed: %d" % -r)
        return out

    def decode_status(self, stream, n: int, dtype: int):
        """Decode; return (status, raw uint8 array)."""
        s = _raw(stream)
        out = np.zeros(max(n, 1) * elem_size(dtype), dtype=np.uint8)
        rc = self.lib.orc_decode(_u8(s), s.size, _u8(out), n)
        return int(rc), out[: n * elem_size(dtype)]

    def decode(self, stream, n: int, dtype: int) -> np.ndarray:
        rc, out = self.decode_status(stream, n, dtype)
        if rc:
            raise ValueError("orc_decode failed: %d" % rc)
        return out


_default = None


def default() -> Oracle:
    """The oracle built from oracle.c as committed (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def compressed_size(dtype, n, E):
    return default().compressed_size(dtype, n, E)


def histogram(dtype, x):
    return default().histogram(dtype, x)


def codebook(dtype, hist):
    return default().codebook(dtype, hist)


def encode(dtype, x, raw_blocks=False):
    return default().encode(dtype, x, raw_blocks)


def encode_status(dtype, x, cap=None, raw_blocks=False):
    return default().encode_status(dtype, x, cap, raw_blocks)


def encode_codebook(dtype, x, cb, raw_blocks=False):
    return default().encode_codebook(dtype, x, cb, raw_blocks)


def encode_codebook_status(dtype, x, cb, cap=None, raw_blocks=False):
    return default().encode_codebook_status(dtype, x, cb, cap, raw_blocks)


def decode(stream, n, dtype):
    return default().decode(stream, n, dtype)


def decode_status(stream, n, dtype):
    return default().decode_status(stream, n, dtype)
