"""CPU oracle of the SplitZip BF16 exponent codec -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The CUDA library never uses it and the two share
no code.  The arithmetic lives in ``sz_oracle.c`` (plain, single-threaded C);
this module builds it with gcc and marshals numpy arrays to it.

Method source: "SplitZip: Ultra Fast Lossless KV Compression for Disaggregated
LLM Serving" (gist.science explainer), sections 1-4 and "Les Resultats".
Parity of the byte layout is pinned by the container specification written in
``sz_oracle.h`` (the pages do not fix bytes) and by hand-written golden files.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sz_oracle.c")
_HDR = os.path.join(_HERE, "sz_oracle.h")
_LIB = os.path.join(_HERE, "libszoracle.so")

OK = 0
ERR_NULL = -1
ERR_TOO_LARGE = -2
ERR_CAPACITY = -3
ERR_CORRUPT = -5
HEADER_BYTES = 48


def build(force: bool = False) -> str:
    """Compile sz_oracle.c into libszoracle.so (gcc, -O2, no threads)."""
    stale = (not os.path.exists(_LIB)) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB) for p in (_SRC, _HDR))
    if force or stale:
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-Werror",
                               "-shared", "-fPIC", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64 = ctypes.c_uint64
        p = ctypes.c_void_p
        lib.szo_histogram.argtypes = [p, u64, p]
        lib.szo_histogram.restype = None
        lib.szo_select_top16.argtypes = [p, p]
        lib.szo_select_top16.restype = None
        lib.szo_container_size.argtypes = [u64, u64]
        lib.szo_container_size.restype = u64
        lib.szo_encode.argtypes = [p, u64, p, u64, p, p]
        lib.szo_encode.restype = ctypes.c_int
        lib.szo_encode_with_codebook.argtypes = [p, u64, p, p, u64, p, p]
        lib.szo_encode_with_codebook.restype = ctypes.c_int
        lib.szo_decode.argtypes = [p, u64, p, u64]
        lib.szo_decode.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a.size else ctypes.c_void_p(None)


def _as_u16(x) -> np.ndarray:
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        x = x.view(np.uint16) if x.dtype.itemsize == 2 else x.astype(np.uint16)
    return x.reshape(-1)


def histogram(x) -> np.ndarray:
    x = _as_u16(x)
    h = np.zeros(256, np.uint64)
    _load().szo_histogram(_ptr(x), x.size, _ptr(h))
    return h


def select_top16(hist) -> np.ndarray:
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    assert h.shape == (256,)
    cb = np.zeros(16, np.uint8)
    _load().szo_select_top16(_ptr(h), _ptr(cb))
    return cb


def container_size(n: int, e: int) -> int:
    return int(_load().szo_container_size(n, e))


def max_container_size(n: int) -> int:
    """Worst case: the top 16 of 256 bins hold at least ceil(n/16) elements."""
    return container_size(n, n - (n + 15) // 16)


def encode(x, codebook=None) -> bytes:
    """Encode a BF16 array (uint16 bit patterns) into a container."""
    x = _as_u16(x)
    cap = max_container_size(x.size) if codebook is None else container_size(x.size, x.size)
    out = np.zeros(cap, np.uint8)
    size = ctypes.c_uint64(0)
    esc = ctypes.c_uint64(0)
    if codebook is None:
        st = _load().szo_encode(_ptr(x), x.size, _ptr(out), cap, ctypes.byref(size),
                                ctypes.byref(esc))
    else:
        cb = np.ascontiguousarray(codebook, dtype=np.uint8)
        assert cb.shape == (16,)
        st = _load().szo_encode_with_codebook(_ptr(x), x.size, _ptr(cb), _ptr(out), cap,
                                              ctypes.byref(size), ctypes.byref(esc))
    if st != OK:
        raise ValueError("oracle encode failed: status %d" % st)
    return out[: size.value].tobytes()


def decode_status(blob, n: int):
    """Decode; returns (status, uint16 array)."""
    b = np.frombuffer(bytes(blob), np.uint8) if not isinstance(blob, np.ndarray) else blob
    b = np.ascontiguousarray(b, dtype=np.uint8)
    in_bytes = b.size
    if in_bytes == 0:
        b = np.zeros(1, np.uint8)  # a valid address; the length says empty
    out = np.zeros(n, np.uint16)
    st = _load().szo_decode(_ptr(b), in_bytes, _ptr(out), n)
    return st, out


def decode(blob, n: int) -> np.ndarray:
    st, out = decode_status(blob, n)
    if st != OK:
        raise ValueError("oracle decode failed: status %d" % st)
    return out
