"""fp64 CPU oracle for paged KV-cache decode -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check and the CPU-baseline / reference leg of
the benchmark may import this package.  The product library never does, and
the oracle never imports the product: the two share only the seeded input
generators (which hold none of the method's arithmetic).

The arithmetic lives in ``pkv_oracle.c`` (plain C, double precision, loops in
the order the pages define them); this module only compiles it with gcc and
marshals numpy arrays through ctypes.  See the C file's header for the source
passages and the readings taken where the pages are silent.

Functions take and return numpy arrays.  16-bit element arrays are passed as
their raw ``uint16`` storage codes together with ``dtype`` ("f16" or "bf16").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()

OK, ERR_ARG, ERR_RANGE = 0, 1, 3
_DTYPE_CODE = {"f16": 0, "bf16": 1}


def compile_source(src: str, out_path: str) -> str:
    """Compile an oracle C source file into a shared library (gcc, OpenMP)."""
    os.makedirs(os.path.dirname(out_path), exist_ok=True)
    tmp = out_path + f".{os.getpid()}.tmp"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out_path)
    return out_path


def build(force: bool = False) -> str:
    """Compile pkv_oracle.c into oracle/_build/liboracle.so."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    return compile_source(_SRC, _LIB_PATH)


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what}: status {code}")
        self.code = code


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected uint16 storage codes, got {a.dtype}")
    return a


def _c(a, dt) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dt)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.pkvo_decode_f16.restype = dbl
        lib.pkvo_decode_f16.argtypes = [ctypes.c_uint16]
        lib.pkvo_decode_bf16.restype = dbl
        lib.pkvo_decode_bf16.argtypes = [ctypes.c_uint16]
        lib.pkvo_decode_array.restype = None
        lib.pkvo_decode_array.argtypes = [P, i64, i32, P]
        lib.pkvo_kv_cache_write.restype = i32
        lib.pkvo_kv_cache_write.argtypes = [P, P, P, i64, i32, i32, P, P, i64, i32]
        lib.pkvo_paged_attention_decode.restype = i32
        lib.pkvo_paged_attention_decode.argtypes = [
            P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64, dbl, i32, P, P, i32]
        lib.pkvo_paged_attention_partitions.restype = i32
        lib.pkvo_paged_attention_partitions.argtypes = [
            P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64, dbl, i32, i32, i32,
            P, P, P, P]
        lib.pkvo_paged_attention_prefill.restype = i32
        lib.pkvo_paged_attention_prefill.argtypes = [
            P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64, dbl, i32, P, P, i32]
        lib.pkvo_copy_blocks.restype = i32
        lib.pkvo_copy_blocks.argtypes = [P, P, P, i32, i64, i64, i64]
        lib.pkvo_lse_merge.restype = None
        lib.pkvo_lse_merge.argtypes = [P, P, P, i64, i32, i32, P]
        self.lib = lib
        self.path = lib_path

    def decode_f16(self, code: int) -> float:
        return self.lib.pkvo_decode_f16(code)

    def decode_bf16(self, code: int) -> float:
        return self.lib.pkvo_decode_bf16(code)

    def decode_array(self, codes, dtype: str) -> np.ndarray:
        codes = _u16(codes)
        out = np.empty(codes.shape, dtype=np.float64)
        self.lib.pkvo_decode_array(_ptr(codes), codes.size, _DTYPE_CODE[dtype], _ptr(out))
        return out

    def kv_cache_write(self, key, value, slot_mapping, key_cache, value_cache,
                       block_size: int) -> None:
        """In-place bit copy of key/value [T, Hkv, D] into the caches
        [num_blocks, block_size, Hkv, D] at slot_mapping[t] (int64)."""
        key, value = _u16(key), _u16(value)
        slots = _c(slot_mapping, np.int64)
        for c in (key_cache, value_cache):
            if c.dtype != np.uint16 or not c.flags["C_CONTIGUOUS"]:
                raise TypeError("caches must be C-contiguous uint16 arrays (written in place)")
        T, Hkv, D = key.shape
        nb = key_cache.shape[0]
        rc = self.lib.pkvo_kv_cache_write(_ptr(key), _ptr(value), _ptr(slots), T, Hkv, D,
                                          _ptr(key_cache), _ptr(value_cache), nb, block_size)
        if rc != OK:
            raise OracleError(rc, "kv_cache_write")

    def paged_attention_prefill(self, query, query_start, key_cache, value_cache, block_tables,
                                context_lens, scale: float, dtype: str,
                                nthreads: int = 1) -> np.ndarray:
        """Causal chunk attention: query [T, Hq, D] (uint16), query_start int32 [B+1]
        -> unrounded fp64 [T, Hq, D]."""
        q, kc, vc = _u16(query), _u16(key_cache), _u16(value_cache)
        qs = _c(query_start, np.int32)
        bt = _c(block_tables, np.int32)
        cl = _c(context_lens, np.int32)
        T, Hq, D = q.shape
        nb, bs, Hkv, _ = kc.shape
        mb = bt.shape[1]
        out = np.zeros((T, Hq, D), dtype=np.float64)
        scratch = np.empty(max(1, mb * bs) * nthreads, dtype=np.float64)
        rc = self.lib.pkvo_paged_attention_prefill(
            _ptr(q), _ptr(qs), _ptr(kc), _ptr(vc), _ptr(bt), mb, _ptr(cl), len(qs) - 1, Hq, Hkv,
            D, bs, nb, float(scale), _DTYPE_CODE[dtype], _ptr(out), _ptr(scratch), nthreads)
        if rc != OK:
            raise OracleError(rc, "paged_attention_prefill")
        return out

    def copy_blocks(self, src_cache, dst_cache, mapping) -> None:
        """In place: dst_cache[mapping[i, 1]] = src_cache[mapping[i, 0]] (bit copy)."""
        src = _u16(src_cache)
        if dst_cache.dtype != np.uint16 or not dst_cache.flags["C_CONTIGUOUS"]:
            raise TypeError("dst_cache must be a C-contiguous uint16 array (written in place)")
        mp = _c(mapping, np.int32).reshape(-1, 2)
        elems = int(np.prod(src.shape[1:]))
        assert int(np.prod(dst_cache.shape[1:])) == elems
        rc = self.lib.pkvo_copy_blocks(_ptr(src), _ptr(dst_cache), _ptr(mp), mp.shape[0],
                                       src.shape[0], dst_cache.shape[0], elems)
        if rc != OK:
            raise OracleError(rc, "copy_blocks")

    def paged_attention_decode(self, query, key_cache, value_cache, block_tables,
                               context_lens, scale: float, dtype: str,
                               nthreads: int = 1) -> np.ndarray:
        """Unrounded fp64 decode output [B, Hq, D]."""
        q, kc, vc = _u16(query), _u16(key_cache), _u16(value_cache)
        bt = _c(block_tables, np.int32)
        cl = _c(context_lens, np.int32)
        B, Hq, D = q.shape
        nb, bs, Hkv, D2 = kc.shape
        assert D2 == D and vc.shape == kc.shape
        mb = bt.shape[1]
        out = np.zeros((B, Hq, D), dtype=np.float64)
        scratch = np.empty(max(1, mb * bs) * nthreads, dtype=np.float64)
        rc = self.lib.pkvo_paged_attention_decode(
            _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), mb, _ptr(cl), B, Hq, Hkv, D, bs, nb,
            float(scale), _DTYPE_CODE[dtype], _ptr(out), _ptr(scratch), nthreads)
        if rc != OK:
            raise OracleError(rc, "paged_attention_decode")
        return out

    def paged_attention_partitions(self, query, key_cache, value_cache, block_tables,
                                   context_lens, scale: float, dtype: str,
                                   partition_tokens: int, num_partitions: int):
        """Per-partition (m, l, o): shapes [B, Hq, P], [B, Hq, P], [B, Hq, P, D]."""
        q, kc, vc = _u16(query), _u16(key_cache), _u16(value_cache)
        bt = _c(block_tables, np.int32)
        cl = _c(context_lens, np.int32)
        B, Hq, D = q.shape
        nb, bs, Hkv, _ = kc.shape
        mb = bt.shape[1]
        P = num_partitions
        m = np.empty((B, Hq, P), dtype=np.float64)
        l = np.empty((B, Hq, P), dtype=np.float64)
        o = np.empty((B, Hq, P, D), dtype=np.float64)
        scratch = np.empty(max(1, partition_tokens), dtype=np.float64)
        rc = self.lib.pkvo_paged_attention_partitions(
            _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), mb, _ptr(cl), B, Hq, Hkv, D, bs, nb,
            float(scale), _DTYPE_CODE[dtype], partition_tokens, P, _ptr(m), _ptr(l),
            _ptr(o), _ptr(scratch))
        if rc != OK:
            raise OracleError(rc, "paged_attention_partitions")
        return m, l, o

    def lse_merge(self, m, l, o) -> np.ndarray:
        """Merge per-partition results: [B, Hq, P] x2 + [B, Hq, P, D] -> [B, Hq, D]."""
        m, l, o = _c(m, np.float64), _c(l, np.float64), _c(o, np.float64)
        B, Hq, P, D = o.shape
        out = np.empty((B, Hq, D), dtype=np.float64)
        self.lib.pkvo_lse_merge(_ptr(m), _ptr(l), _ptr(o), B * Hq, P, D, _ptr(out))
        return out


def default() -> Oracle:
    """The oracle built from this directory's pkv_oracle.c (compiled on demand)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
        return _default


_default = None


def decode_array(codes, dtype):
    return default().decode_array(codes, dtype)


def kv_cache_write(*a, **k):
    return default().kv_cache_write(*a, **k)


def paged_attention_decode(*a, **k):
    return default().paged_attention_decode(*a, **k)


def paged_attention_partitions(*a, **k):
    return default().paged_attention_partitions(*a, **k)


def lse_merge(*a, **k):
    return default().lse_merge(*a, **k)


def copy_blocks(*a, **k):
    return default().copy_blocks(*a, **k)


def paged_attention_prefill(*a, **k):
    return default().paged_attention_prefill(*a, **k)
