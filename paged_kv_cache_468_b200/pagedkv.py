"""ctypes binding of libpagedkv.so -- argument marshalling only.

Every step of the hot path runs in the library's CUDA kernels; this module
turns torch tensors into pointers, sizes and a stream handle, calls the C ABI
declared in include/pagedkv.h, and raises on a non-OK status.  There is no
fallback: if the library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# PKV_LIBRARY selects another build of the library (e.g. a tuning variant).
LIB_PATH = os.environ.get("PKV_LIBRARY") or os.path.join(_HERE, "libpagedkv.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_OUT_OF_RANGE, ERR_OOM, ERR_CUDA, ERR_WORKSPACE, \
    ERR_MISALIGNED = range(8)
DEVFLAG_SLOT_RANGE, DEVFLAG_BLOCK_RANGE, DEVFLAG_CONTEXT_RANGE, DEVFLAG_WAIT_TIMEOUT = 1, 2, 4, 8
F16, BF16 = 0, 1
_DTYPES = {torch.float16: F16, torch.bfloat16: BF16}

_lock = threading.Lock()
_lib = None


class PagedKVError(RuntimeError):
    def __init__(self, status: int, call: str, detail: str):
        super().__init__(f"{call} -> {status_name(status)}: {detail}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded library (raises RuntimeError if it is not built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_468_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
        sz, f32 = ctypes.c_size_t, ctypes.c_float
        pi32 = ctypes.POINTER(ctypes.c_int32)
        pint = ctypes.POINTER(ctypes.c_int)
        L.pkv_status_str.restype = ctypes.c_char_p
        L.pkv_status_str.argtypes = [i32]
        L.pkv_last_error.restype = ctypes.c_char_p
        L.pkv_last_error.argtypes = []
        L.pkv_version.restype = ctypes.c_char_p
        L.pkv_version.argtypes = []
        L.pkv_device_flags.restype = i32
        L.pkv_device_flags.argtypes = [i32, ctypes.POINTER(ctypes.c_uint), i32]
        L.pkv_copy_blocks.restype = i32
        L.pkv_copy_blocks.argtypes = [P, P, P, P, P, i32, i64, i64, i64, P]
        L.pkv_selftest_bounded_wait.restype = i32
        L.pkv_selftest_bounded_wait.argtypes = [i64, P]
        L.pkv_kv_cache_write.restype = i32
        L.pkv_kv_cache_write.argtypes = [P, P, P, i64, i32, i32, P, P, i64, i32, i32, P]
        L.pkv_decode_plan.restype = i32
        L.pkv_decode_plan.argtypes = [i32, i32, i32, i32, i32, i32, i32, pint, pint]
        L.pkv_decode_workspace_bytes.restype = sz
        L.pkv_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32]
        L.pkv_paged_attention_decode.restype = i32
        L.pkv_paged_attention_decode.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64,
                                                 f32, i32, P, sz, P, i32, P]
        L.pkv_paged_attention_prefill.restype = i32
        L.pkv_paged_attention_prefill.argtypes = [P, i32, P, i32, P, P, P, i32, P, i32, i32, i32,
                                                  i32, i32, i64, f32, P, i32, P]
        L.pkv_decode_cascade_workspace_bytes.restype = sz
        L.pkv_decode_cascade_workspace_bytes.argtypes = [i32] * 9
        L.pkv_decode_cascade_plan.restype = i32
        L.pkv_decode_cascade_plan.argtypes = [i32] * 10 + [pint, pint]
        L.pkv_paged_attention_decode_cascade.restype = i32
        L.pkv_paged_attention_decode_cascade.argtypes = [
            P, P, P, P, i32, P, P, i32, i32, P, i32, P, i32, i32, i32, i32, i32, i64, f32, i32, P,
            sz, P, i32, P]
        L.pkv_alloc_create.restype = P
        L.pkv_alloc_create.argtypes = [i64, i32, u64]
        L.pkv_alloc_destroy.restype = None
        L.pkv_alloc_destroy.argtypes = [P]
        L.pkv_alloc_num_free.restype = i64
        L.pkv_alloc_num_free.argtypes = [P]
        L.pkv_alloc_block_size.restype = i32
        L.pkv_alloc_block_size.argtypes = [P]
        L.pkv_alloc_refcount.restype = ctypes.c_int32
        L.pkv_alloc_refcount.argtypes = [P, ctypes.c_int32]
        L.pkv_alloc_new_seq.restype = i32
        L.pkv_alloc_new_seq.argtypes = [P, i64, pi32, i32, pint]
        L.pkv_alloc_fork.restype = i32
        L.pkv_alloc_fork.argtypes = [P, pi32, i32]
        L.pkv_alloc_append.restype = i32
        L.pkv_alloc_append.argtypes = [P, pi32, i32, pint, i64, i64, pi32, pi32, pint]
        L.pkv_alloc_free.restype = i32
        L.pkv_alloc_free.argtypes = [P, pi32, i32]
        L.pkv_block_hash.restype = u64
        L.pkv_block_hash.argtypes = [u64, pi32, i32]
        L.pkv_alloc_cache_insert.restype = i32
        L.pkv_alloc_cache_insert.argtypes = [P, u64, ctypes.c_int32]
        L.pkv_alloc_cache_lookup.restype = ctypes.c_int32
        L.pkv_alloc_cache_lookup.argtypes = [P, u64]
        L.pkv_alloc_new_seq_cached.restype = i32
        L.pkv_alloc_new_seq_cached.argtypes = [P, ctypes.POINTER(ctypes.c_uint64), i32, i64, pi32,
                                               i32, pint, pint]
        L.pkv_hbm_read_probe.restype = i32
        L.pkv_hbm_read_probe.argtypes = [P, sz, P, i32, P]
        L.pkv_hbm_gather_probe.restype = i32
        L.pkv_hbm_gather_probe.argtypes = [P, sz, P, i64, P, i32, P]
        _lib = L
        return L


def status_name(status: int) -> str:
    return lib().pkv_status_str(status).decode()


def _check(status: int, call: str) -> None:
    if status != OK:
        raise PagedKVError(status, call, lib().pkv_last_error().decode())


def _stream_handle(stream: Optional[torch.cuda.Stream], device: torch.device) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise ValueError(f"unsupported element type {t.dtype} (float16 or bfloat16)")
    return _DTYPES[t.dtype]


def version() -> str:
    return lib().pkv_version().decode()


def device_flags(device: Optional[int] = None, clear: bool = True) -> int:
    """Device error word (PKV_DEVFLAG_* bits); waits for the device."""
    dev = torch.cuda.current_device() if device is None else int(device)
    v = ctypes.c_uint(0)
    _check(lib().pkv_device_flags(dev, ctypes.byref(v), int(clear)), "pkv_device_flags")
    return v.value


def _block_ptr(t: torch.Tensor, name: str) -> int:
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    return t.data_ptr()


def copy_blocks(src_key_cache: torch.Tensor, src_value_cache: torch.Tensor,
                dst_key_cache: torch.Tensor, dst_value_cache: torch.Tensor,
                block_mapping: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """dst[block_mapping[i, 1]] = src[block_mapping[i, 0]] for K and V (copy-on-write
    within one pool, or swap between a device pool and pinned host memory)."""
    if block_mapping.dtype != torch.int32 or block_mapping.dim() != 2 or block_mapping.shape[1] != 2:
        raise ValueError("block_mapping must be int32 [num_pairs, 2]")
    for t in (src_value_cache, dst_key_cache, dst_value_cache):
        if t.shape[1:] != src_key_cache.shape[1:] or t.dtype != src_key_cache.dtype:
            raise ValueError("all caches must share block shape and element type")
    if src_value_cache.shape[0] != src_key_cache.shape[0] or dst_value_cache.shape[0] != dst_key_cache.shape[0]:
        raise ValueError("K and V pools must have the same number of blocks")
    block_bytes = src_key_cache[0].numel() * src_key_cache.element_size()
    dev = torch.device("cuda", torch.cuda.current_device())
    st = lib().pkv_copy_blocks(
        _block_ptr(src_key_cache, "src_key_cache"), _block_ptr(src_value_cache, "src_value_cache"),
        _block_ptr(dst_key_cache, "dst_key_cache"), _block_ptr(dst_value_cache, "dst_value_cache"),
        _block_ptr(block_mapping, "block_mapping"), block_mapping.shape[0], src_key_cache.shape[0],
        dst_key_cache.shape[0], block_bytes, _stream_handle(stream, dev))
    _check(st, "pkv_copy_blocks")


def selftest_bounded_wait(limit_ns: int, stream: Optional[torch.cuda.Stream] = None) -> None:
    """Launch the bounded-wait self-test kernel (see pkv_selftest_bounded_wait)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(lib().pkv_selftest_bounded_wait(int(limit_ns), _stream_handle(stream, dev)),
           "pkv_selftest_bounded_wait")


def hbm_read_probe(buf: torch.Tensor, sink: torch.Tensor, grid: int,
                   stream: Optional[torch.cuda.Stream] = None) -> None:
    """Read all of `buf` once (measurement of the read-only HBM ceiling); the
    fold of what was read lands in `sink` (an int32 CUDA tensor)."""
    if sink.dtype != torch.int32 or not sink.is_cuda:
        raise ValueError("sink must be an int32 CUDA tensor")
    _check(lib().pkv_hbm_read_probe(_dev(buf, "buf"), buf.numel() * buf.element_size(),
                                    _dev(sink, "sink"), int(grid), _stream_handle(stream, buf.device)),
           "pkv_hbm_read_probe")


def hbm_gather_probe(buf: torch.Tensor, chunk_bytes: int, order: torch.Tensor, sink: torch.Tensor,
                     grid: int, stream: Optional[torch.cuda.Stream] = None) -> None:
    """Read `buf` as whole chunks of chunk_bytes in the order `order` (int32 CUDA
    tensor of chunk indices) lists them; measurement of the paged-read ceiling."""
    if order.dtype != torch.int32 or not order.is_cuda or sink.dtype != torch.int32:
        raise ValueError("order and sink must be int32 CUDA tensors")
    n = (buf.numel() * buf.element_size()) // int(chunk_bytes)
    if order.numel() != n:
        raise ValueError("order must list every chunk of buf once")
    _check(lib().pkv_hbm_gather_probe(_dev(buf, "buf"), int(chunk_bytes), _dev(order, "order"), n,
                                      _dev(sink, "sink"), int(grid), _stream_handle(stream, buf.device)),
           "pkv_hbm_gather_probe")


def kv_cache_write(key: torch.Tensor, value: torch.Tensor, slot_mapping: torch.Tensor,
                   key_cache: torch.Tensor, value_cache: torch.Tensor,
                   stream: Optional[torch.cuda.Stream] = None) -> None:
    """key/value [T, Hkv, D] -> caches [NB, bs, Hkv, D] at slot_mapping[t] (int64)."""
    if key.dim() != 3 or key.shape != value.shape:
        raise ValueError("key/value must both be [num_tokens, num_kv_heads, head_dim]")
    if key_cache.dim() != 4 or key_cache.shape != value_cache.shape:
        raise ValueError("caches must both be [num_blocks, block_size, num_kv_heads, head_dim]")
    T, Hkv, D = key.shape
    NB, bs, Hkv2, D2 = key_cache.shape
    if (Hkv2, D2) != (Hkv, D):
        raise ValueError("cache heads/head_dim differ from key's")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape != (T,):
        raise ValueError("slot_mapping must be int64 [num_tokens]")
    dt = _dtype_code(key)
    for t in (value, key_cache, value_cache):
        if t.dtype != key.dtype:
            raise ValueError("key, value and caches must share one element type")
    st = lib().pkv_kv_cache_write(
        _dev(key, "key"), _dev(value, "value"), _dev(slot_mapping, "slot_mapping"), T, Hkv, D,
        _dev(key_cache, "key_cache"), _dev(value_cache, "value_cache"), NB, bs, dt,
        _stream_handle(stream, key.device))
    _check(st, "pkv_kv_cache_write")


def decode_plan(batch: int, num_heads: int, num_kv_heads: int, head_dim: int, max_blocks: int,
                block_size: int, partition_tokens: int = 0) -> tuple:
    """(partition length in tokens, partitions per sequence) the decode call will use."""
    pt, npart = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().pkv_decode_plan(batch, num_heads, num_kv_heads, head_dim, max_blocks, block_size,
                                 partition_tokens, ctypes.byref(pt), ctypes.byref(npart)),
           "pkv_decode_plan")
    return pt.value, npart.value


def decode_workspace_bytes(batch: int, num_heads: int, num_kv_heads: int, head_dim: int,
                           max_blocks: int, block_size: int, partition_tokens: int = 0) -> int:
    return int(lib().pkv_decode_workspace_bytes(batch, num_heads, num_kv_heads, head_dim,
                                                max_blocks, block_size, partition_tokens))


def paged_attention_decode(query: torch.Tensor, key_cache: torch.Tensor, value_cache: torch.Tensor,
                           block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                           partition_tokens: int = 0, out: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """query [B, Hq, D]; caches [NB, bs, Hkv, D]; block_tables int32 [B, max_blocks];
    context_lens int32 [B] -> out [B, Hq, D].  A workspace tensor (any dtype, at least
    decode_workspace_bytes(...) bytes) is allocated by torch when not given."""
    if query.dim() != 3:
        raise ValueError("query must be [batch, num_heads, head_dim]")
    if key_cache.dim() != 4 or key_cache.shape != value_cache.shape:
        raise ValueError("caches must both be [num_blocks, block_size, num_kv_heads, head_dim]")
    B, Hq, D = query.shape
    NB, bs, Hkv, D2 = key_cache.shape
    if D2 != D:
        raise ValueError("head_dim differs between query and caches")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be int32 [batch, max_blocks]")
    if context_lens.dtype != torch.int32 or context_lens.shape != (B,):
        raise ValueError("context_lens must be int32 [batch]")
    dt = _dtype_code(query)
    for t in (key_cache, value_cache):
        if t.dtype != query.dtype:
            raise ValueError("query and caches must share one element type")
    MB = block_tables.shape[1]
    if out is None:
        out = torch.empty_like(query)
    elif out.shape != query.shape or out.dtype != query.dtype:
        raise ValueError("out must match query's shape and type")
    need = decode_workspace_bytes(B, Hq, Hkv, D, MB, bs, partition_tokens)
    ws_ptr, ws_bytes = None, 0
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
        ws_ptr = _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    st = lib().pkv_paged_attention_decode(
        _dev(query, "query"), _dev(key_cache, "key_cache"), _dev(value_cache, "value_cache"),
        _dev(block_tables, "block_tables"), MB, _dev(context_lens, "context_lens"), B, Hq, Hkv, D,
        bs, NB, float(scale), int(partition_tokens), ws_ptr, ws_bytes, _dev(out, "out"), dt,
        _stream_handle(stream, query.device))
    _check(st, "pkv_paged_attention_decode")
    return out


def paged_attention_prefill(query: torch.Tensor, query_start: torch.Tensor, max_query_len: int,
                            key_cache: torch.Tensor, value_cache: torch.Tensor,
                            block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                            out: Optional[torch.Tensor] = None,
                            stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Causal chunk attention: query [T, Hq, D], query_start int32 [B+1] -> out [T, Hq, D]."""
    if query.dim() != 3:
        raise ValueError("query must be [total_tokens, num_heads, head_dim]")
    T, Hq, D = query.shape
    NB, bs, Hkv, _ = key_cache.shape
    B = block_tables.shape[0]
    if query_start.dtype != torch.int32 or query_start.shape != (B + 1,):
        raise ValueError("query_start must be int32 [batch + 1]")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables / context_lens must be int32")
    dt = _dtype_code(query)
    if out is None:
        out = torch.empty_like(query)
    st = lib().pkv_paged_attention_prefill(
        _dev(query, "query"), T, _dev(query_start, "query_start"), int(max_query_len),
        _dev(key_cache, "key_cache"), _dev(value_cache, "value_cache"),
        _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"),
        B, Hq, Hkv, D, bs, NB, float(scale), _dev(out, "out"), dt, _stream_handle(stream, query.device))
    _check(st, "pkv_paged_attention_prefill")
    return out


def decode_cascade_plan(batch: int, num_heads: int, num_kv_heads: int, head_dim: int,
                        max_prefix_blocks: int, max_suffix_blocks: int, max_group_size: int,
                        num_groups: int, block_size: int, partition_tokens: int = 0) -> tuple:
    """(one_pass, prefix_partitions) the cascade decode will use."""
    op, pp = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().pkv_decode_cascade_plan(batch, num_heads, num_kv_heads, head_dim, max_prefix_blocks,
                                         max_suffix_blocks, max_group_size, num_groups, block_size,
                                         partition_tokens, ctypes.byref(op), ctypes.byref(pp)),
           "pkv_decode_cascade_plan")
    return bool(op.value), pp.value


def paged_attention_decode_cascade(query: torch.Tensor, key_cache: torch.Tensor,
                                   value_cache: torch.Tensor, prefix_tables: torch.Tensor,
                                   prefix_lens: torch.Tensor, group_start: torch.Tensor,
                                   suffix_tables: torch.Tensor, suffix_lens: torch.Tensor,
                                   scale: float, max_group_size: int, partition_tokens: int = 0,
                                   out: Optional[torch.Tensor] = None,
                                   workspace: Optional[torch.Tensor] = None,
                                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Decode with shared prefixes read once per group (see include/pagedkv.h).
    prefix_tables int32 [G, MPB], prefix_lens int32 [G], group_start int32 [G+1],
    suffix_tables int32 [B, MSB], suffix_lens int32 [B] -> out [B, Hq, D]."""
    B, Hq, D = query.shape
    NB, bs, Hkv, _ = key_cache.shape
    for name, t, nd in (("prefix_tables", prefix_tables, 2), ("prefix_lens", prefix_lens, 1),
                        ("group_start", group_start, 1), ("suffix_tables", suffix_tables, 2),
                        ("suffix_lens", suffix_lens, 1)):
        if t.dtype != torch.int32 or t.dim() != nd:
            raise ValueError(f"{name} must be int32 with {nd} dims")
    G = prefix_tables.shape[0]
    if prefix_lens.shape != (G,) or group_start.shape != (G + 1,):
        raise ValueError("prefix_lens must be [num_groups], group_start [num_groups + 1]")
    if suffix_tables.shape[0] != B or suffix_lens.shape != (B,):
        raise ValueError("suffix_tables must be [batch, max_suffix_blocks], suffix_lens [batch]")
    dt = _dtype_code(query)
    if out is None:
        out = torch.empty_like(query)
    MPB, MSB = prefix_tables.shape[1], suffix_tables.shape[1]
    need = int(lib().pkv_decode_cascade_workspace_bytes(B, Hq, Hkv, D, MPB, MSB, max_group_size, bs,
                                                        partition_tokens))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=query.device)
    st = lib().pkv_paged_attention_decode_cascade(
        _dev(query, "query"), _dev(key_cache, "key_cache"), _dev(value_cache, "value_cache"),
        _dev(prefix_tables, "prefix_tables"), MPB, _dev(prefix_lens, "prefix_lens"),
        _dev(group_start, "group_start"), G, int(max_group_size), _dev(suffix_tables, "suffix_tables"),
        MSB, _dev(suffix_lens, "suffix_lens"), B, Hq, Hkv, D, bs, NB, float(scale),
        int(partition_tokens), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _dev(out, "out"), dt,
        _stream_handle(stream, query.device))
    _check(st, "pkv_paged_attention_decode_cascade")
    return out


class BlockAllocator:
    """Host block pool with free list, refcounts and copy-on-write (C++ in the library)."""

    def __init__(self, num_blocks: int, block_size: int, shuffle_seed: int = 0):
        h = lib().pkv_alloc_create(int(num_blocks), int(block_size), int(shuffle_seed))
        if not h:
            raise ValueError("pkv_alloc_create failed (bad sizes or host memory exhausted)")
        self._h = ctypes.c_void_p(h)
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().pkv_alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def num_free(self) -> int:
        return int(lib().pkv_alloc_num_free(self._h))

    def refcount(self, block: int) -> int:
        return int(lib().pkv_alloc_refcount(self._h, int(block)))

    @staticmethod
    def _arr(blocks, capacity=None):
        n = len(blocks) if capacity is None else capacity
        arr = (ctypes.c_int32 * max(1, n))()
        for i, b in enumerate(blocks):
            arr[i] = int(b)
        return arr

    def new_seq(self, num_tokens: int) -> list:
        cap = -(-int(num_tokens) // self.block_size)
        arr = self._arr([], cap)
        n = ctypes.c_int(0)
        _check(lib().pkv_alloc_new_seq(self._h, int(num_tokens), arr, cap, ctypes.byref(n)),
               "pkv_alloc_new_seq")
        return [arr[i] for i in range(n.value)]

    def fork(self, blocks: list) -> list:
        _check(lib().pkv_alloc_fork(self._h, self._arr(blocks), len(blocks)), "pkv_alloc_fork")
        return list(blocks)

    def append(self, blocks: list, old_len: int, new_len: int):
        """Grow in place; returns the copy-on-write pair (src, dst) or None."""
        cap = max(len(blocks), -(-int(new_len) // self.block_size))
        arr = self._arr(blocks, cap)
        n = ctypes.c_int(len(blocks))
        src, dst, ncow = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int(0)
        _check(lib().pkv_alloc_append(self._h, arr, cap, ctypes.byref(n), int(old_len), int(new_len),
                                      ctypes.byref(src), ctypes.byref(dst), ctypes.byref(ncow)),
               "pkv_alloc_append")
        blocks[:] = [arr[i] for i in range(n.value)]
        return (src.value, dst.value) if ncow.value else None

    def free(self, blocks: list) -> None:
        _check(lib().pkv_alloc_free(self._h, self._arr(blocks), len(blocks)), "pkv_alloc_free")

    # ---- automatic prefix caching ----
    def block_hashes(self, tokens: list) -> list:
        """Chained hashes of the full blocks of a token list."""
        out, parent, bs = [], 0, self.block_size
        for i in range(len(tokens) // bs):
            chunk = self._arr(tokens[i * bs:(i + 1) * bs])
            parent = int(lib().pkv_block_hash(parent, chunk, bs))
            out.append(parent)
        return out

    def cache_insert(self, block_hash: int, block: int) -> None:
        _check(lib().pkv_alloc_cache_insert(self._h, int(block_hash), int(block)),
               "pkv_alloc_cache_insert")

    def cache_lookup(self, block_hash: int) -> int:
        return int(lib().pkv_alloc_cache_lookup(self._h, int(block_hash)))

    def new_seq_cached(self, tokens: list) -> tuple:
        """(blocks, cached leading blocks reused) for a prompt of `tokens`."""
        hashes = self.block_hashes(tokens)
        cap = -(-len(tokens) // self.block_size)
        arr = self._arr([], cap)
        harr = (ctypes.c_uint64 * max(1, len(hashes)))(*hashes)
        n, hits = ctypes.c_int(0), ctypes.c_int(0)
        _check(lib().pkv_alloc_new_seq_cached(self._h, harr, len(hashes), len(tokens), arr, cap,
                                              ctypes.byref(n), ctypes.byref(hits)),
               "pkv_alloc_new_seq_cached")
        return [arr[i] for i in range(n.value)], hits.value
