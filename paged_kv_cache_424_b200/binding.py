"""Python binding of ``libpa.so``: the C-ABI calls of ``include/pa.h`` with the
same names, taking torch CUDA tensors.

Argument marshalling only: shapes and dtypes are read off the tensors into a
``pa_dims`` struct, pointers come from ``data_ptr()``, the stream from
``torch.cuda.current_stream()`` unless one is given.  Every operation runs in
the library's CUDA kernels; there is no fallback.  Importing this module
loads the library and raises :class:`LibraryMissing` if it is not built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_OK = 0
STATUS = {0: "PA_OK", -1: "PA_ERR_NULL", -2: "PA_ERR_DTYPE", -3: "PA_ERR_SHAPE", -4: "PA_ERR_UNSUPPORTED",
          -5: "PA_ERR_WORKSPACE", -6: "PA_ERR_CUDA", -7: "PA_ERR_ALIGN", -8: "PA_ERR_MEMORY"}
PA_F16, PA_BF16, PA_FP8_E4M3 = 0, 1, 2
DEVERR = {1: "BLOCK_ID", 2: "CONTEXT", 4: "SLOT", 8: "COPY_PAIR", 16: "TIMEOUT", 32: "LAYOUT"}
# torch dtypes accepted for an FP8 E4M3 cache (the codes as bytes, or torch's own e4m3fn type)
FP8_CACHE_DTYPES = (torch.uint8, torch.float8_e4m3fn)

# The C entry points declared in include/pa.h, in declaration order.
EXPORTS = ["pa_decode_workspace_size", "pa_decode_num_partitions", "pa_decode", "pa_decode_noalloc",
           "pa_decode_fp8", "pa_reshape_and_cache_fp8", "pa_decode_ext_workspace_size", "pa_decode_ext",
           "pa_prefix_cache_create", "pa_prefix_cache_destroy", "pa_prefix_cache_match", "pa_prefix_cache_insert",
           "pa_prefix_cache_release", "pa_prefix_cache_evict", "pa_prefix_cache_stats", "pa_prefix_order",
           "pa_reshape_and_cache", "pa_copy_blocks", "pa_swap_blocks", "pa_check_wait_timeout", "pa_last_error",
           "pa_device_error", "pa_version"]


class LibraryMissing(RuntimeError):
    pass


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class pa_dims(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32),
                ("num_blocks", ctypes.c_int64), ("dtype", ctypes.c_int32), ("kv_dtype", ctypes.c_int32)]


class pa_decode_opts(ctypes.Structure):
    _fields_ = [("q_len", ctypes.c_int32), ("window", ctypes.c_int32), ("k_scale", ctypes.c_float),
                ("v_scale", ctypes.c_float), ("seq_order", ctypes.c_void_p)]


def _load(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise LibraryMissing(f"{path} is not built; run `python -m paged_kv_cache_424_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    dp = ctypes.POINTER(pa_dims)
    lib.pa_decode_workspace_size.argtypes = [dp, i32, i32]
    lib.pa_decode_workspace_size.restype = u64
    lib.pa_decode_num_partitions.argtypes = [dp, i32, i32]
    lib.pa_decode_num_partitions.restype = i32
    lib.pa_decode.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_float, i32, dp, i32, i32, vp, u64, vp]
    lib.pa_decode.restype = ctypes.c_int
    lib.pa_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_float, i32, dp, i32, i32, vp]
    lib.pa_decode_noalloc.restype = ctypes.c_int
    f32 = ctypes.c_float
    lib.pa_decode_fp8.argtypes = [vp, vp, vp, vp, vp, vp, f32, f32, f32, i32, dp, i32, i32, vp, u64, vp]
    lib.pa_decode_fp8.restype = ctypes.c_int
    lib.pa_reshape_and_cache_fp8.argtypes = [vp, vp, vp, vp, vp, i32, dp, f32, f32, vp]
    lib.pa_reshape_and_cache_fp8.restype = ctypes.c_int
    op = ctypes.POINTER(pa_decode_opts)
    lib.pa_decode_ext_workspace_size.argtypes = [dp, op, i32, i32]
    lib.pa_decode_ext_workspace_size.restype = u64
    lib.pa_decode_ext.argtypes = [vp, vp, vp, vp, vp, vp, f32, i32, dp, op, i32, i32, vp, u64, vp]
    lib.pa_decode_ext.restype = ctypes.c_int
    ip = ctypes.POINTER(ctypes.c_int32)
    lp = ctypes.POINTER(ctypes.c_int64)
    lib.pa_prefix_cache_create.argtypes = [i64]
    lib.pa_prefix_cache_create.restype = vp
    lib.pa_prefix_cache_destroy.argtypes = [vp]
    lib.pa_prefix_cache_destroy.restype = None
    lib.pa_prefix_cache_match.argtypes = [vp, ip, i32, ip, i32]
    lib.pa_prefix_cache_match.restype = i32
    lib.pa_prefix_cache_insert.argtypes = [vp, ip, i32, ip, i32]
    lib.pa_prefix_cache_insert.restype = ctypes.c_int
    lib.pa_prefix_cache_release.argtypes = [vp, ip, i32]
    lib.pa_prefix_cache_release.restype = i32
    lib.pa_prefix_cache_evict.argtypes = [vp, i32, ip]
    lib.pa_prefix_cache_evict.restype = i32
    lib.pa_prefix_cache_stats.argtypes = [vp, lp, lp, lp, lp]
    lib.pa_prefix_cache_stats.restype = ctypes.c_int
    lib.pa_prefix_order.argtypes = [ip, ip, i32, i32, ip]
    lib.pa_prefix_order.restype = ctypes.c_int
    lib.pa_reshape_and_cache.argtypes = [vp, vp, vp, vp, vp, i32, dp, vp]
    lib.pa_reshape_and_cache.restype = ctypes.c_int
    lib.pa_copy_blocks.argtypes = [vp, vp, i32, vp, i32, dp, vp]
    lib.pa_copy_blocks.restype = ctypes.c_int
    lib.pa_swap_blocks.argtypes = [vp, vp, i64, vp, vp, i64, vp, i32, dp, vp]
    lib.pa_swap_blocks.restype = ctypes.c_int
    lib.pa_last_error.argtypes = []
    lib.pa_last_error.restype = ctypes.c_char_p
    lib.pa_check_wait_timeout.argtypes = [i32, vp]
    lib.pa_check_wait_timeout.restype = ctypes.c_int
    lib.pa_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.pa_device_error.restype = ctypes.c_int
    lib.pa_version.argtypes = []
    lib.pa_version.restype = i32
    return lib


LIB = _load()


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------
def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError(f"expected float16 or bfloat16, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _check(status: int) -> None:
    if status != PA_OK:
        raise PagedAttentionError(status, LIB.pa_last_error().decode(errors="replace"))


def _need_cuda(*ts: Optional[torch.Tensor]) -> None:
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _kv_code(cache: torch.Tensor) -> int:
    return PA_FP8_E4M3 if cache.dtype in FP8_CACHE_DTYPES else _dtype_code(cache)


def make_dims(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int, block_size: int,
              max_blocks_per_seq: int, num_blocks: int, dtype: int, kv_dtype: int = 0) -> pa_dims:
    return pa_dims(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, dtype,
                   kv_dtype)


def dims_of(q: torch.Tensor, k_cache: torch.Tensor, block_tables: torch.Tensor) -> pa_dims:
    S, H, D = q.shape
    NB, Hk, B, D2 = k_cache.shape
    if D2 != D:
        raise ValueError("q and k_cache disagree on head_dim")
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    return make_dims(S, H, Hk, D, B, MB, NB, _dtype_code(q), _kv_code(k_cache))


def cache_dims(k_cache: torch.Tensor, dtype: Optional[torch.dtype] = None) -> pa_dims:
    """Block geometry of a cache; `dtype` is the 16-bit type of the tokens
    written into it (taken from the cache itself unless it is FP8)."""
    NB, Hk, B, D = k_cache.shape
    kv = _kv_code(k_cache)
    if dtype is not None:
        code = _dtype_code(torch.empty(0, dtype=dtype))
    else:
        code = PA_F16 if kv == PA_FP8_E4M3 else kv
    return make_dims(0, Hk, Hk, D, B, 0, NB, code, kv)


# ---------------------------------------------------------------------------
# the C-ABI calls
# ---------------------------------------------------------------------------
def pa_version() -> int:
    return int(LIB.pa_version())


def pa_last_error() -> str:
    return LIB.pa_last_error().decode(errors="replace")


def pa_decode_workspace_size(dims: pa_dims, max_context_len: int, partition_tokens: int = 0) -> int:
    n = LIB.pa_decode_workspace_size(ctypes.byref(dims), int(max_context_len), int(partition_tokens))
    if n == ctypes.c_size_t(-1).value:
        raise PagedAttentionError(-3, pa_last_error())
    return int(n)


def pa_decode_num_partitions(dims: pa_dims, max_context_len: int, partition_tokens: int = 0) -> int:
    n = int(LIB.pa_decode_num_partitions(ctypes.byref(dims), int(max_context_len), int(partition_tokens)))
    if n < 0:
        raise PagedAttentionError(n, pa_last_error())
    return n


def pa_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, num_kv_heads: int,
              max_context_len: int, partition_tokens: int = 0, workspace: Optional[torch.Tensor] = None,
              stream=None) -> torch.Tensor:
    """out[s, h] = softmax(scale * q[s, h] . K_s^T) V_s over the paged cache."""
    _need_cuda(out, q, k_cache, v_cache, block_tables, context_lens, workspace)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    dims = dims_of(q, k_cache, block_tables)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = LIB.pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
                       float(scale), int(num_kv_heads), ctypes.byref(dims), int(max_context_len),
                       int(partition_tokens), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st)
    return out


def pa_decode_noalloc(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, num_kv_heads: int,
                      max_context_len: int, partition_tokens: int = 0, stream=None) -> torch.Tensor:
    """pa_decode without a workspace argument: the split-KV scratch is the
    library's own 64 MiB device array, for callers that cannot allocate.
    Calls that overlap on the GPU race on that shared scratch."""
    _need_cuda(out, q, k_cache, v_cache, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    dims = dims_of(q, k_cache, block_tables)
    st = LIB.pa_decode_noalloc(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                               _ptr(context_lens), float(scale), int(num_kv_heads), ctypes.byref(dims),
                               int(max_context_len), int(partition_tokens), _stream(stream))
    _check(st)
    return out


def pa_decode_fp8(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, k_scale: float,
                  v_scale: float, num_kv_heads: int, max_context_len: int, partition_tokens: int = 0,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """pa_decode over FP8 E4M3 caches (uint8 or float8_e4m3fn tensors):
    K = code * k_scale, V = code * v_scale."""
    _need_cuda(out, q, k_cache, v_cache, block_tables, context_lens, workspace)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if k_cache.dtype not in FP8_CACHE_DTYPES or v_cache.dtype not in FP8_CACHE_DTYPES:
        raise TypeError("FP8 caches must be uint8 or float8_e4m3fn tensors")
    dims = dims_of(q, k_cache, block_tables)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = LIB.pa_decode_fp8(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
                           float(scale), float(k_scale), float(v_scale), int(num_kv_heads), ctypes.byref(dims),
                           int(max_context_len), int(partition_tokens), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st)
    return out


def pa_decode_ext_workspace_size(dims: pa_dims, opts: pa_decode_opts, max_context_len: int,
                                 partition_tokens: int = 0) -> int:
    n = LIB.pa_decode_ext_workspace_size(ctypes.byref(dims), ctypes.byref(opts), int(max_context_len),
                                         int(partition_tokens))
    if n == ctypes.c_size_t(-1).value:
        raise PagedAttentionError(-3, pa_last_error())
    return int(n)


def ext_dims(q: torch.Tensor, k_cache: torch.Tensor, block_tables: torch.Tensor) -> pa_dims:
    """dims of a [S, q_len, H, D] query batch."""
    S, QL, H, D = q.shape
    return dims_of(q.view(S, QL * H, D)[:, :H], k_cache, block_tables)


def pa_decode_ext(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, num_kv_heads: int,
                  max_context_len: int, q_len: int = 1, window: int = 0, k_scale: float = 1.0, v_scale: float = 1.0,
                  partition_tokens: int = 0, workspace: Optional[torch.Tensor] = None, stream=None,
                  seq_order: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Multi-token / sliding-window decode: q and out are [S, q_len, H, D];
    query i of sequence s sits at position context_lens[s] - q_len + i and
    attends to its `window` most recent positions (all when 0).  The caches
    may be 16-bit or FP8 E4M3 (uint8 / float8_e4m3fn)."""
    _need_cuda(out, q, k_cache, v_cache, block_tables, context_lens, workspace)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if q.dim() != 4 or q.shape[1] != q_len or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q and out must be [num_seqs, q_len, num_heads, head_dim]")
    dims = ext_dims(q, k_cache, block_tables)
    if seq_order is not None:
        _need_cuda(seq_order)
        if seq_order.dtype != torch.int32 or seq_order.numel() != q.shape[0]:
            raise TypeError("seq_order must be int32 [num_seqs]")
    opts = pa_decode_opts(int(q_len), int(window), float(k_scale), float(v_scale),
                          None if seq_order is None else seq_order.data_ptr())
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = LIB.pa_decode_ext(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
                           float(scale), int(num_kv_heads), ctypes.byref(dims), ctypes.byref(opts),
                           int(max_context_len), int(partition_tokens), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st)
    return out


# ---------------------------------------------------------------------------
# prefix caching (host)
# ---------------------------------------------------------------------------
def _i32p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


class PrefixCache:
    """The library's host prefix cache (pa_prefix_cache_*): token ids of
    full 16-token blocks -> the physical blocks holding their K/V."""

    def __init__(self, num_blocks: int):
        self._h = LIB.pa_prefix_cache_create(int(num_blocks))
        if not self._h:
            raise PagedAttentionError(-3, pa_last_error())

    def close(self) -> None:
        if self._h:
            LIB.pa_prefix_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def match(self, tokens) -> list:
        import numpy as np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        out = np.zeros(max(1, t.size // 16), dtype=np.int32)
        n = LIB.pa_prefix_cache_match(self._h, _i32p(t), int(t.size), _i32p(out), int(t.size // 16))
        if n < 0:
            raise PagedAttentionError(n, pa_last_error())
        return out[:n].tolist()

    def insert(self, tokens, blocks) -> None:
        import numpy as np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        b = np.ascontiguousarray(blocks, dtype=np.int32)
        _check(LIB.pa_prefix_cache_insert(self._h, _i32p(t), int(t.size), _i32p(b), int(b.size)))

    def release(self, blocks) -> int:
        import numpy as np
        b = np.ascontiguousarray(blocks, dtype=np.int32)
        n = LIB.pa_prefix_cache_release(self._h, _i32p(b), int(b.size))
        if n < 0:
            raise PagedAttentionError(n, pa_last_error())
        return int(n)

    def evict(self, max_blocks: int) -> list:
        import numpy as np
        out = np.zeros(max(1, max_blocks), dtype=np.int32)
        n = LIB.pa_prefix_cache_evict(self._h, int(max_blocks), _i32p(out))
        if n < 0:
            raise PagedAttentionError(n, pa_last_error())
        return out[:n].tolist()

    def stats(self) -> dict:
        v = [ctypes.c_int64(0) for _ in range(4)]
        _check(LIB.pa_prefix_cache_stats(self._h, *[ctypes.byref(x) for x in v]))
        return dict(zip(("cached", "evictable", "hits", "lookups"), (x.value for x in v)))


def pa_prefix_order(block_tables, context_lens):
    """Host: the shared-prefix-aware order of the batch (numpy int32 [S])."""
    import numpy as np
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S = cl.shape[0]
    MB = bt.shape[1] if bt.ndim == 2 else 0
    order = np.zeros(max(1, S), dtype=np.int32)
    _check(LIB.pa_prefix_order(_i32p(bt), _i32p(cl), int(S), int(MB), _i32p(order)))
    return order[:S]


def pa_reshape_and_cache_fp8(key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                             slot_mapping: torch.Tensor, k_scale: float, v_scale: float, stream=None) -> None:
    """k_cache[slot // 16, :, slot % 16] = e4m3(key[t] / k_scale) (and V) for slot >= 0."""
    _need_cuda(key, value, k_cache, v_cache, slot_mapping)
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    if k_cache.dtype not in FP8_CACHE_DTYPES or v_cache.dtype not in FP8_CACHE_DTYPES:
        raise TypeError("FP8 caches must be uint8 or float8_e4m3fn tensors")
    dims = cache_dims(k_cache, key.dtype)
    st = LIB.pa_reshape_and_cache_fp8(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                                      int(slot_mapping.numel()), ctypes.byref(dims), float(k_scale), float(v_scale),
                                      _stream(stream))
    _check(st)


def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                         slot_mapping: torch.Tensor, stream=None) -> None:
    """k_cache[slot // 16, :, slot % 16] = key[t] (and V) for slot >= 0."""
    _need_cuda(key, value, k_cache, v_cache, slot_mapping)
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    dims = cache_dims(k_cache)
    st = LIB.pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                                  int(slot_mapping.numel()), ctypes.byref(dims), _stream(stream))
    _check(st)


def pa_copy_blocks(k_caches: Sequence[torch.Tensor], v_caches: Sequence[torch.Tensor],
                   block_mapping: torch.Tensor, stream=None) -> None:
    """Per layer: block dst of K and V becomes a copy of block src."""
    if len(k_caches) != len(v_caches) or not k_caches:
        raise ValueError("need matching, non-empty lists of K and V caches")
    _need_cuda(*k_caches, *v_caches, block_mapping)
    if block_mapping.dtype != torch.int64:
        raise TypeError("block_mapping must be int64")
    L = len(k_caches)
    kp = (ctypes.c_void_p * L)(*[t.data_ptr() for t in k_caches])
    vp = (ctypes.c_void_p * L)(*[t.data_ptr() for t in v_caches])
    dims = cache_dims(k_caches[0])
    pairs = block_mapping.numel() // 2
    st = LIB.pa_copy_blocks(ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p), L,
                            _ptr(block_mapping), int(pairs), ctypes.byref(dims), _stream(stream))
    _check(st)


def pa_swap_blocks(src_k: torch.Tensor, src_v: torch.Tensor, dst_k: torch.Tensor, dst_v: torch.Tensor,
                   block_mapping: torch.Tensor, stream=None) -> None:
    """Block dst of the destination pools becomes a copy of block src of the
    source pools; each pool a CUDA tensor or a pinned CPU tensor."""
    for t in (src_k, src_v, dst_k, dst_v, block_mapping):
        if not t.is_contiguous() or not (t.is_cuda or t.is_pinned()):
            raise ValueError("pools and mapping must be contiguous CUDA tensors or pinned CPU tensors")
    if block_mapping.dtype != torch.int64:
        raise TypeError("block_mapping must be int64")
    if src_k.shape[1:] != dst_k.shape[1:] or src_v.shape != src_k.shape or dst_v.shape != dst_k.shape:
        raise ValueError("pools disagree on the block shape")
    dims = cache_dims(src_k)
    st = LIB.pa_swap_blocks(_ptr(src_k), _ptr(src_v), int(src_k.shape[0]), _ptr(dst_k), _ptr(dst_v),
                            int(dst_k.shape[0]), _ptr(block_mapping), int(block_mapping.numel() // 2),
                            ctypes.byref(dims), _stream(stream))
    _check(st)


def pa_check_wait_timeout(milliseconds: int = 50, stream=None) -> None:
    """Enqueue the bounded-wait diagnostic (a wait that can never complete
    gives up after about `milliseconds` and flags PA_DEVERR_TIMEOUT)."""
    _check(LIB.pa_check_wait_timeout(int(milliseconds), _stream(stream)))


def pa_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    w = ctypes.c_uint32(0)
    _check(LIB.pa_device_error(_stream(stream), ctypes.byref(w)))
    return int(w.value)
