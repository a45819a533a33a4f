"""CPU oracle for paged decode attention, reshape_and_cache and copy_blocks.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library (``paged_kv_cache_424_b200``) and never imports it.

The arithmetic lives in ``pa_oracle.c`` (plain C, double precision, OpenMP over
(sequence, head) pairs), built into ``liboracle.so`` by :func:`build`.  This
module only marshals numpy arrays into it.  ``brute.py`` holds a pure-Python
restatement for tiny inputs.

Every function below states what it computes; the C source cites the pages.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F16 = 0
BF16 = 1
_DTYPE_CODE = {"f16": F16, "fp16": F16, "float16": F16, "bf16": BF16, "bfloat16": BF16}

_lib = None


def build(src: str = _SRC, out: str = _LIB, extra: Sequence[str] = ()) -> str:
    """Compile the C oracle with gcc into a shared library and return its path.

    The library is written to a temporary name and renamed over ``out``, so a
    process that already has the old library mapped keeps a valid mapping."""
    tmp = f"{out}.tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", *extra, "-o", tmp, src, "-lm"]
    try:
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    finally:
        if os.path.exists(tmp):
            os.remove(tmp)
    return out


def _stale(lib: str, src: str) -> bool:
    return not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src)


def load(path: str | None = None):
    """Load (building first if missing or stale) and return an :class:`Oracle`."""
    global _lib
    if path is not None:
        return Oracle(path)
    if _lib is None:
        if _stale(_LIB, _SRC):
            build()
        _lib = Oracle(_LIB)
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class OracleError(RuntimeError):
    pass


class Oracle:
    """ctypes handle on one build of ``pa_oracle.c``."""

    def __init__(self, path: str):
        self.path = path
        lib = ctypes.CDLL(path)
        vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_paged_decode.argtypes = [vp, vp, vp, vp, vp, vp, dbl, i32, i32, i32, i32, i32, i32, i64, i32]
        lib.oracle_paged_decode.restype = ctypes.c_int
        lib.oracle_reshape_and_cache.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i64]
        lib.oracle_reshape_and_cache.restype = ctypes.c_int
        lib.oracle_copy_blocks.argtypes = [vp, vp, i32, vp, i32, i32, i32, i32, i64]
        lib.oracle_copy_blocks.restype = ctypes.c_int
        lib.oracle_swap_blocks.argtypes = [vp, vp, i64, vp, vp, i64, vp, i32, i32, i32, i32]
        lib.oracle_swap_blocks.restype = ctypes.c_int
        lib.oracle_paged_decode_fp8.argtypes = [vp, vp, vp, vp, vp, vp, dbl, dbl, dbl, i32, i32, i32, i32, i32,
                                                 i32, i64, i32]
        lib.oracle_paged_decode_fp8.restype = ctypes.c_int
        lib.oracle_reshape_and_cache_fp8.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i64, i32,
                                                     ctypes.c_float, ctypes.c_float]
        lib.oracle_reshape_and_cache_fp8.restype = ctypes.c_int
        lib.oracle_paged_decode_ext.argtypes = [vp, vp, vp, vp, vp, vp, dbl, dbl, dbl, i32, i32, i32, i32, i32,
                                                i32, i64, i32, i32, i32, i32]
        lib.oracle_paged_decode_ext.restype = ctypes.c_int
        lib.oracle_quantize_e4m3_n.argtypes = [vp, vp, i64]
        lib.oracle_quantize_e4m3_n.restype = None
        lib.oracle_widen_e4m3_n.argtypes = [vp, vp, i64]
        lib.oracle_widen_e4m3_n.restype = None
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = ctypes.c_int
        lib.oracle_max_threads.restype = ctypes.c_int
        self._lib = lib

    # -- threads ---------------------------------------------------------
    def set_num_threads(self, n: int) -> int:
        return int(self._lib.oracle_set_num_threads(int(n)))

    def max_threads(self) -> int:
        return int(self._lib.oracle_max_threads())

    # -- operations ------------------------------------------------------
    def paged_decode(self, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                     dtype: str) -> np.ndarray:
        """out[s, h, :] = softmax(scale * q[s,h] . K_s^T) V_s, in float64.

        ``q`` is ``[S, H, D]`` and the caches ``[NB, Hk, B, D]``, all uint16
        bit patterns of ``dtype``; K_s / V_s are gathered through
        ``block_tables`` (``[S, MB]`` int32) for the first ``context_lens[s]``
        positions.
        """
        q = np.ascontiguousarray(q, dtype=np.uint16)
        k_cache = np.ascontiguousarray(k_cache, dtype=np.uint16)
        v_cache = np.ascontiguousarray(v_cache, dtype=np.uint16)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, H, D = q.shape
        NB, Hk, B, D2 = k_cache.shape
        if D2 != D or v_cache.shape != k_cache.shape or bt.shape[0] != S or cl.shape != (S,):
            raise OracleError("shape mismatch")
        MB = bt.shape[1] if bt.ndim == 2 else 0
        out = np.zeros((S, H, D), dtype=np.float64)
        rc = self._lib.oracle_paged_decode(_p(out), _p(q), _p(k_cache), _p(v_cache), _p(bt), _p(cl),
                                           float(scale), S, H, Hk, D, B, MB, NB, _DTYPE_CODE[dtype])
        if rc != 0:
            raise OracleError(f"oracle_paged_decode returned {rc}")
        return out

    def reshape_and_cache(self, k_cache, v_cache, key, value, slot_mapping) -> None:
        """In place: k_cache[slot // B, :, slot % B, :] = key[t] for slot >= 0."""
        for a in (k_cache, v_cache):
            if a.dtype != np.uint16 or not a.flags.c_contiguous:
                raise OracleError("caches must be C-contiguous uint16")
        key = np.ascontiguousarray(key, dtype=np.uint16)
        value = np.ascontiguousarray(value, dtype=np.uint16)
        sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        NB, Hk, B, D = k_cache.shape
        T = sm.shape[0]
        if key.shape != (T, Hk, D) or value.shape != (T, Hk, D):
            raise OracleError("key/value shape mismatch")
        rc = self._lib.oracle_reshape_and_cache(_p(k_cache), _p(v_cache), _p(key), _p(value), _p(sm),
                                                T, Hk, D, B, NB)
        if rc != 0:
            raise OracleError(f"oracle_reshape_and_cache returned {rc}")

    def copy_blocks(self, k_caches, v_caches, block_mapping) -> None:
        """In place, per layer: block dst of K and V becomes a copy of block src."""
        bm = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
        L = len(k_caches)
        if L != len(v_caches) or L == 0:
            raise OracleError("need matching non-empty K and V cache lists")
        NB, Hk, B, D = k_caches[0].shape
        for a in list(k_caches) + list(v_caches):
            if a.shape != (NB, Hk, B, D) or a.dtype != np.uint16 or not a.flags.c_contiguous:
                raise OracleError("every cache must be C-contiguous uint16 of one shape")
        kp = (ctypes.c_void_p * L)(*[a.ctypes.data for a in k_caches])
        vp = (ctypes.c_void_p * L)(*[a.ctypes.data for a in v_caches])
        rc = self._lib.oracle_copy_blocks(ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p),
                                          L, _p(bm), bm.shape[0], Hk, D, B, NB)
        if rc != 0:
            raise OracleError(f"oracle_copy_blocks returned {rc}")

    def swap_blocks(self, dst_k, dst_v, src_k, src_v, block_mapping) -> None:
        """In place: block dst of the destination pools becomes a copy of block
        src of the source pools (K and V)."""
        bm = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
        NBd, Hk, B, D = dst_k.shape
        NBs = src_k.shape[0]
        for a, nb in ((dst_k, NBd), (dst_v, NBd), (src_k, NBs), (src_v, NBs)):
            if a.shape != (nb, Hk, B, D) or a.dtype != np.uint16 or not a.flags.c_contiguous:
                raise OracleError("pools must be C-contiguous uint16 with matching block shapes")
        rc = self._lib.oracle_swap_blocks(_p(dst_k), _p(dst_v), NBd, _p(src_k), _p(src_v), NBs, _p(bm),
                                          bm.shape[0], Hk, D, B)
        if rc != 0:
            raise OracleError(f"oracle_swap_blocks returned {rc}")

    # -- FP8 E4M3 KV cache ---------------------------------------------------
    def quantize_e4m3(self, y) -> np.ndarray:
        """float32 values -> E4M3 codes (nearest, ties to even, clamped to 448)."""
        y = np.ascontiguousarray(y, dtype=np.float32)
        out = np.empty(y.shape, dtype=np.uint8)
        self._lib.oracle_quantize_e4m3_n(_p(out), _p(y), y.size)
        return out

    def widen_e4m3(self, c) -> np.ndarray:
        c = np.ascontiguousarray(c, dtype=np.uint8)
        out = np.empty(c.shape, dtype=np.float64)
        self._lib.oracle_widen_e4m3_n(_p(out), _p(c), c.size)
        return out

    def paged_decode_fp8(self, q, k_cache, v_cache, block_tables, context_lens, scale: float, k_scale: float,
                         v_scale: float, dtype: str) -> np.ndarray:
        """paged_decode over E4M3 caches: K = decode(code) * k_scale, V likewise."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        k_cache = np.ascontiguousarray(k_cache, dtype=np.uint8)
        v_cache = np.ascontiguousarray(v_cache, dtype=np.uint8)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, H, D = q.shape
        NB, Hk, B, D2 = k_cache.shape
        if D2 != D or v_cache.shape != k_cache.shape or bt.shape[0] != S or cl.shape != (S,):
            raise OracleError("shape mismatch")
        MB = bt.shape[1] if bt.ndim == 2 else 0
        out = np.zeros((S, H, D), dtype=np.float64)
        rc = self._lib.oracle_paged_decode_fp8(_p(out), _p(q), _p(k_cache), _p(v_cache), _p(bt), _p(cl),
                                               float(scale), float(k_scale), float(v_scale), S, H, Hk, D, B, MB,
                                               NB, _DTYPE_CODE[dtype])
        if rc != 0:
            raise OracleError(f"oracle_paged_decode_fp8 returned {rc}")
        return out

    def paged_decode_ext(self, q, k_cache, v_cache, block_tables, context_lens, scale: float, dtype: str,
                         q_len: int = 1, window: int = 0, k_scale: float = 1.0, v_scale: float = 1.0) -> np.ndarray:
        """Multi-token / sliding-window decode: q and the result are
        ``[S, q_len, H, D]``; query i of sequence s sits at position
        ``context_lens[s] - q_len + i`` and attends causally to the ``window``
        most recent positions (all when 0).  The caches hold 16-bit bit
        patterns (uint16) or E4M3 codes (uint8); K and V are scaled by
        ``k_scale`` / ``v_scale``."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        if k_cache.dtype not in (np.uint16, np.uint8) or v_cache.dtype != k_cache.dtype:
            raise OracleError("caches must both be uint16 (16-bit) or uint8 (E4M3)")
        k_cache = np.ascontiguousarray(k_cache)
        v_cache = np.ascontiguousarray(v_cache)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, QL, H, D = q.shape
        NB, Hk, B, D2 = k_cache.shape
        if QL != q_len or D2 != D or v_cache.shape != k_cache.shape or bt.shape[0] != S or cl.shape != (S,):
            raise OracleError("shape mismatch")
        MB = bt.shape[1] if bt.ndim == 2 else 0
        out = np.zeros((S, q_len, H, D), dtype=np.float64)
        rc = self._lib.oracle_paged_decode_ext(_p(out), _p(q), _p(k_cache), _p(v_cache), _p(bt), _p(cl),
                                               float(scale), float(k_scale), float(v_scale), S, H, Hk, D, B, MB,
                                               NB, _DTYPE_CODE[dtype], int(k_cache.dtype == np.uint8), int(q_len),
                                               int(window))
        if rc != 0:
            raise OracleError(f"oracle_paged_decode_ext returned {rc}")
        return out

    def reshape_and_cache_fp8(self, k_cache, v_cache, key, value, slot_mapping, dtype: str, k_scale: float,
                              v_scale: float) -> None:
        """In place: E4M3 codes of key[t] / k_scale (value[t] / v_scale) into slot[t]."""
        for a in (k_cache, v_cache):
            if a.dtype != np.uint8 or not a.flags.c_contiguous:
                raise OracleError("FP8 caches must be C-contiguous uint8")
        key = np.ascontiguousarray(key, dtype=np.uint16)
        value = np.ascontiguousarray(value, dtype=np.uint16)
        sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        NB, Hk, B, D = k_cache.shape
        T = sm.shape[0]
        if key.shape != (T, Hk, D) or value.shape != (T, Hk, D):
            raise OracleError("key/value shape mismatch")
        rc = self._lib.oracle_reshape_and_cache_fp8(_p(k_cache), _p(v_cache), _p(key), _p(value), _p(sm), T, Hk,
                                                    D, B, NB, _DTYPE_CODE[dtype], float(k_scale), float(v_scale))
        if rc != 0:
            raise OracleError(f"oracle_reshape_and_cache_fp8 returned {rc}")


def paged_decode(*args, **kw):
    return load().paged_decode(*args, **kw)


def reshape_and_cache(*args, **kw):
    return load().reshape_and_cache(*args, **kw)


def copy_blocks(*args, **kw):
    return load().copy_blocks(*args, **kw)
