"""Replays workload steps on a host-memory KV pool through the C oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The device pool has ``num_blocks`` physical blocks, most of them never
touched.  On the host only the touched blocks are kept, as rows of a compact
slab; ``row_of[physical id]`` names a block's row.  Oracle calls see the slab
and block ids relabelled to rows.  Relabelling is allowed because decode
attention depends only on the logical order of blocks, not on where they sit
(a property the pin tests check on the oracle itself).
"""
from __future__ import annotations

from typing import List, Optional

import numpy as np

from . import load

NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0, "fp8": 0x7F}


class HostPool:
    """Compact host mirror of a paged K/V pool: uint16 bit patterns of a
    16-bit cache, or uint8 codes of an FP8 E4M3 cache (``dtype="fp8"``)."""

    def __init__(self, num_blocks: int, num_kv_heads: int, block_size: int, head_dim: int,
                 dtype: str, capacity: int = 64):
        self.num_blocks = num_blocks
        self.shape = (num_kv_heads, block_size, head_dim)
        self.dtype = dtype
        self.store = np.uint8 if dtype == "fp8" else np.uint16
        self.row_of = np.full(num_blocks, -1, dtype=np.int64)
        self.ids: List[int] = []
        cap = max(1, capacity)
        self.k = np.full((cap, *self.shape), NAN_BITS[dtype], dtype=self.store)
        self.v = np.full((cap, *self.shape), NAN_BITS[dtype], dtype=self.store)
        self.n = 0

    def _grow(self, need: int) -> None:
        cap = self.k.shape[0]
        if need <= cap:
            return
        new = max(need, 2 * cap)
        for name in ("k", "v"):
            old = getattr(self, name)
            arr = np.full((new, *self.shape), NAN_BITS[self.dtype], dtype=self.store)
            arr[:self.n] = old[:self.n]
            setattr(self, name, arr)

    def rows(self, ids: np.ndarray) -> np.ndarray:
        """Rows of the given physical ids, creating NaN rows for new ones."""
        ids = np.asarray(ids, dtype=np.int64).ravel()
        if ids.size and (ids.min() < 0 or ids.max() >= self.num_blocks):
            raise ValueError("physical block id out of range")
        fresh = np.unique(ids[self.row_of[ids] < 0])
        if fresh.size:
            self._grow(self.n + fresh.size)
            self.row_of[fresh] = np.arange(self.n, self.n + fresh.size)
            self.ids.extend(int(x) for x in fresh)
            self.n += fresh.size
        return self.row_of[ids]

    def admit(self, ids: np.ndarray, k: np.ndarray, v: np.ndarray) -> None:
        r = self.rows(ids)
        self.k[r] = k
        self.v[r] = v

    def block(self, phys: int):
        r = self.row_of[phys]
        if r < 0:
            raise KeyError(phys)
        return self.k[r], self.v[r]

    def relabel_slots(self, slot_mapping: np.ndarray, block_size: int) -> np.ndarray:
        sm = np.asarray(slot_mapping, dtype=np.int64)
        out = sm.copy()
        live = sm >= 0
        if live.any():
            out[live] = self.rows(sm[live] // block_size) * block_size + sm[live] % block_size
        return out

    def relabel_tables(self, block_tables: np.ndarray, context_lens: np.ndarray,
                       block_size: int) -> np.ndarray:
        """Relabel the referenced entries; unreferenced ones become row 0
        (never read, since only ceil(len / block_size) entries are used)."""
        bt = np.asarray(block_tables, dtype=np.int64)
        out = np.zeros(bt.shape, dtype=np.int32)
        for s in range(bt.shape[0]):
            nb = -(-int(context_lens[s]) // block_size)
            if nb:
                out[s, :nb] = self.rows(bt[s, :nb])
        return out

    def view(self):
        """(k, v) slabs holding exactly the resident rows (C-contiguous)."""
        return self.k[:self.n], self.v[:self.n]


def _as_u16(a: np.ndarray) -> np.ndarray:
    """A uint8 pool seen as uint16 pairs (block copies move bytes, so the
    16-bit copy routine copies an FP8 block exactly)."""
    return a if a.dtype == np.uint16 else a.view(np.uint16)


class OracleSession:
    """Applies :class:`Step` objects in order: admit, copy, writes, decode.

    Over an FP8 cache (``scenario.kv_dtype == "fp8"``) admitted 16-bit blocks
    and new tokens enter the pool through the oracle's quantising cache
    write, and decode reads the codes with the scenario's scales."""

    def __init__(self, scenario, oracle=None):
        self.sc = scenario
        d = scenario.dims
        self.fp8 = getattr(scenario, "kv_dtype", "") == "fp8"
        self.orc = oracle if oracle is not None else load()
        self.pool = HostPool(d.num_blocks, d.num_kv_heads, d.block_size, d.head_dim,
                             "fp8" if self.fp8 else d.dtype)

    def write(self, key, value, slot_mapping) -> None:
        """The cache write of tokens (16-bit bit patterns) into their slots."""
        d = self.sc.dims
        sm = self.pool.relabel_slots(slot_mapping, d.block_size)
        k, v = self.pool.view()
        if self.fp8:
            self.orc.reshape_and_cache_fp8(k, v, key, value, sm, d.dtype, self.sc.k_scale, self.sc.v_scale)
        else:
            self.orc.reshape_and_cache(k, v, key, value, sm)

    def apply_cache_ops(self, step) -> None:
        d = self.sc.dims
        if step.admit_ids.size:
            if self.fp8:
                # every slot of each admitted block, token-major, through the cache write
                ids = np.asarray(step.admit_ids, np.int64)
                B = d.block_size
                self.pool.rows(ids)
                key = np.ascontiguousarray(step.admit_k.transpose(0, 2, 1, 3)).reshape(-1, d.num_kv_heads, d.head_dim)
                val = np.ascontiguousarray(step.admit_v.transpose(0, 2, 1, 3)).reshape(-1, d.num_kv_heads, d.head_dim)
                slots = (ids[:, None] * B + np.arange(B)[None, :]).reshape(-1)
                self.write(key, val, slots)
            else:
                self.pool.admit(step.admit_ids, step.admit_k, step.admit_v)
        if step.block_mapping.size:
            bm = step.block_mapping.reshape(-1, 2)
            rel = np.stack([self.pool.rows(bm[:, 0]), self.pool.rows(bm[:, 1])], axis=1)
            k, v = self.pool.view()
            self.orc.copy_blocks([_as_u16(k)], [_as_u16(v)], rel)
        for w in step.writes:
            self.write(w.key, w.value, w.slot_mapping)

    def decode(self, step, seqs: Optional[np.ndarray] = None) -> np.ndarray:
        """float64 ``[S, H, D]`` (or only the rows ``seqs``)."""
        d = self.sc.dims
        q, bt, cl = step.q, step.block_tables, step.context_lens
        if seqs is not None:
            seqs = np.asarray(seqs, dtype=np.int64)
            q, bt, cl = q[seqs], bt[seqs], cl[seqs]
        q_len, window = getattr(self.sc, "q_len", 1), getattr(self.sc, "window", 0)
        if q_len != 1 or window != 0:
            rel = self.relabel_attended(bt, cl, q_len, window)
            k, v = self.pool.view()
            q4 = q if q.ndim == 4 else q[:, None]
            out = self.orc.paged_decode_ext(q4, k, v, rel, cl, self.sc.scale, d.dtype, q_len, window,
                                            self.sc.k_scale, self.sc.v_scale)
            return out if q.ndim == 4 else out[:, 0]
        rel = self.pool.relabel_tables(bt, cl, d.block_size)
        k, v = self.pool.view()
        if self.fp8:
            return self.orc.paged_decode_fp8(q, k, v, rel, cl, self.sc.scale, self.sc.k_scale, self.sc.v_scale,
                                             d.dtype)
        return self.orc.paged_decode(q, k, v, rel, cl, self.sc.scale, d.dtype)

    def relabel_attended(self, block_tables, context_lens, q_len: int, window: int) -> np.ndarray:
        """Relabel only the entries of blocks some query attends to; entries
        before a sequence's window become -1 (the oracle never reads them)."""
        B = self.sc.dims.block_size
        bt = np.asarray(block_tables, dtype=np.int64)
        out = np.full(bt.shape, -1, dtype=np.int32)
        for s in range(bt.shape[0]):
            L = int(context_lens[s])
            nb = -(-L // B)
            lo = max(0, L - q_len - window + 1) if window > 0 else 0
            first = lo // B
            if nb > first:
                out[s, first:nb] = self.pool.rows(bt[s, first:nb])
        return out

    def run_step(self, step, seqs: Optional[np.ndarray] = None) -> np.ndarray:
        self.apply_cache_ops(step)
        return self.decode(step, seqs)
