"""Seeded synthetic decode workloads shaped like the five benchmark scenarios.

This module only draws random numbers and does block bookkeeping (through
:mod:`.block_manager`); it contains none of the attention arithmetic.  Both
the CUDA path and the CPU oracle consume what it produces.

A :class:`Scenario` is a list of :class:`Step` objects.  Each step is applied
in this order on either side:

1. ``admit``: set the contents of some physical blocks (the prefill output of
   newly admitted sequences; untouched slots stay NaN),
2. ``block_mapping``: copy-on-write pairs for ``copy_blocks``,
3. ``writes``: ``reshape_and_cache`` calls (key, value, slot_mapping), in order,
4. decode attention over ``q``, ``block_tables``, ``context_lens``.

``context_lens`` count the token written in this step: the decode query
attends to its own key, at logical position ``context_len - 1``.

Values are bit patterns (uint16) of fp16 or bf16, rounded to nearest-even
from float32 draws.  Every slot that is not written, every block that is not
referenced and the padding block that fills unused table entries hold NaN,
so a read of anything outside a sequence's context shows up as NaN.

Recipes (one per scenario; the lognormal sigma and pool sizes that the
scenario text leaves open are fixed here):

1. ``tiny``: 4 sequences of lengths {1, 17, 33, 100}, 8 heads = 8 KV heads,
   head_dim 64, fp16, pool of 64 blocks handed out in seeded-permutation order.
2. ``mha7b``: 64 sequences, lengths uniform on [128, 2048], 32 = 32 heads,
   head_dim 128, fp16, pool of 16384 blocks.
3. ``gqa8b``: 256 sequences, 32 query heads over 8 KV heads, head_dim 128,
   bf16, lengths round(1024 * exp(Z)), Z ~ N(0, 1), clamped to [1, 4096],
   pool of 131072 blocks; every later step retires round(0.1 * 256) = 26
   sequences, admits 26 new ones of length uniform on [32, 512] and grows the
   rest by one token.
4. ``long70b``: 8 sequences of 32768 tokens, 64 query heads over 8 KV heads,
   head_dim 128, bf16, pool of 32768 blocks, 512-token KV partitions.
5. ``cow``: 16 prompts x 8 samples, 32 / 8 heads, head_dim 128, bf16, pool
   of 8192 blocks; each prompt's 1000-token prefix is stored once and shared
   by its 8 samples; each sample then appends a tail of uniform [0, 256]
   tokens plus the decode token; the first write into the shared partial
   block makes a private copy while the block is still shared (7 copies per
   prompt), or for every sample with ``cow_every_sample``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import List, Optional, Sequence, Tuple

import numpy as np

from .block_manager import BlockManager, SeqBlocks, block_tables as _tables

NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}
BLOCK_SIZE = 16


# --------------------------------------------------------------------------
# value generation
# --------------------------------------------------------------------------
def to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to fp16 / bf16 (nearest-even) and return the bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        b = x.view(np.uint32).astype(np.uint64)
        return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)
    raise ValueError(f"unknown dtype {dtype}")


def uniform_bits(rng: np.random.Generator, shape, dtype: str, lo: float = -1.0,
                 hi: float = 1.0) -> np.ndarray:
    x = rng.random(size=shape, dtype=np.float32)
    x *= np.float32(hi - lo)
    x += np.float32(lo)
    return to_bits(x, dtype)


def nan_bits(shape, dtype: str) -> np.ndarray:
    return np.full(shape, NAN_BITS[dtype], dtype=np.uint16)


# --------------------------------------------------------------------------
# data classes
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Dims:
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    max_blocks_per_seq: int
    num_blocks: int
    dtype: str

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads


@dataclass
class Write:
    key: np.ndarray           # uint16 [T, Hk, D]
    value: np.ndarray         # uint16 [T, Hk, D]
    slot_mapping: np.ndarray  # int64 [T]


@dataclass
class Step:
    admit_ids: np.ndarray                 # int64 [n] physical block ids
    admit_k: np.ndarray                   # uint16 [n, Hk, B, D]
    admit_v: np.ndarray                   # uint16 [n, Hk, B, D]
    block_mapping: np.ndarray             # int64 [P, 2]
    writes: List[Write]
    q: np.ndarray                         # uint16 [S, H, D]
    block_tables: np.ndarray              # int32 [S, MB]
    context_lens: np.ndarray              # int32 [S]

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.context_lens.size else 0


@dataclass
class Scenario:
    name: str
    dims: Dims
    scale: float
    pad_block: int
    steps: List[Step]
    partition_tokens: int = 0
    note: str = ""
    shared_blocks: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))
    # KV cache element type: "" = the 16-bit dtype of the tokens, "fp8" =
    # E4M3 codes with per-tensor scales (K = code * k_scale, V likewise).
    # The step data stays 16-bit: admitted blocks and new tokens reach an
    # FP8 cache through the quantising cache write on either side.
    kv_dtype: str = ""
    k_scale: float = 1.0
    v_scale: float = 1.0
    # Multi-token / sliding-window decode: each step writes q_len new tokens
    # per sequence and queries all of them (q is [S, q_len, H, D] when
    # q_len > 1); window > 0 limits every query to its `window` most recent
    # positions.
    q_len: int = 1
    window: int = 0
    # decode in the shared-prefix-aware order (pa_prefix_order / seq_order)
    prefix_order: bool = False

    @property
    def ext(self) -> bool:
        return self.q_len != 1 or self.window != 0 or self.prefix_order

    @property
    def kv_elem_bytes(self) -> int:
        return 1 if self.kv_dtype == "fp8" else 2


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------
class _Builder:
    """Allocates blocks for sequences and collects admitted contents."""

    def __init__(self, rng: np.random.Generator, dims: Dims, v_lo: float = -1.0):
        self.rng = rng
        self.dims = dims
        self.v_lo = v_lo
        self.pad_block = dims.num_blocks - 1
        self.bm = BlockManager(dims.num_blocks, dims.block_size, rng=rng, reserved=[self.pad_block])
        self._ids: List[np.ndarray] = []
        self._k: List[np.ndarray] = []
        self._v: List[np.ndarray] = []

    def fill(self, blocks: Sequence[int], n_tokens: int) -> None:
        """Admit ``blocks`` holding ``n_tokens`` random tokens (rest NaN)."""
        d = self.dims
        nb = len(blocks)
        if nb == 0:
            return
        shape = (nb, d.num_kv_heads, d.block_size, d.head_dim)
        k = uniform_bits(self.rng, shape, d.dtype)
        v = uniform_bits(self.rng, shape, d.dtype, lo=self.v_lo)
        full, rem = divmod(n_tokens, d.block_size)
        nanv = NAN_BITS[d.dtype]
        if full < nb:
            k[full, :, rem:, :] = nanv
            v[full, :, rem:, :] = nanv
            k[full + 1:] = nanv
            v[full + 1:] = nanv
        self._ids.append(np.asarray(blocks, dtype=np.int64))
        self._k.append(k)
        self._v.append(v)

    def admit_pad(self) -> None:
        d = self.dims
        shape = (1, d.num_kv_heads, d.block_size, d.head_dim)
        self._ids.append(np.asarray([self.pad_block], dtype=np.int64))
        self._k.append(nan_bits(shape, d.dtype))
        self._v.append(nan_bits(shape, d.dtype))

    def take_admitted(self) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        d = self.dims
        if not self._ids:
            e = np.zeros((0, d.num_kv_heads, d.block_size, d.head_dim), np.uint16)
            return np.zeros(0, np.int64), e, e.copy()
        out = (np.concatenate(self._ids), np.concatenate(self._k), np.concatenate(self._v))
        self._ids, self._k, self._v = [], [], []
        return out

    def new_sequence(self, length: int) -> Tuple[SeqBlocks, int]:
        """A sequence whose first ``length - 1`` tokens are prefilled; returns
        it and the slot of its last token, which the step's write fills."""
        seq, slots = self.new_sequence_multi(length, 1)
        return seq, slots[0]

    def new_sequence_multi(self, length: int, new: int) -> Tuple[SeqBlocks, List[int]]:
        """A sequence whose first ``length - new`` tokens are prefilled (at
        least none); returns it and the slots of its last ``new`` tokens,
        which the step's write fills."""
        seq = self.bm.new_sequence()
        pre = max(0, length - new)
        for _ in range(pre):
            self.bm.append_slot(seq)
        self.fill(seq.blocks, pre)
        before = len(seq.blocks)
        slots = [self.bm.append_slot(seq) for _ in range(length - pre)]
        if len(seq.blocks) > before:
            # the new tokens opened blocks: admit them as all-NaN
            self.fill(seq.blocks[before:], 0)
        return seq, slots

    def new_tokens(self, n: int) -> Tuple[np.ndarray, np.ndarray]:
        d = self.dims
        shape = (n, d.num_kv_heads, d.head_dim)
        return uniform_bits(self.rng, shape, d.dtype), uniform_bits(self.rng, shape, d.dtype, lo=self.v_lo)

    def queries(self, q_len: int = 1) -> np.ndarray:
        d = self.dims
        shape = (d.num_seqs, d.num_heads, d.head_dim) if q_len == 1 else (d.num_seqs, q_len, d.num_heads, d.head_dim)
        return uniform_bits(self.rng, shape, d.dtype)

    def step(self, seqs: List[SeqBlocks], writes: List[Write], q_len: int = 1) -> Step:
        d = self.dims
        ids, k, v = self.take_admitted()
        return Step(admit_ids=ids, admit_k=k, admit_v=v,
                    block_mapping=self.bm.take_copy_pairs(), writes=writes,
                    q=self.queries(q_len),
                    block_tables=_tables(seqs, d.max_blocks_per_seq, self.pad_block),
                    context_lens=np.asarray([s.length for s in seqs], dtype=np.int32))


def _scale(head_dim: int) -> float:
    return float(np.float32(1.0 / math.sqrt(head_dim)))


def _fresh_batch(name: str, dims: Dims, lengths: Sequence[int], rng: np.random.Generator,
                 partition_tokens: int = 0, v_lo: float = -1.0, note: str = "", q_len: int = 1,
                 window: int = 0) -> Scenario:
    """One decode step over new sequences of the given lengths (the last
    q_len tokens of each are the step's new tokens)."""
    b = _Builder(rng, dims, v_lo=v_lo)
    b.admit_pad()
    seqs, slots = [], []
    for L in lengths:
        s, sl = b.new_sequence_multi(int(L), q_len)
        seqs.append(s)
        slots.extend(sl)
    key, value = b.new_tokens(len(slots))
    w = Write(key, value, np.asarray(slots, dtype=np.int64))
    st = b.step(seqs, [w], q_len)
    return Scenario(name, dims, _scale(dims.head_dim), b.pad_block, [st], partition_tokens, note, q_len=q_len,
                    window=window)


# --------------------------------------------------------------------------
# the five scenarios
# --------------------------------------------------------------------------
def tiny(seed: int = 0, v_lo: float = -1.0) -> Scenario:
    dims = Dims(4, 8, 8, 64, BLOCK_SIZE, 7, 64, "f16")
    rng = np.random.default_rng(seed)
    return _fresh_batch("tiny", dims, [1, 17, 33, 100], rng, v_lo=v_lo,
                        note="4 seqs {1,17,33,100}, H=Hk=8, D=64, fp16, pool 64")


def mha7b(seed: int = 1, num_seqs: int = 64, min_len: int = 128, max_len: int = 2048,
          num_blocks: int = 16384, v_lo: float = -1.0) -> Scenario:
    rng = np.random.default_rng(seed)
    lengths = rng.integers(min_len, max_len + 1, size=num_seqs)
    mb = -(-max_len // BLOCK_SIZE)
    dims = Dims(num_seqs, 32, 32, 128, BLOCK_SIZE, mb, num_blocks, "f16")
    return _fresh_batch("mha7b", dims, lengths, rng, v_lo=v_lo,
                        note=f"{num_seqs} seqs, L~U[{min_len},{max_len}], H=Hk=32, D=128, fp16, "
                             f"pool {num_blocks}")


def lognormal_lengths(rng: np.random.Generator, n: int, median: int = 1024, sigma: float = 1.0,
                      cap: int = 4096) -> np.ndarray:
    z = rng.standard_normal(n)
    return np.clip(np.rint(median * np.exp(sigma * z)), 1, cap).astype(np.int64)


def gqa8b(seed: int = 2, num_seqs: int = 256, num_steps: int = 1, churn: float = 0.1,
          median: int = 1024, cap: int = 4096, new_min: int = 32, new_max: int = 512,
          num_blocks: int = 131072, v_lo: float = -1.0) -> Scenario:
    """Continuous batching: step 0 admits ``num_seqs`` sequences; each later
    step retires round(churn * S) of them (chosen by the seeded RNG), admits
    as many new ones and appends one token to every survivor."""
    rng = np.random.default_rng(seed)
    mb = -(-(max(cap, new_max) + num_steps) // BLOCK_SIZE)  # admitted sequences grow too
    dims = Dims(num_seqs, 32, 8, 128, BLOCK_SIZE, mb, num_blocks, "bf16")
    b = _Builder(rng, dims, v_lo=v_lo)
    b.admit_pad()
    seqs, slots = [], []
    for L in lognormal_lengths(rng, num_seqs, median, 1.0, cap):
        s, slot = b.new_sequence(int(L))
        seqs.append(s)
        slots.append(slot)
    key, value = b.new_tokens(num_seqs)
    steps = [b.step(seqs, [Write(key, value, np.asarray(slots, np.int64))])]
    n_churn = int(round(churn * num_seqs))
    for _ in range(1, num_steps):
        done = set(int(i) for i in rng.choice(num_seqs, size=n_churn, replace=False))
        slots = []
        for i in range(num_seqs):
            if i in done:
                b.bm.free_sequence(seqs[i])
                s, slot = b.new_sequence(int(rng.integers(new_min, new_max + 1)))
                seqs[i] = s
            else:
                before = len(seqs[i].blocks)
                slot = b.bm.append_slot(seqs[i])
                if len(seqs[i].blocks) > before:
                    b.fill(seqs[i].blocks[-1:], 0)
            slots.append(slot)
        key, value = b.new_tokens(num_seqs)
        steps.append(b.step(seqs, [Write(key, value, np.asarray(slots, np.int64))]))
    return Scenario("gqa8b", dims, _scale(128), b.pad_block, steps,
                    note=f"{num_seqs} seqs, lognormal(median {median}, sigma 1, cap {cap}), "
                         f"H=32/Hk=8, D=128, bf16, pool {num_blocks}, {num_steps} steps, "
                         f"churn {n_churn}/step with new L~U[{new_min},{new_max}]")


def long70b(seed: int = 3, num_seqs: int = 8, context_len: int = 32768, num_blocks: int = 32768,
            partition_tokens: int = 512, v_lo: float = -1.0) -> Scenario:
    rng = np.random.default_rng(seed)
    mb = -(-context_len // BLOCK_SIZE)
    dims = Dims(num_seqs, 64, 8, 128, BLOCK_SIZE, mb, num_blocks, "bf16")
    return _fresh_batch("long70b", dims, [context_len] * num_seqs, rng, partition_tokens, v_lo=v_lo,
                        note=f"{num_seqs} seqs x {context_len} tokens, H=64/Hk=8, D=128, bf16, "
                             f"pool {num_blocks}, partitions of {partition_tokens}")


def cow(seed: int = 4, num_prompts: int = 16, samples: int = 8, prefix: int = 1000,
        max_tail: int = 256, num_blocks: int = 8192, cow_every_sample: bool = False,
        v_lo: float = -1.0, shuffle: bool = False, name: str = "cow") -> Scenario:
    """Parallel sampling: prefixes shared by ``samples`` sequences each.
    With ``shuffle`` the batch lists the sequences in a seeded random order
    (as a scheduler admitting requests over time would), so sharers of one
    prefix are scattered through the batch."""
    rng = np.random.default_rng(seed)
    S = num_prompts * samples
    mb = -(-(prefix + max_tail + 1) // BLOCK_SIZE)
    dims = Dims(S, 32, 8, 128, BLOCK_SIZE, mb, num_blocks, "bf16")
    b = _Builder(rng, dims, v_lo=v_lo)
    b.admit_pad()
    seqs: List[SeqBlocks] = []
    shared = []
    for _ in range(num_prompts):
        parent = b.bm.new_sequence()
        for _ in range(prefix):
            b.bm.append_slot(parent)
        b.fill(parent.blocks, prefix)
        shared.extend(parent.blocks)
        kids = [b.bm.fork(parent) for _ in range(samples)]
        b.bm.free_sequence(parent)
        seqs.extend(kids)
    if shuffle:
        seqs = [seqs[i] for i in rng.permutation(S)]
    tails = rng.integers(0, max_tail + 1, size=S)
    tail_slots, dec_slots = [], []
    for s, t in zip(seqs, tails):
        if cow_every_sample and prefix % BLOCK_SIZE:
            b.bm.copy_last_block(s)
        before = len(s.blocks)
        for _ in range(int(t)):
            tail_slots.append(b.bm.append_slot(s))
        dec_slots.append(b.bm.append_slot(s))
        if len(s.blocks) > before:
            b.fill(s.blocks[before:], 0)
    k1, v1 = b.new_tokens(len(tail_slots))
    k2, v2 = b.new_tokens(S)
    writes = [Write(k1, v1, np.asarray(tail_slots, np.int64)),
              Write(k2, v2, np.asarray(dec_slots, np.int64))]
    st = b.step(seqs, writes)
    return Scenario(name, dims, _scale(128), b.pad_block, [st],
                    note=f"{num_prompts} prompts x {samples} samples, prefix {prefix}, tails "
                         f"U[0,{max_tail}], H=32/Hk=8, D=128, bf16, pool {num_blocks}, "
                         f"{'copy per sample' if cow_every_sample else 'copy while shared'}"
                         f"{', shuffled batch order' if shuffle else ''}",
                    shared_blocks=np.asarray(shared, np.int64))


def prefix8b(seed: int = 7, num_prompts: int = 64, samples: int = 8, prefix: int = 2000, max_tail: int = 64,
             num_blocks: int = 16384, shuffle: bool = True, v_lo: float = -1.0) -> Scenario:
    """Shared prefixes larger than L2: 64 prompts of 2000 tokens (500 MiB of
    K/V on the 8B shape), each shared by 8 sequences listed in a shuffled
    batch order; decode visits them in the order pa_prefix_order gives."""
    sc = cow(seed, num_prompts, samples, prefix, max_tail, num_blocks, v_lo=v_lo, shuffle=shuffle, name="prefix8b")
    return replace(sc, prefix_order=True, note=sc.note + ", decoded in shared-prefix order")


def spec8b(seed: int = 5, num_seqs: int = 256, q_len: int = 4, median: int = 1024, cap: int = 4096,
           num_blocks: int = 131072, window: int = 0, v_lo: float = -1.0) -> Scenario:
    """Speculative verification on the 8B shape: every sequence of a
    lognormal length mix (as gqa8b) writes q_len new tokens (the token being
    decoded and q_len - 1 draft tokens) and queries all of them, each
    causally; group 4 x 4 tokens fill the 16 query rows of a KV head."""
    rng = np.random.default_rng(seed)
    lengths = np.maximum(lognormal_lengths(rng, num_seqs, median, 1.0, cap), q_len)
    mb = -(-cap // BLOCK_SIZE)
    dims = Dims(num_seqs, 32, 8, 128, BLOCK_SIZE, mb, num_blocks, "bf16")
    return _fresh_batch("spec8b", dims, lengths, rng, v_lo=v_lo, q_len=q_len, window=window,
                        note=f"{num_seqs} seqs, lognormal(median {median}, sigma 1, cap {cap}), {q_len} query "
                             f"tokens each, H=32/Hk=8, D=128, bf16, pool {num_blocks}")


def window70b(seed: int = 6, num_seqs: int = 8, context_len: int = 32768, window: int = 4096,
              num_blocks: int = 32768, q_len: int = 1, partition_tokens: int = 0, v_lo: float = -1.0) -> Scenario:
    """The 70B long-context shape with a sliding window: each query attends
    to its `window` most recent positions, so a step reads window tokens per
    sequence whatever the context length."""
    rng = np.random.default_rng(seed)
    mb = -(-context_len // BLOCK_SIZE)
    dims = Dims(num_seqs, 64, 8, 128, BLOCK_SIZE, mb, num_blocks, "bf16")
    return _fresh_batch("window70b", dims, [context_len] * num_seqs, rng, partition_tokens, v_lo=v_lo,
                        q_len=q_len, window=window,
                        note=f"{num_seqs} seqs x {context_len} tokens, sliding window {window}, H=64/Hk=8, "
                             f"D=128, bf16, pool {num_blocks}")


# Per-tensor FP8 scales for inputs in [-1, 1]: |x| / scale reaches 81 (K)
# and 141 (V), inside E4M3's range (448).  Not powers of two, so the
# division before rounding is inexact and both sides must round it alike.
FP8_K_SCALE = 0.0123
FP8_V_SCALE = 0.0071


def with_fp8_cache(sc: Scenario, k_scale: float = FP8_K_SCALE, v_scale: float = FP8_V_SCALE) -> Scenario:
    """The same scenario over an FP8 E4M3 cache."""
    return replace(sc, name=f"{sc.name}-fp8", kv_dtype="fp8", k_scale=float(np.float32(k_scale)),
                   v_scale=float(np.float32(v_scale)),
                   note=f"{sc.note}; FP8 E4M3 cache, k_scale {k_scale}, v_scale {v_scale}")


SCENARIOS = {"tiny": tiny, "mha7b": mha7b, "gqa8b": gqa8b, "long70b": long70b, "cow": cow, "spec8b": spec8b,
             "window70b": window70b, "prefix8b": prefix8b}
CONFIG_ORDER = ["tiny", "mha7b", "gqa8b", "long70b", "cow"]


def attended_tokens(step: Step, q_len: int = 1, window: int = 0) -> np.ndarray:
    """Per sequence, the positions some query attends to: all of them, or
    with a window those from query 0's first (len - q_len - window + 1)."""
    L = step.context_lens.astype(np.int64)
    if window <= 0:
        return L
    return L - np.maximum(0, L - q_len - window + 1)


def kv_bytes(step: Step, dims: Dims, unique: bool = False, elem_bytes: int = 2, q_len: int = 1,
             window: int = 0) -> int:
    """KV bytes a decode step must read: sum of attended tokens (the context
    lengths, or the window spans) x 2 (K and V) x KV heads x head_dim x
    element size (2 bytes; 1 for an FP8 cache).  With ``unique``, blocks
    shared by several sequences count once (whole blocks, partial tails as
    their token count)."""
    el = elem_bytes
    per_tok = 2 * dims.num_kv_heads * dims.head_dim * el
    if not unique:
        return int(attended_tokens(step, q_len, window).sum()) * per_tok
    seen = {}
    for s in range(dims.num_seqs):
        L = int(step.context_lens[s])
        nb = -(-L // dims.block_size)
        for i in range(nb):
            blk = int(step.block_tables[s, i])
            used = min(dims.block_size, L - i * dims.block_size)
            seen[blk] = max(seen.get(blk, 0), used)
    return sum(seen.values()) * per_tok


def qo_bytes(dims: Dims, q_len: int = 1) -> int:
    """Query read + output write: 2 x S x q_len x H x D x 2 bytes."""
    return 2 * dims.num_seqs * q_len * dims.num_heads * dims.head_dim * 2
