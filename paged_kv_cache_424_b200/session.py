"""Device-side replay of workload steps through the C ABI.

A :class:`DeviceSession` owns a K and a V pool of ``num_blocks`` physical
blocks on the GPU (NaN-filled, so any stray read shows), takes the prefill
contents of admitted blocks from a :class:`~.workload.Step` (a host-to-device
copy: that data stands for the prefill output of newly admitted sequences),
then runs the step's ``pa_copy_blocks``, ``pa_reshape_and_cache`` and
``pa_decode`` calls through :mod:`.binding`.  torch provides the device
memory and the stream; the three operations run in the library's kernels.

Over an FP8 E4M3 cache (``scenario.kv_dtype == "fp8"``) the pools hold
uint8 codes (NaN code 0x7F where nothing was written), admitted blocks enter
through ``pa_reshape_and_cache_fp8`` like new tokens, and decode is
``pa_decode_fp8`` with the scenario's scales.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import binding as pa
from .workload import NAN_BITS, Scenario, Step

TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16}


def to_device(bits: np.ndarray, dtype: str, device) -> torch.Tensor:
    """uint16 bit patterns -> a CUDA tensor of the 16-bit float type."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device, non_blocking=False).view(TORCH_DTYPE[dtype])


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


FP8_NAN_CODE = 0x7F
ADMIT_CHUNK_BLOCKS = 4096  # admitted blocks per quantising write (bounds the staging copy)


class DeviceSession:
    def __init__(self, scenario: Scenario, device: str = "cuda"):
        self.sc = scenario
        self.device = torch.device(device)
        d = scenario.dims
        self.dtype = TORCH_DTYPE[d.dtype]
        self.fp8 = scenario.kv_dtype == "fp8"
        shape = (d.num_blocks, d.num_kv_heads, d.block_size, d.head_dim)
        if self.fp8:
            self.k_cache = torch.full(shape, FP8_NAN_CODE, dtype=torch.uint8, device=self.device)
            self.v_cache = torch.full(shape, FP8_NAN_CODE, dtype=torch.uint8, device=self.device)
        else:
            nan = np.array([NAN_BITS[d.dtype]], dtype=np.uint16).view(np.int16)[0]
            self.k_cache = torch.full(shape, int(nan), dtype=torch.int16, device=self.device).view(self.dtype)
            self.v_cache = torch.full(shape, int(nan), dtype=torch.int16, device=self.device).view(self.dtype)
        self._ws: Optional[torch.Tensor] = None

    # -- inputs ------------------------------------------------------------
    def admit(self, step: Step) -> None:
        if step.admit_ids.size == 0:
            return
        d = self.sc.dims
        if not self.fp8:
            ids = torch.from_numpy(step.admit_ids).to(self.device)
            self.k_cache.index_copy_(0, ids, to_device(step.admit_k, d.dtype, self.device))
            self.v_cache.index_copy_(0, ids, to_device(step.admit_v, d.dtype, self.device))
            return
        # FP8: every slot of each admitted block, token-major, through the quantising write
        B = d.block_size
        for c0 in range(0, step.admit_ids.size, ADMIT_CHUNK_BLOCKS):
            sl = slice(c0, c0 + ADMIT_CHUNK_BLOCKS)
            ids = torch.from_numpy(step.admit_ids[sl]).to(self.device)
            key = to_device(step.admit_k[sl], d.dtype, self.device).transpose(1, 2).reshape(-1, d.num_kv_heads,
                                                                                           d.head_dim)
            val = to_device(step.admit_v[sl], d.dtype, self.device).transpose(1, 2).reshape(-1, d.num_kv_heads,
                                                                                           d.head_dim)
            slots = (ids[:, None] * B + torch.arange(B, device=self.device)[None, :]).reshape(-1)
            pa.pa_reshape_and_cache_fp8(key.contiguous(), val.contiguous(), self.k_cache, self.v_cache, slots,
                                        self.sc.k_scale, self.sc.v_scale)

    def decode_inputs(self, step: Step) -> Dict[str, torch.Tensor]:
        d = self.sc.dims
        inp = {
            "q": to_device(step.q, d.dtype, self.device),
            "block_tables": torch.from_numpy(step.block_tables).to(self.device),
            "context_lens": torch.from_numpy(step.context_lens).to(self.device),
        }
        if self.sc.prefix_order:
            # the host schedule: sequences sharing a prefix next to each other
            order = pa.pa_prefix_order(step.block_tables, step.context_lens)
            inp["seq_order"] = torch.from_numpy(order).to(self.device)
        return inp

    def write_inputs(self, step: Step):
        d = self.sc.dims
        return [(to_device(w.key, d.dtype, self.device), to_device(w.value, d.dtype, self.device),
                 torch.from_numpy(w.slot_mapping).to(self.device)) for w in step.writes]

    def workspace(self, nbytes: int) -> Optional[torch.Tensor]:
        if nbytes == 0:
            return None
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self._ws

    # -- operations ----------------------------------------------------------
    def apply_cache_ops(self, step: Step) -> None:
        self.admit(step)
        if step.block_mapping.size:
            bm = torch.from_numpy(np.ascontiguousarray(step.block_mapping)).to(self.device)
            pa.pa_copy_blocks([self.k_cache], [self.v_cache], bm)
        for key, value, slots in self.write_inputs(step):
            self.write(key, value, slots)

    def write(self, key: torch.Tensor, value: torch.Tensor, slots: torch.Tensor) -> None:
        if self.fp8:
            pa.pa_reshape_and_cache_fp8(key, value, self.k_cache, self.v_cache, slots, self.sc.k_scale,
                                        self.sc.v_scale)
        else:
            pa.pa_reshape_and_cache(key, value, self.k_cache, self.v_cache, slots)

    def decode(self, step: Step, partition_tokens: Optional[int] = None,
               inputs: Optional[Dict[str, torch.Tensor]] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        d = self.sc.dims
        inp = inputs or self.decode_inputs(step)
        P = self.sc.partition_tokens if partition_tokens is None else partition_tokens
        maxlen = step.max_context_len
        if self.sc.ext:
            return self.decode_ext(inp, maxlen, P, out)
        dims = pa.dims_of(inp["q"], self.k_cache, inp["block_tables"])
        ws = self.workspace(pa.pa_decode_workspace_size(dims, maxlen, P))
        if out is None:
            out = torch.empty((d.num_seqs, d.num_heads, d.head_dim), dtype=self.dtype, device=self.device)
        if self.fp8:
            pa.pa_decode_fp8(out, inp["q"], self.k_cache, self.v_cache, inp["block_tables"], inp["context_lens"],
                             self.sc.scale, self.sc.k_scale, self.sc.v_scale, d.num_kv_heads, maxlen, P, ws)
        else:
            pa.pa_decode(out, inp["q"], self.k_cache, self.v_cache, inp["block_tables"], inp["context_lens"],
                         self.sc.scale, d.num_kv_heads, maxlen, P, ws)
        return out

    def ext_workspace_bytes(self, inp: Dict[str, torch.Tensor], maxlen: int, P: int) -> int:
        sc = self.sc
        q4 = inp["q"] if inp["q"].dim() == 4 else inp["q"][:, None]
        dims = pa.ext_dims(q4, self.k_cache, inp["block_tables"])
        opts = pa.pa_decode_opts(sc.q_len, sc.window, sc.k_scale, sc.v_scale)
        return pa.pa_decode_ext_workspace_size(dims, opts, maxlen, P)

    def decode_ext(self, inp: Dict[str, torch.Tensor], maxlen: int, P: int,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Multi-token / sliding-window decode of the scenario (q [S, q_len,
        H, D], or [S, H, D] for one token with a window)."""
        sc = self.sc
        q = inp["q"]
        q4 = q if q.dim() == 4 else q[:, None]
        ws = self.workspace(self.ext_workspace_bytes(inp, maxlen, P))
        if out is None:
            out = torch.empty_like(q)
        out4 = out if out.dim() == 4 else out[:, None]
        pa.pa_decode_ext(out4, q4, self.k_cache, self.v_cache, inp["block_tables"], inp["context_lens"], sc.scale,
                         sc.dims.num_kv_heads, maxlen, sc.q_len, sc.window, sc.k_scale, sc.v_scale, P, ws,
                         stream=stream, seq_order=inp.get("seq_order"))
        return out

    def run_step(self, step: Step, partition_tokens: Optional[int] = None) -> torch.Tensor:
        self.apply_cache_ops(step)
        return self.decode(step, partition_tokens)
