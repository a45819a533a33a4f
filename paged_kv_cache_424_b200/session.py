"""Device-side replay of workload steps through the C ABI.

A :class:`DeviceSession` owns a K and a V pool of ``num_blocks`` physical
blocks on the GPU (NaN-filled, so any stray read shows), takes the prefill
contents of admitted blocks from a :class:`~.workload.Step` (a host-to-device
copy: that data stands for the prefill output of newly admitted sequences),
then runs the step's ``pa_copy_blocks``, ``pa_reshape_and_cache`` and
``pa_decode`` calls through :mod:`.binding`.  torch provides the device
memory and the stream; the three operations run in the library's kernels.
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


class DeviceSession:
    def __init__(self, scenario: Scenario, device: str = "cuda"):
        self.sc = scenario
        self.device = torch.device(device)
        d = scenario.dims
        self.dtype = TORCH_DTYPE[d.dtype]
        shape = (d.num_blocks, d.num_kv_heads, d.block_size, d.head_dim)
        nan = np.array([NAN_BITS[d.dtype]], dtype=np.uint16).view(np.int16)[0]
        self.k_cache = torch.full(shape, int(nan), dtype=torch.int16, device=self.device).view(self.dtype)
        self.v_cache = torch.full(shape, int(nan), dtype=torch.int16, device=self.device).view(self.dtype)
        self._ws: Optional[torch.Tensor] = None

    # -- inputs ------------------------------------------------------------
    def admit(self, step: Step) -> None:
        if step.admit_ids.size == 0:
            return
        ids = torch.from_numpy(step.admit_ids).to(self.device)
        self.k_cache.index_copy_(0, ids, to_device(step.admit_k, self.sc.dims.dtype, self.device))
        self.v_cache.index_copy_(0, ids, to_device(step.admit_v, self.sc.dims.dtype, self.device))

    def decode_inputs(self, step: Step) -> Dict[str, torch.Tensor]:
        d = self.sc.dims
        return {
            "q": to_device(step.q, d.dtype, self.device),
            "block_tables": torch.from_numpy(step.block_tables).to(self.device),
            "context_lens": torch.from_numpy(step.context_lens).to(self.device),
        }

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
            pa.pa_reshape_and_cache(key, value, self.k_cache, self.v_cache, slots)

    def decode(self, step: Step, partition_tokens: Optional[int] = None,
               inputs: Optional[Dict[str, torch.Tensor]] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        d = self.sc.dims
        inp = inputs or self.decode_inputs(step)
        P = self.sc.partition_tokens if partition_tokens is None else partition_tokens
        maxlen = step.max_context_len
        dims = pa.dims_of(inp["q"], self.k_cache, inp["block_tables"])
        ws = self.workspace(pa.pa_decode_workspace_size(dims, maxlen, P))
        if out is None:
            out = torch.empty((d.num_seqs, d.num_heads, d.head_dim), dtype=self.dtype, device=self.device)
        pa.pa_decode(out, inp["q"], self.k_cache, self.v_cache, inp["block_tables"], inp["context_lens"],
                     self.sc.scale, d.num_kv_heads, maxlen, P, ws)
        return out

    def run_step(self, step: Step, partition_tokens: Optional[int] = None) -> torch.Tensor:
        self.apply_cache_ops(step)
        return self.decode(step, partition_tokens)
