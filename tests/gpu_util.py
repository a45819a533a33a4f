"""Helpers for the GPU parity tests: run one workload step through the C ABI
and through the CPU oracle, then compare.

Tolerances (written here, used by every attention comparison):
  max-abs error <= 2e-3 (fp16) / 1e-2 (bf16) on the output, and
  relative L2 error ||out - ref|| / ||ref|| <= 2e-3 (fp16) / 1e-2 (bf16).
The absolute bounds are the stated target; the relative bound stops long
contexts (outputs ~3e-3) from passing with a near-zero result.  Cache writes
and copies must match bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle.harness import OracleSession

MAX_ABS = {"f16": 2e-3, "bf16": 1e-2}
REL_L2 = {"f16": 2e-3, "bf16": 1e-2}
NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


def require_gpu():
    import pytest
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def widen(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def compare(out_gpu: torch.Tensor, ref: np.ndarray, dtype: str, what: str) -> dict:
    got = widen(out_gpu)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    assert np.isfinite(got).all(), f"{what}: non-finite output (a NaN slot or block was read)"
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    nrm = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / nrm) if nrm > 0 else max_abs
    assert max_abs <= MAX_ABS[dtype], f"{what}: max abs err {max_abs:.3e} > {MAX_ABS[dtype]}"
    assert rel <= REL_L2[dtype], f"{what}: rel L2 err {rel:.3e} > {REL_L2[dtype]}"
    return {"max_abs": max_abs, "rel_l2": rel}


def compare_pools(dev, orc_ses: OracleSession, what: str) -> None:
    """Every block the oracle side touched matches bit for bit; every other
    block of the device pool still holds only NaN."""
    pool = orc_ses.pool
    ids = np.asarray(pool.ids, dtype=np.int64)
    rows = pool.row_of[ids]
    idx = torch.from_numpy(ids).to(dev.k_cache.device)
    fp8 = pool.dtype == "fp8"
    for name, cache, host in (("K", dev.k_cache, pool.k), ("V", dev.v_cache, pool.v)):
        if fp8:  # uint8 E4M3 codes; 0x7F (NaN) where nothing was written
            got = cache.index_select(0, idx).cpu().numpy()
            raw, nan = cache, 0x7F
        else:
            got = cache.view(torch.int16).index_select(0, idx).cpu().numpy().view(np.uint16)
            raw = cache.view(torch.int16)
            nan = int(np.array([NAN_BITS[orc_ses.sc.dims.dtype]], np.uint16).view(np.int16)[0])
        want = host[rows]
        bad = np.nonzero((got != want).reshape(len(ids), -1).any(axis=1))[0]
        assert bad.size == 0, f"{what}: {name} blocks differ at physical ids {ids[bad[:8]].tolist()}"
        mask = torch.ones(cache.shape[0], dtype=torch.bool, device=cache.device)
        mask[idx] = False
        untouched = raw[mask]
        assert bool((untouched == nan).all()), f"{what}: {name} bytes outside the written blocks changed"


def run_and_compare(scenario, partition_tokens=None, seqs=None, check_pools=True, steps=None):
    """Replay every step on both sides; compare caches and outputs."""
    from paged_kv_cache_424_b200.session import DeviceSession
    dev = DeviceSession(scenario)
    orc = OracleSession(scenario)
    stats = []
    for i, st in enumerate(scenario.steps if steps is None else steps):
        dev.apply_cache_ops(st)
        orc.apply_cache_ops(st)
        if check_pools:
            compare_pools(dev, orc, f"{scenario.name} step {i}")
        out = dev.decode(st, partition_tokens)
        torch.cuda.synchronize()
        sel = None if seqs is None else np.asarray(seqs)
        ref = orc.decode(st, sel)
        got = out if sel is None else out[torch.from_numpy(sel).to(out.device)]
        stats.append(compare(got, ref, scenario.dims.dtype, f"{scenario.name} step {i}"))
    return dev, orc, stats
