#!/usr/bin/env python
"""Benchmark: paged decode attention on B200, one JSON line on stdout.

A step is one pass of the whole hot path over one batch: the cache write of
every sequence's new token (pa_reshape_and_cache), copy-on-write copies when
the workload has them (pa_copy_blocks), and decode attention of every
sequence over its paged KV cache (pa_decode, with the split-KV merge when a
context spans several partitions).

Default workload: the Llama-3-8B-shaped GQA batch under continuous batching
(256 sequences, lognormal lengths with median 1024 capped at 4096, 32 query
heads over 8 KV heads, head_dim 128, bf16, 131072-block pool).  Every step
retires 26 sequences and admits 26 new ones of 32-512 tokens; the rest grow
by one token.  The scenario is built with two set-up steps followed by a
cycle of --cycle churned steps (8 by default), all of whose inputs are on
the device before timing; the timed loop walks through the cycle, so
consecutive timed steps decode different batch mixes.  The same JSON line
carries `config.also`: the decode time and roofline fraction of the
long-context 70B shape at its stated 512-token partitions, the
copy-on-write batch and the 7B MHA batch, measured in the same run.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--kv 16|fp8]
  python bench.py --impl reference ...      # the CPU oracle, timed the same way

Other workloads: mha7b, long70b, cow (the pages' other shapes), spec8b (4
query tokens per sequence, pa_decode_ext), window70b (4096-token sliding
window), prefix8b (shared prefixes in a shuffled batch, decoded in the
pa_prefix_order schedule; the batch-order time is reported beside), swap
(pa_swap_blocks device <-> pinned host).  --kv fp8 runs a workload over an
FP8 E4M3 cache (pa_reshape_and_cache_fp8 + pa_decode_fp8).

With N > 1 (torchrun, one process per GPU) every rank runs its own batch of
the same shape (sequences are independent; no collective on the data path),
so per-GPU work is fixed: weak scaling.  Timing is CUDA events on the
launching stream, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention seqs/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
FALLBACK_HBM_GBS = 6650.0
TARGET_GBS = 8000.0  # the HBM peak the 70 % target is stated against
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
WORKLOADS = ["tiny", "mha7b", "gqa8b", "long70b", "cow", "spec8b", "window70b", "prefix8b", "swap"]
DEFAULT_ALSO = "long70b,cow,mha7b,gqa8b:fp8,long70b:fp8"


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gqa8b", choices=WORKLOADS,
                    help="decode scenario (spec8b: 4 query tokens per sequence; window70b: 4096-token sliding "
                         "window; prefix8b: shuffled batch of shared 2000-token prefixes, decoded in "
                         "shared-prefix order), or 'swap' for pa_swap_blocks device <-> pinned host throughput")
    ap.add_argument("--cycle", type=int, default=8,
                    help="gqa8b: churned steps in the timed cycle (after two set-up steps)")
    ap.add_argument("--also", default=None,
                    help=f"comma-separated workloads whose decode is measured after the main one and reported "
                         f"in config.also (default for gqa8b: {DEFAULT_ALSO}; 'none' for none; a name may end "
                         f"in ':fp8' for an FP8 cache)")
    ap.add_argument("--num-seqs", type=int, default=None, help="override the batch size (profiling cases)")
    ap.add_argument("--num-blocks", type=int, default=None, help="override the pool size (profiling cases)")
    ap.add_argument("--partition", type=int, default=None, help="partition tokens (default: the workload's)")
    ap.add_argument("--kv", choices=["16", "fp8"], default="16",
                    help="KV cache element type: the 16-bit dtype of the workload, or FP8 E4M3 with scales")
    ap.add_argument("--no-prefix-order", action="store_true",
                    help="prefix8b: decode in plain batch order (no seq_order), for profiling the difference")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline sample budget")
    return ap.parse_args(argv)


def make_scenario(name: str, seed: int, num_seqs=None, num_blocks=None, kv: str = "16", cycle: int = 8):
    from paged_kv_cache_424_b200 import workload as W
    sc = _base_scenario(name, seed, num_seqs, num_blocks, cycle)
    return W.with_fp8_cache(sc) if kv == "fp8" else sc


def _base_scenario(name: str, seed: int, num_seqs=None, num_blocks=None, cycle: int = 8):
    from paged_kv_cache_424_b200 import workload as W
    kw = {}
    if num_seqs is not None:
        kw["num_seqs"] = num_seqs
    if num_blocks is not None:
        kw["num_blocks"] = num_blocks
    if name == "tiny":
        return W.tiny(seed)
    if name == "gqa8b":
        return W.gqa8b(seed, num_steps=2 + max(1, cycle), **kw)
    if name in ("cow", "prefix8b"):
        if num_seqs is not None:
            kw = {"num_prompts": max(1, num_seqs // 8), **({"num_blocks": num_blocks} if num_blocks else {})}
        return getattr(W, name)(seed, **kw)
    return getattr(W, name)(seed, **kw)


def scenario_cycle(sc):
    """(set-up steps, timed cycle).  A continuous-batching scenario with
    churned steps keeps its first two steps as set-up and times the rest in
    turn; a one-step scenario times its one step over and over."""
    if len(sc.steps) > 2:
        return sc.steps[:2], sc.steps[2:]
    return sc.steps[:-1], sc.steps[-1:]


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Sources that only the tensor-core kernel is built from: the CUDA-core
# kernel's traffic does not depend on them.
TC_ONLY_SOURCES = ("pa_decode_tc.cu", "pa_tc.cuh")


def kernel_source_hash(tensor_core: bool = True, root: str = ROOT) -> str:
    """Hash of the sources a decode kernel is built and launched from: all of
    csrc/ for the tensor-core kernel, csrc/ without the tensor-core kernel's
    own files for the CUDA-core kernel."""
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(root, "paged_kv_cache_424_b200", "csrc", "*"))):
        if not tensor_core and os.path.basename(p) in TC_ONLY_SOURCES:
            continue
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, units: float):
    """DRAM bytes per decode launch from the committed ncu summary, scaled to
    this launch's units, or None if absent or taken on other kernel sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except Exception:
        return None
    ent = rec.get("workloads", {}).get(workload)
    if not ent:
        return None
    if ent.get("kernel_src_sha") != kernel_source_hash("decode_tc_kernel" in ent.get("kernel", "")):
        return None
    return float(ent["dram_bytes_per_unit"]) * units


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that instead of clocks
            self.nv = None
            self.err = str(e)

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._sample()  # at least one sample inside the region, however short
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": f"NVML unavailable: {self.err}"}
        names = [n for b, n in self.REASONS.items() if self.reasons & b]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def also_list(args):
    spec = args.also if args.also is not None else (DEFAULT_ALSO if args.workload == "gqa8b" else "none")
    if spec.strip().lower() in ("", "none"):
        return []
    out = []
    for item in spec.split(","):
        name, _, kv = item.strip().partition(":")
        if name not in WORKLOADS or name == "swap":
            raise SystemExit(f"--also: unknown workload {name!r}")
        out.append((name, "fp8" if kv == "fp8" else "16"))
    return out


# ---------------------------------------------------------------------------
# our arm: one workload on the device
# ---------------------------------------------------------------------------
class DeviceWorkload:
    """A scenario resident on the device: every cache operation of every
    step applied (admissions, copies, writes), and for each step of the timed
    cycle its decode inputs, new tokens, slots and copy pairs on the device,
    so that a timed step enqueues only the library's kernels."""

    def __init__(self, sc, device, partition, pa, W):
        import torch
        from paged_kv_cache_424_b200.session import DeviceSession
        self.sc, self.pa, self.W, self.torch = sc, pa, W, torch
        self.device = device
        self.fp8 = sc.kv_dtype == "fp8"
        self.P = sc.partition_tokens if partition is None else partition
        self.dev = DeviceSession(sc, device=str(device))
        setup, cycle = scenario_cycle(sc)
        for st in setup + cycle:
            self.dev.apply_cache_ops(st)
        self.items = []
        for st in cycle:
            inp = self.dev.decode_inputs(st)
            writes = self.dev.write_inputs(st)
            bm = torch.from_numpy(np.ascontiguousarray(st.block_mapping)).to(device) if st.block_mapping.size \
                else None
            maxlen = st.max_context_len
            if sc.ext:
                ws_bytes = self.dev.ext_workspace_bytes(inp, maxlen, self.P)
                nparts = None
            else:
                dims = pa.dims_of(inp["q"], self.dev.k_cache, inp["block_tables"])
                nparts = pa.pa_decode_num_partitions(dims, maxlen, self.P)
                ws_bytes = pa.pa_decode_workspace_size(dims, maxlen, self.P)
            kv_logical = W.kv_bytes(st, sc.dims, elem_bytes=sc.kv_elem_bytes, q_len=sc.q_len, window=sc.window)
            kv = (W.kv_bytes(st, sc.dims, unique=True, elem_bytes=sc.kv_elem_bytes)
                  if sc.name.split("-")[0] in ("cow", "prefix8b") else kv_logical)
            qo = W.qo_bytes(sc.dims, sc.q_len)
            launches = (1 if bm is not None else 0) + len(writes) + (2 if ws_bytes else 1)
            self.items.append(dict(step=st, inp=inp, writes=writes, bm=bm, maxlen=maxlen, ws_bytes=ws_bytes,
                                   nparts=nparts, kv=kv, kv_logical=kv_logical, algo=kv + qo,
                                   logical=kv_logical + qo, launches=launches))
        self.ws = self.dev.workspace(max(it["ws_bytes"] for it in self.items))
        self.out = torch.empty_like(self.items[0]["inp"]["q"])

    # -- the library calls of one step -----------------------------------------
    def write(self, key, value, slots, stream):
        sc, pa, dev = self.sc, self.pa, self.dev
        if self.fp8:
            pa.pa_reshape_and_cache_fp8(key, value, dev.k_cache, dev.v_cache, slots, sc.k_scale, sc.v_scale,
                                        stream=stream)
        else:
            pa.pa_reshape_and_cache(key, value, dev.k_cache, dev.v_cache, slots, stream=stream)

    def decode(self, it, q, bt, cl, out, stream, seq_order=None):
        sc, pa, dev = self.sc, self.pa, self.dev
        if sc.ext:
            dev.decode_ext({"q": q, "block_tables": bt, "context_lens": cl, "seq_order": seq_order}, it["maxlen"],
                           self.P, out, stream=stream)
        elif self.fp8:
            pa.pa_decode_fp8(out, q, dev.k_cache, dev.v_cache, bt, cl, sc.scale, sc.k_scale, sc.v_scale,
                             sc.dims.num_kv_heads, it["maxlen"], self.P, self.ws, stream=stream)
        else:
            pa.pa_decode(out, q, dev.k_cache, dev.v_cache, bt, cl, sc.scale, sc.dims.num_kv_heads, it["maxlen"],
                         self.P, self.ws, stream=stream)

    def step(self, it, stream, e0=None, e1=None, seq_order="default"):
        pa, dev = self.pa, self.dev
        if it["bm"] is not None:
            pa.pa_copy_blocks([dev.k_cache], [dev.v_cache], it["bm"], stream=stream)
        for key, value, slots in it["writes"]:
            self.write(key, value, slots, stream)
        if e0 is not None:
            e0.record(stream)
        inp = it["inp"]
        so = inp.get("seq_order") if seq_order == "default" else seq_order
        self.decode(it, inp["q"], inp["block_tables"], inp["context_lens"], self.out, stream, so)
        if e1 is not None:
            e1.record(stream)

    # -- timing ----------------------------------------------------------------
    def time_steps(self, K, warmup, stream, world, seq_order="default", clocks=None):
        """Three timed loops over the cycle, after `warmup` untimed steps.
        The step loop (K steps) has events only at its two ends, so
        consecutive kernels keep their programmatic-dependent-launch
        overlap: total ms (max over ranks).  The decode loop launches the K
        steps' decodes back to back between two events: the decode's device
        time per launch in steady state (ms, max over ranks), the roofline's
        denominator.  The bracket loop repeats the steps with an event pair
        around every decode launch, which also charges each launch its
        launch latency: per-launch ms (this rank).  Returns (step total ms,
        decode ms per launch, bracketed per-launch ms, cycle item of each)."""
        torch = self.torch
        C = len(self.items)
        for i in range(warmup):
            self.step(self.items[i % C], stream, seq_order=seq_order)
        torch.cuda.synchronize(self.device)
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(self.device)
        ctx = clocks if clocks is not None else _NullCtx()
        with ctx:
            start.record(stream)
            for i in range(K):
                self.step(self.items[(warmup + i) % C], stream, seq_order=seq_order)
            end.record(stream)
            torch.cuda.synchronize(self.device)
            barrier(world)
            d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            d0.record(stream)
            for i in range(K):
                it = self.items[(warmup + i) % C]
                inp = it["inp"]
                so = inp.get("seq_order") if seq_order == "default" else seq_order
                self.decode(it, inp["q"], inp["block_tables"], inp["context_lens"], self.out, stream, so)
            d1.record(stream)
            torch.cuda.synchronize(self.device)
            barrier(world)
            for i in range(K):
                self.step(self.items[(warmup + i) % C], stream, e0[i], e1[i], seq_order=seq_order)
            torch.cuda.synchronize(self.device)
        barrier(world)
        ms_total = max_over_ranks(start.elapsed_time(end), world, self.device)
        dec_ms = max_over_ranks(d0.elapsed_time(d1), world, self.device) / K
        bracket_ms = [a.elapsed_time(b) for a, b in zip(e0, e1)]
        idx = [(warmup + i) % C for i in range(K)]
        return ms_total, dec_ms, bracket_ms, idx

    def roofline_of(self, dec_ms, idx):
        """Algorithmic bytes of the timed decodes over their time (dec_ms per
        launch): GB/s, logical GB/s, bytes per launch."""
        algo = sum(self.items[j]["algo"] for j in idx)
        logical = sum(self.items[j]["logical"] for j in idx)
        t = dec_ms * len(idx) / 1e3
        return algo / t / 1e9, logical / t / 1e9, algo / len(idx)

    # -- end to end ------------------------------------------------------------
    def e2e(self, K, warmup, stream, world):
        """The same steps through the same calls with their inputs in pinned
        host memory: per step, one host-to-device copy of all the step's
        inputs (query, tables, lengths, new keys / values / slots, copy
        pairs, schedule) packed in one buffer, the step's kernels reading
        them in place, and one device-to-host copy of the output.  Copies run
        on their own streams, double-buffered and ordered by events, so the
        upload of step i + 1 and the download of step i - 1 overlap step i."""
        torch, pa = self.torch, self.pa
        dev = self.device
        C = len(self.items)
        packs = [self._pack(it) for it in self.items]
        nbytes = max(p["nbytes"] for p in packs)
        staging = [torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        views = [[self._views(p, staging[b]) for b in range(2)] for p in packs]
        outs = [torch.empty_like(self.out) for _ in range(2)]
        h_out = [torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory() for _ in range(2)]
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        ev_host = [torch.cuda.Event() for _ in range(C)]  # last upload that read host pack j
        host_order = self.sc.prefix_order

        def run(i):
            b, j = i % 2, i % C
            p, v = packs[j], views[j][b]
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(ev_done[b])  # staging b: step i - 2 has finished with it
                if host_order:
                    ev_host[j].synchronize()      # the host pack is free again
                    p["arrays"]["seq_order"][:] = pa.pa_prefix_order(p["arrays"]["block_tables"],
                                                                     p["arrays"]["context_lens"])
                staging[b].copy_(p["host"], non_blocking=True)
                ev_in[b].record(h2d_s)
                ev_host[j].record(h2d_s)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])      # outs[b]: step i - 2's output has been read back
            it = self.items[j]
            if "bm" in v:
                pa.pa_copy_blocks([self.dev.k_cache], [self.dev.v_cache], v["bm"], stream=stream)
            for w in range(len(it["writes"])):
                self.write(v[f"key{w}"], v[f"value{w}"], v[f"slots{w}"], stream)
            self.decode(it, v["q"], v["block_tables"], v["context_lens"], outs[b], stream, v.get("seq_order"))
            ev_done[b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_done[b])
                h_out[b].copy_(outs[b], non_blocking=True)
                ev_out[b].record(d2h_s)

        for i in range(warmup):
            run(i)
        torch.cuda.synchronize(dev)
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(dev)
        a.record(stream)
        h2d_s.wait_event(a)
        for i in range(warmup, warmup + K):
            run(i)
        stream.wait_event(ev_out[(warmup + K - 1) % 2])
        z.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        ms = max_over_ranks(a.elapsed_time(z), world, dev)
        h2d = sum(packs[(warmup + i) % C]["nbytes"] for i in range(K)) / K
        d2h = self.out.numel() * self.out.element_size()
        return {"value": self.sc.dims.num_seqs * K * world / (ms / 1e3), "unit": "seqs/s",
                "h2d_bytes_per_step": int(round(h2d)), "d2h_bytes_per_step": int(d2h), "steps": K,
                "ms_per_step": ms / K,
                "path": "pinned host pack -> one cudaMemcpyAsync (copy stream) -> pa_* C-ABI calls reading the "
                        "device pack -> one cudaMemcpyAsync of the output back (second copy stream); "
                        "double-buffered, event-ordered"}

    def _pack(self, it):
        """The step's host inputs laid out in one pinned buffer (256-byte
        aligned pieces)."""
        torch = self.torch
        st = it["step"]
        pieces = {"q": np.ascontiguousarray(st.q).view(np.uint16),
                  "block_tables": np.ascontiguousarray(st.block_tables, dtype=np.int32),
                  "context_lens": np.ascontiguousarray(st.context_lens, dtype=np.int32)}
        for w, wr in enumerate(st.writes):
            pieces[f"key{w}"] = np.ascontiguousarray(wr.key)
            pieces[f"value{w}"] = np.ascontiguousarray(wr.value)
            pieces[f"slots{w}"] = np.ascontiguousarray(wr.slot_mapping, dtype=np.int64)
        if st.block_mapping.size:
            pieces["bm"] = np.ascontiguousarray(st.block_mapping, dtype=np.int64)
        if self.sc.prefix_order:
            pieces["seq_order"] = np.zeros(st.context_lens.shape, np.int32)
        layout, off = {}, 0
        for k, a in pieces.items():
            layout[k] = (off, a.dtype, a.shape, a.nbytes)
            off += (a.nbytes + 255) // 256 * 256
        host = torch.empty(off, dtype=torch.uint8).pin_memory()
        hb = host.numpy()
        arrays = {}
        for k, a in pieces.items():
            o, dt, shape, n = layout[k]
            hb[o:o + n] = a.view(np.uint8).ravel()
            arrays[k] = hb[o:o + n].view(dt).reshape(shape)
        return {"host": host, "layout": layout, "nbytes": off, "arrays": arrays}

    def _views(self, p, buf):
        torch = self.torch
        tdt = {"q": self.dev.dtype}
        for k in p["layout"]:
            if k.startswith("key") or k.startswith("value"):
                tdt[k] = self.dev.dtype
        npt = {np.dtype(np.int32): torch.int32, np.dtype(np.int64): torch.int64}
        out = {}
        for k, (o, dt, shape, n) in p["layout"].items():
            t = buf[o:o + n]
            t = t.view(tdt[k]) if k in tdt else t.view(npt[np.dtype(dt)])
            out[k] = t.view(shape)
        return out


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def cpu_baseline(sc, seconds: float):
    """The oracle as it stands on this host's cores, on the first step of the
    timed cycle (the cache write of the step plus decode of as many of its
    sequences as fit the time budget, repeated)."""
    import oracle
    from oracle.harness import OracleSession
    orc = oracle.load()
    cores = orc.max_threads()
    setup, cycle = scenario_cycle(sc)
    st = cycle[0]
    ses = OracleSession(sc, oracle=orc)
    for s in setup + [st]:
        ses.apply_cache_ops(s)       # admission + writes, outside the timing
    S = sc.dims.num_seqs
    t0 = time.perf_counter()
    ses.decode(st, np.arange(min(S, 4)))
    t_seq = (time.perf_counter() - t0) / min(S, 4)
    n = int(max(1, min(S, seconds / max(t_seq, 1e-9))))
    seqs_done, t_total, reps = 0, 0.0, 0
    while t_total < seconds or reps == 0:
        sel = (np.arange(n) + reps * n) % S
        t0 = time.perf_counter()
        for w in st.writes:   # the step's cache write, on the host pool
            ses.write(w.key, w.value, w.slot_mapping)
        ses.decode(st, sel)
        t_total += time.perf_counter() - t0
        seqs_done += n
        reps += 1
        if t_total > 3 * seconds:
            break
    return {"value": seqs_done / t_total, "unit": "seqs/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} x ({n} of {S} sequences of the first timed step: cache write of the step + "
                      f"float64 decode), {t_total:.1f} s, {cores} OpenMP threads"}


def also_entry(args, name, kv, rank, world, device, stream, pa, W, K):
    """Decode time and roofline fraction of another workload, same box."""
    import torch
    sc = make_scenario(name, seed=1 + rank, kv=kv)
    wl = DeviceWorkload(sc, device, None, pa, W)
    clocks = ClockSampler(device.index if device.index is not None else 0)
    ms_total, dec, bracket, idx = wl.time_steps(K, max(3, min(args.warmup, 20)), stream, world, clocks=clocks)
    if pa.pa_device_error(stream) != 0:
        raise SystemExit(f"device error word set while timing {name}")
    gbs, eff, algo = wl.roofline_of(dec, idx)
    peak, _ = measured_hbm_peak()
    it = wl.items[0]
    ent = {"workload": f"{sc.name}: {sc.note}", "decode_us": dec * 1e3, "decode_gbs": gbs,
           "decode_us_bracketed": sum(bracket) / len(bracket) * 1e3,
           "frac": gbs / peak, "frac_of_8000": gbs / TARGET_GBS, "step_us": ms_total / K * 1e3,
           "seqs_per_s": sc.dims.num_seqs * K * world / (ms_total / 1e3), "algorithmic_bytes": algo,
           "partition_tokens": wl.P, "num_partitions": it["nparts"], "steps": K,
           "clocks": clocks.summary()}
    if name in ("cow", "prefix8b"):
        ent["effective_gbs_logical"] = eff
    del wl
    torch.cuda.empty_cache()
    return ent


def run_ours(args):
    import torch
    world, rank, local = dist_setup(args)
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    from paged_kv_cache_424_b200 import build
    build.build()
    from paged_kv_cache_424_b200 import binding as pa
    from paged_kv_cache_424_b200 import workload as W

    sc = make_scenario(args.workload, seed=1 + rank, num_seqs=args.num_seqs, num_blocks=args.num_blocks, kv=args.kv,
                       cycle=args.cycle)
    if args.no_prefix_order and sc.prefix_order:
        import dataclasses
        sc = dataclasses.replace(sc, prefix_order=False)
    d = sc.dims
    fp8 = sc.kv_dtype == "fp8"
    stream = torch.cuda.current_stream(device)
    wl = DeviceWorkload(sc, device, args.partition, pa, W)
    if pa.pa_device_error(stream) != 0:
        raise SystemExit("device error word set during set-up")

    K = args.steps
    clocks = ClockSampler(device.index if device.index is not None else 0)
    ms_total, dec_avg_ms, bracket_ms, idx = wl.time_steps(K, args.warmup, stream, world, clocks=clocks)
    if pa.pa_device_error(stream) != 0:
        raise SystemExit("device error word set during the timed region")
    achieved, eff_logical, algo = wl.roofline_of(dec_avg_ms, idx)

    # shared-prefix order: the same decode in plain batch order, for comparison
    no_order_ms = None
    if sc.prefix_order:
        _, no_order_ms, _, _ = wl.time_steps(K, 3, stream, world, seq_order=None)

    e2e = None
    if not args.no_e2e:
        e2e = wl.e2e(max(1, min(K, 500)), min(args.warmup, 10), stream, world)
        if pa.pa_device_error(stream) != 0:
            raise SystemExit("device error word set during the end-to-end run")

    launches = sum(wl.items[j]["launches"] for j in idx)
    it0 = wl.items[0]
    lens = np.concatenate([wl.items[j]["step"].context_lens for j in range(len(wl.items))])
    kv_step = sum(wl.items[j]["kv"] for j in idx) / K
    kv_logical_step = sum(wl.items[j]["kv_logical"] for j in idx) / K
    nparts = sorted({it["nparts"] for it in wl.items if it["nparts"] is not None})
    C = len(wl.items)
    kernel = ("pa_decode_ext" if sc.ext else "pa_decode_fp8" if fp8 else "pa_decode") + \
        (" (decode kernel + log-sum-exp merge)" if any(it["ws_bytes"] for it in wl.items) else "")
    units = float(sum(int(wl.items[j]["step"].context_lens.sum()) for j in idx)) / K
    del wl
    torch.cuda.empty_cache()

    also = {}
    for name, kv in also_list(args):
        key = name + ("-fp8" if kv == "fp8" else "")
        also[key] = also_entry(args, name, kv, rank, world, device, stream, pa, W, min(max(K, 100), 500))

    part_tokens = sc.partition_tokens if args.partition is None else args.partition
    peak, peak_kind = measured_hbm_peak()
    traffic = ncu_traffic(args.workload + ("-fp8" if fp8 else ""), units=units)
    result = {
        "metric": METRIC,
        "value": d.num_seqs * K * world / (ms_total / 1e3),
        "unit": "seqs/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_total / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": f"{d.dtype} q/out, e4m3 KV cache" if fp8 else d.dtype,
        "data": "synthetic (seeded U[-1,1] fp16/bf16 values, NaN in every unused slot; no dataset)",
        "config": {"workload": f"{sc.name}: {sc.note}", "global_batch": d.num_seqs * world,
                   "seq_len": f"per-sequence, mean {float(lens.mean()):.0f}, max {int(lens.max())} over the cycle",
                   "timed_cycle": (f"{C} churned steps (after 2 set-up steps), walked in turn: each timed step "
                                   f"decodes a different batch mix" if C > 1 else "one step, repeated"),
                   "partition_tokens": part_tokens or "auto",
                   "num_partitions": nparts if nparts else "split" if "merge" in kernel else 1,
                   **({"q_len": sc.q_len, "window": sc.window} if sc.ext else {}),
                   **({"seq_order": "pa_prefix_order", "decode_ms_batch_order": no_order_ms,
                       "decode_ms_prefix_order": dec_avg_ms,
                       "prefix_order_speedup": no_order_ms / dec_avg_ms} if no_order_ms else {}),
                   "parallelism": f"{world} independent batches (one per GPU, no data-path collective)",
                   "l2": f"inputs larger than L2: {kv_step / 1e9:.2f} GB of KV read per step vs 126 MB L2",
                   "kv_bytes_per_step": kv_step, "kv_bytes_logical_per_step": kv_logical_step,
                   "algorithmic_bytes_per_step": algo,
                   **({"also": also} if also else {})},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "peak_kind": f"{peak_kind} copy bandwidth",
                     "kernel": kernel, "kernel_ms": dec_avg_ms,
                     "kernel_ms_how": "K decode launches back to back between two CUDA events, cycling through the "
                                      "timed steps' batches: device time per launch in steady state",
                     "kernel_ms_bracketed": max_over_ranks(sum(bracket_ms) / K, world, device),
                     "frac_of_8000": achieved / TARGET_GBS,
                     "effective_gbs_logical": eff_logical},
        "clocks": clocks.summary(),
        "e2e": e2e,
        "gpu_launches": launches,
    }
    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(sc, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle, timed like our arm
# ---------------------------------------------------------------------------
def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return
    import oracle
    from oracle.harness import OracleSession
    orc = oracle.load()
    cores = orc.max_threads()
    sc = make_scenario(args.workload, seed=1, num_seqs=args.num_seqs, num_blocks=args.num_blocks, kv=args.kv,
                       cycle=args.cycle)
    setup, cycle = scenario_cycle(sc)
    S = sc.dims.num_seqs
    ses = OracleSession(sc, oracle=orc)
    for st in setup + cycle:
        ses.apply_cache_ops(st)
    t0 = time.perf_counter()
    ses.decode(cycle[0], np.arange(min(S, 2)))
    t_seq = (time.perf_counter() - t0) / min(S, 2)
    budget = 120.0 / max(1, args.steps + args.warmup)          # seconds per step
    n = int(max(1, min(S, budget / max(t_seq, 1e-9))))

    def one(i):
        st = cycle[i % len(cycle)]
        sel = (np.arange(n) + i * n) % S
        for w in st.writes:
            ses.write(w.key, w.value, w.slot_mapping)
        ses.decode(st, sel)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(args.warmup + i)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    sample = (f"each step: {n} of {S} sequences of the step's batch (cache write + float64 decode), walking the "
              f"{len(cycle)}-step cycle, {cores} OpenMP threads")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "seqs/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{sc.name}: {sc.note}", "global_batch": S, "sample_seqs_per_step": n},
        "cpu_baseline": {"value": value, "unit": "seqs/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "seqs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---------------------------------------------------------------------------
# swap_blocks: device <-> page-locked host block copies (preemption)
# ---------------------------------------------------------------------------
def run_swap(args):
    """Swap 2048 blocks of the 7B shape (32 KV heads x 16 x 128 fp16: 128 KiB
    of K and 128 KiB of V each) out to a pinned host pool and back in.  One
    step = one swap-out + one swap-in; value = GB/s moved per direction."""
    import torch
    from paged_kv_cache_424_b200 import build
    build.build()
    from paged_kv_cache_424_b200 import binding as pa
    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    nb_dev, nb_host, pairs, shape = 8192, 4096, 2048, (32, 16, 128)
    rng = np.random.default_rng(7 + rank)
    dk = torch.randn((nb_dev, *shape), device=dev, dtype=torch.float16)
    dv = torch.randn((nb_dev, *shape), device=dev, dtype=torch.float16)
    hk = torch.empty((nb_host, *shape), dtype=torch.float16).pin_memory()
    hv = torch.empty((nb_host, *shape), dtype=torch.float16).pin_memory()
    out_map = torch.from_numpy(np.stack([rng.choice(nb_dev, pairs, replace=False),
                                         rng.choice(nb_host, pairs, replace=False)], 1).astype(np.int64)).to(dev)
    in_map = torch.stack([out_map[:, 1], out_map[:, 0]], 1).contiguous()
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        pa.pa_swap_blocks(dk, dv, hk, hv, out_map, stream=stream)
        pa.pa_swap_blocks(hk, hv, dk, dv, in_map, stream=stream)
    torch.cuda.synchronize(dev)
    K = args.steps
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    barrier(world)
    e[0].record(stream)
    for _ in range(K):
        pa.pa_swap_blocks(dk, dv, hk, hv, out_map, stream=stream)
    e[1].record(stream)
    for _ in range(K):
        pa.pa_swap_blocks(hk, hv, dk, dv, in_map, stream=stream)
    e[2].record(stream)
    torch.cuda.synchronize(dev)
    out_ms = max_over_ranks(e[0].elapsed_time(e[1]) / K, world, dev)
    in_ms = max_over_ranks(e[1].elapsed_time(e[2]) / K, world, dev)
    if pa.pa_device_error(stream) != 0:
        raise SystemExit("device error word set")
    nbytes = pairs * 2 * int(np.prod(shape)) * 2
    if rank == 0:
        print(json.dumps({
            "metric": "pa_swap_blocks throughput, device <-> page-locked host (GB/s per direction)",
            "value": nbytes * world / ((out_ms + in_ms) / 2 / 1e3) / 1e9, "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": out_ms + in_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": f"swap {pairs} blocks of 32x16x128 fp16 K+V ({nbytes / 2**20:.0f} MiB) "
                                   f"out of a {nb_dev}-block device pool and back in",
                       "swap_out_gbs": nbytes / (out_ms / 1e3) / 1e9, "swap_in_gbs": nbytes / (in_ms / 1e3) / 1e9},
            "gpu_launches": 2 * K}), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.workload == "swap":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "swap throughput has no CPU-oracle arm"}))
            return
        run_swap(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
