#!/usr/bin/env python
"""Benchmark: paged decode attention on B200, one JSON line on stdout.

A step is one pass of the whole hot path over one batch: the cache write of
every sequence's new token (pa_reshape_and_cache), copy-on-write copies when
the workload has them (pa_copy_blocks), and decode attention of every
sequence over its paged KV cache (pa_decode, with the split-KV merge when a
context spans several 512-token partitions).  Default workload: the
Llama-2-7B-shaped MHA batch (64 sequences, lengths U[128, 2048], 32 heads,
head_dim 128, fp16, 16384-block pool).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--kv 16|fp8]
  python bench.py --impl reference ...      # the CPU oracle, timed the same way

Other workloads: gqa8b, long70b, cow (the pages' other shapes), spec8b (4
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
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mha7b",
                    choices=["tiny", "mha7b", "gqa8b", "long70b", "cow", "spec8b", "window70b", "prefix8b", "swap"],
                    help="decode scenario (spec8b: 4 query tokens per sequence; window70b: 4096-token sliding "
                         "window; prefix8b: shuffled batch of shared 2000-token prefixes, decoded in "
                         "shared-prefix order), or 'swap' for pa_swap_blocks device <-> pinned host throughput")
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


def make_scenario(name: str, seed: int, num_seqs=None, num_blocks=None, kv: str = "16"):
    from paged_kv_cache_424_b200 import workload as W
    sc = _base_scenario(name, seed, num_seqs, num_blocks)
    return W.with_fp8_cache(sc) if kv == "fp8" else sc


def _base_scenario(name: str, seed: int, num_seqs=None, num_blocks=None):
    from paged_kv_cache_424_b200 import workload as W
    kw = {}
    if num_seqs is not None:
        kw["num_seqs"] = num_seqs
    if num_blocks is not None:
        kw["num_blocks"] = num_blocks
    if name == "tiny":
        return W.tiny(seed)
    if name in ("cow", "prefix8b"):
        if num_seqs is not None:
            kw = {"num_prompts": max(1, num_seqs // 8), **({"num_blocks": num_blocks} if num_blocks else {})}
        return getattr(W, name)(seed, **kw)
    return getattr(W, name)(seed, **kw)


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

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
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


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def cpu_baseline(sc, seconds: float):
    """The oracle as it stands on this host's cores, on repeated full steps of
    the workload (or a subset of its sequences when one step is too long)."""
    import oracle
    from oracle.harness import OracleSession
    orc = oracle.load()
    cores = orc.max_threads()
    st = sc.steps[0]
    ses = OracleSession(sc, oracle=orc)
    ses.apply_cache_ops(st)          # admission + writes, outside the timing
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
            "sample": f"{reps} x ({n} of {S} sequences: cache write of the step + float64 decode), "
                      f"{t_total:.1f} s, {cores} OpenMP threads"}


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
    from paged_kv_cache_424_b200.session import DeviceSession, to_device

    sc = make_scenario(args.workload, seed=1 + rank, num_seqs=args.num_seqs, num_blocks=args.num_blocks, kv=args.kv)
    if args.no_prefix_order and sc.prefix_order:
        import dataclasses
        sc = dataclasses.replace(sc, prefix_order=False)
    st = sc.steps[0]
    d = sc.dims
    fp8 = sc.kv_dtype == "fp8"
    P = sc.partition_tokens if args.partition is None else args.partition
    dev = DeviceSession(sc, device=str(device))
    dev.apply_cache_ops(st)                      # prefill admission + first writes (untimed set-up)
    inp = dev.decode_inputs(st)
    writes = dev.write_inputs(st)
    bm = torch.from_numpy(np.ascontiguousarray(st.block_mapping)).to(device) if st.block_mapping.size else None
    maxlen = st.max_context_len
    if sc.ext:
        ws_bytes = dev.ext_workspace_bytes(inp, maxlen, P)
        nparts = "split" if ws_bytes else 1
    else:
        dims = pa.dims_of(inp["q"], dev.k_cache, inp["block_tables"])
        nparts = pa.pa_decode_num_partitions(dims, maxlen, P)
        ws_bytes = pa.pa_decode_workspace_size(dims, maxlen, P)
    ws = dev.workspace(ws_bytes)
    out = torch.empty_like(inp["q"])
    stream = torch.cuda.current_stream(device)

    def write(key, value, slots):
        if fp8:
            pa.pa_reshape_and_cache_fp8(key, value, dev.k_cache, dev.v_cache, slots, sc.k_scale, sc.v_scale,
                                        stream=stream)
        else:
            pa.pa_reshape_and_cache(key, value, dev.k_cache, dev.v_cache, slots, stream=stream)

    def decode(q, bt, cl, seq_order=None):
        if sc.ext:
            dev.decode_ext({"q": q, "block_tables": bt, "context_lens": cl, "seq_order": seq_order}, maxlen, P, out,
                           stream=stream)
        elif fp8:
            pa.pa_decode_fp8(out, q, dev.k_cache, dev.v_cache, bt, cl, sc.scale, sc.k_scale, sc.v_scale,
                             d.num_kv_heads, maxlen, P, ws, stream=stream)
        else:
            pa.pa_decode(out, q, dev.k_cache, dev.v_cache, bt, cl, sc.scale, d.num_kv_heads, maxlen, P, ws,
                         stream=stream)

    def step(e0=None, e1=None):
        if bm is not None:
            pa.pa_copy_blocks([dev.k_cache], [dev.v_cache], bm, stream=stream)
        for key, value, slots in writes:
            write(key, value, slots)
        if e0 is not None:
            e0.record(stream)
        decode(inp["q"], inp["block_tables"], inp["context_lens"], inp.get("seq_order"))
        if e1 is not None:
            e1.record(stream)

    launches_per_step = (1 if bm is not None else 0) + len(writes) + (2 if ws_bytes else 1)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if pa.pa_device_error(stream) != 0:
        raise SystemExit("device error word set during warm-up")

    K = args.steps
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as clocks:
        start.record(stream)
        for i in range(K):
            step(e0[i], e1[i])
        end.record(stream)
        torch.cuda.synchronize(device)
    barrier(world)
    ms_total = max_over_ranks(start.elapsed_time(end), world, device)
    dec_ms = [a.elapsed_time(b) for a, b in zip(e0, e1)]
    dec_avg_ms = max_over_ranks(sum(dec_ms) / K, world, device)

    # shared-prefix order: the same decode in plain batch order, for comparison
    no_order_ms = None
    if sc.prefix_order:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(3):
            decode(inp["q"], inp["block_tables"], inp["context_lens"], None)
        barrier(world)
        torch.cuda.synchronize(device)
        a.record(stream)
        for _ in range(K):
            decode(inp["q"], inp["block_tables"], inp["context_lens"], None)
        b.record(stream)
        torch.cuda.synchronize(device)
        no_order_ms = max_over_ranks(a.elapsed_time(b) / K, world, device)

    # ---- end to end: host buffers in, result out, through the same calls ----
    e2e = None
    if not args.no_e2e:
        h_q = inp["q"].cpu().pin_memory()
        h_bt = inp["block_tables"].cpu().pin_memory()
        h_cl = inp["context_lens"].cpu().pin_memory()
        h_w = [(k.cpu().pin_memory(), v.cpu().pin_memory(), s.cpu().pin_memory()) for k, v, s in writes]
        h_bm = st.block_mapping
        h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        d_q, d_bt, d_cl = torch.empty_like(inp["q"]), torch.empty_like(inp["block_tables"]), torch.empty_like(
            inp["context_lens"])
        d_w = [(torch.empty_like(k), torch.empty_like(v), torch.empty_like(s)) for k, v, s in writes]
        h_bm_t = torch.from_numpy(np.ascontiguousarray(h_bm)).pin_memory() if bm is not None else None
        d_bm = torch.empty_like(bm) if bm is not None else None
        d_so = torch.empty(d.num_seqs, dtype=torch.int32, device=device) if sc.prefix_order else None
        h_so = torch.empty(d.num_seqs, dtype=torch.int32).pin_memory() if sc.prefix_order else None
        h2d = ((h_so.numel() * 4 if h_so is not None else 0) +
               h_q.numel() * h_q.element_size() + h_bt.numel() * 4 + h_cl.numel() * 4 +
               sum(k.numel() * k.element_size() * 2 + s.numel() * 8 for k, _, s in h_w) +
               (h_bm_t.numel() * 8 if h_bm_t is not None else 0))
        d2h = h_out.numel() * h_out.element_size()

        def e2e_step():
            d_q.copy_(h_q, non_blocking=True)
            d_bt.copy_(h_bt, non_blocking=True)
            d_cl.copy_(h_cl, non_blocking=True)
            for (hk, hv, hs), (dk, dv, ds) in zip(h_w, d_w):
                dk.copy_(hk, non_blocking=True)
                dv.copy_(hv, non_blocking=True)
                ds.copy_(hs, non_blocking=True)
            if d_bm is not None:
                d_bm.copy_(h_bm_t, non_blocking=True)
                pa.pa_copy_blocks([dev.k_cache], [dev.v_cache], d_bm, stream=stream)
            for dk, dv, ds in d_w:
                write(dk, dv, ds)
            if h_so is not None:  # the host schedule of this step, then its copy
                h_so.numpy()[:] = pa.pa_prefix_order(h_bt.numpy(), h_cl.numpy())
                d_so.copy_(h_so, non_blocking=True)
            decode(d_q, d_bt, d_cl, d_so)
            h_out.copy_(out, non_blocking=True)

        for _ in range(min(args.warmup, 10)):
            e2e_step()
        torch.cuda.synchronize(device)
        Ke = max(1, min(K, 500))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(device)
        a.record(stream)
        for _ in range(Ke):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(device)
        barrier(world)
        e2e_ms = max_over_ranks(a.elapsed_time(b), world, device)
        e2e = {"value": d.num_seqs * Ke * world / (e2e_ms / 1e3), "unit": "seqs/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": Ke,
               "path": "pinned host buffers -> cudaMemcpyAsync -> pa_* C-ABI calls -> output copied back"}

    if pa.pa_device_error(stream) != 0:
        raise SystemExit("device error word set during the timed region")

    # Algorithmic bytes: KV of the referenced tokens; blocks shared by several
    # sequences (copy-on-write prefixes) count once, as the pool holds them once.
    kv_logical = W.kv_bytes(st, d, elem_bytes=sc.kv_elem_bytes, q_len=sc.q_len, window=sc.window)
    kv = (W.kv_bytes(st, d, unique=True, elem_bytes=sc.kv_elem_bytes) if args.workload in ("cow", "prefix8b")
          else kv_logical)
    algo = kv + W.qo_bytes(d, sc.q_len)
    peak, peak_kind = measured_hbm_peak()
    achieved = algo / (dec_avg_ms / 1e3) / 1e9
    traffic = ncu_traffic(args.workload + ("-fp8" if fp8 else ""), units=float(st.context_lens.sum()))
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
                   "seq_len": "per-sequence, " + f"mean {float(st.context_lens.mean()):.0f}, "
                              f"max {int(st.context_lens.max())}",
                   "partition_tokens": P, "num_partitions": nparts,
                   **({"q_len": sc.q_len, "window": sc.window} if sc.ext else {}),
                   **({"seq_order": "pa_prefix_order", "decode_ms_batch_order": no_order_ms,
                       "decode_ms_prefix_order": dec_avg_ms,
                       "prefix_order_speedup": no_order_ms / dec_avg_ms} if no_order_ms else {}),
                   "parallelism": f"{world} independent batches (one per GPU, no data-path collective)",
                   "l2": f"inputs larger than L2: {kv / 1e9:.2f} GB of KV read per step vs 126 MB L2",
                   "kv_bytes_per_step": kv, "kv_bytes_logical_per_step": kv_logical,
                   "algorithmic_bytes_per_step": algo},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "peak_kind": f"{peak_kind} copy bandwidth",
                     "kernel": ("pa_decode_ext" if sc.ext else "pa_decode_fp8" if fp8 else "pa_decode") +
                               (" (decode kernel + log-sum-exp merge)" if ws_bytes else ""),
                     "kernel_ms": dec_avg_ms, "frac_of_8000": achieved / 8000.0,
                     "effective_gbs_logical": (kv_logical + W.qo_bytes(d, sc.q_len)) / (dec_avg_ms / 1e3) / 1e9},
        "clocks": clocks.summary(),
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,
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
    sc = make_scenario(args.workload, seed=1, num_seqs=args.num_seqs, num_blocks=args.num_blocks, kv=args.kv)
    st = sc.steps[0]
    S = sc.dims.num_seqs
    ses = OracleSession(sc, oracle=orc)
    ses.apply_cache_ops(st)
    t0 = time.perf_counter()
    ses.decode(st, np.arange(min(S, 2)))
    t_seq = (time.perf_counter() - t0) / min(S, 2)
    budget = 120.0 / max(1, args.steps + args.warmup)          # seconds per step
    n = int(max(1, min(S, budget / max(t_seq, 1e-9))))

    def one(i):
        sel = (np.arange(n) + i * n) % S
        for w in st.writes:
            ses.write(w.key, w.value, w.slot_mapping)
        ses.decode(st, sel)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(i)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    sample = f"each step: {n} of {S} sequences (cache write + float64 decode), {cores} OpenMP threads"
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
