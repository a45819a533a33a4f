"""GPU parity of multi-token and sliding-window decode (pa_decode_ext)
against the oracle's masked definition: several query tokens per sequence
(speculative verification, "vLLM PagedAttention 大模型推理架构深度实战" section
九 item 2) and a sliding window (the same page, section 7.2), over 16-bit and
FP8 caches, on both kernels, at reduced and full sizes.  Table entries of
blocks before a sequence's window hold invalid ids: the kernels must never
read them (the device error word stays clear).
"""
import numpy as np
import pytest
import torch

from gpu_util import compare, require_gpu, run_and_compare
from pins import Paged, rand_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    from paged_kv_cache_424_b200 import build
    build.build()
    from paged_kv_cache_424_b200 import binding
    assert binding.pa_device_error() == 0, "device error word set before the test"
    yield
    assert binding.pa_device_error() == 0, "a kernel flagged a device error"


def W():
    from paged_kv_cache_424_b200 import workload
    return workload


TORCH = {"f16": torch.float16, "bf16": torch.bfloat16}


def _dev16(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(TORCH[dtype])


def poison_before_window(tables, lens, q_len, window, B=16):
    """Entries of blocks wholly before every query's window -> -1."""
    t = tables.copy()
    if window > 0:
        for s, L in enumerate(lens):
            lo = max(0, int(L) - q_len - window + 1)
            t[s, :lo // B] = -1
    return t


def run_ext(q_bits, kc, vc, tables, lens, scale, dtype, q_len, window, P, k_scale=1.0, v_scale=1.0, kv8=False):
    from paged_kv_cache_424_b200 import binding as pa
    q = _dev16(q_bits, dtype)
    k = torch.from_numpy(kc).cuda() if kv8 else _dev16(kc, dtype)
    v = torch.from_numpy(vc).cuda() if kv8 else _dev16(vc, dtype)
    bt = torch.from_numpy(np.ascontiguousarray(tables)).cuda()
    cl = torch.from_numpy(np.asarray(lens, np.int32)).cuda()
    maxlen = int(max(lens))
    dims = pa.ext_dims(q, k, bt)
    n = pa.pa_decode_ext_workspace_size(dims, pa.pa_decode_opts(q_len, window, k_scale, v_scale), maxlen, P)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda") if n else None
    out = torch.full_like(q, float("nan"))
    pa.pa_decode_ext(out, q, k, v, bt, cl, scale, kc.shape[1], maxlen, q_len, window, k_scale, v_scale, P, ws)
    torch.cuda.synchronize()
    return out


# (group, q_len) pairs: every row capacity on both kernels, odd token counts
SHAPES = [(1, 1), (1, 3), (1, 4), (2, 2), (2, 8), (4, 1), (4, 3), (4, 4), (8, 2), (16, 1)]
LENS = [1, 2, 5, 15, 16, 17, 250, 513, 1100]


@pytest.mark.parametrize("window", [0, 37, 300])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("g,q_len", SHAPES)
def test_ext_16bit(orc, g, q_len, D, window):
    dtype = "bf16" if (g + q_len + D) % 2 else "f16"
    rng = np.random.default_rng(1000 + 37 * g + 7 * q_len + D + window)
    Hk = 2
    p = Paged(rng, LENS, Hk * g, Hk, D, dtype)
    q = rand_bits(rng, (len(LENS), q_len, Hk * g, D), dtype)
    scale = float(np.float32(1 / np.sqrt(D)))
    ref = orc.paged_decode_ext(q, p.k_cache, p.v_cache, p.tables, p.lens, scale, dtype, q_len, window)
    tables = poison_before_window(p.tables, LENS, q_len, window)
    for P in (0, 16, 1104):
        out = run_ext(q, p.k_cache, p.v_cache, tables, LENS, scale, dtype, q_len, window, P)
        compare(out, ref, dtype, f"g={g} q_len={q_len} D={D} W={window} P={P}")


@pytest.mark.parametrize("g,q_len", [(1, 2), (4, 2), (8, 2), (16, 1)])
@pytest.mark.parametrize("window", [0, 100])
def test_ext_fp8(orc, g, q_len, window):
    rng = np.random.default_rng(2000 + g * 10 + q_len + window)
    Hk, D = 2, 128
    p = Paged(rng, LENS, Hk * g, Hk, D, "f16")
    NB = p.k_cache.shape[0]
    kc = rng.integers(0, 256, size=(NB, Hk, 16, D), dtype=np.uint8)
    kc[(kc & 0x7F) == 0x7F] = 0x38
    kc[((kc >> 3) & 0xF) > 9] &= 0x87
    vc = np.roll(kc, 3, axis=0)
    q = rand_bits(rng, (len(LENS), q_len, Hk * g, D), "f16")
    ks, vs = float(np.float32(0.07)), float(np.float32(0.11))
    ref = orc.paged_decode_ext(q, kc, vc, p.tables, p.lens, 0.088, "f16", q_len, window, ks, vs)
    tables = poison_before_window(p.tables, LENS, q_len, window)
    for P in (0, 16):
        out = run_ext(q, kc, vc, tables, LENS, 0.088, "f16", q_len, window, P, ks, vs, kv8=True)
        compare(out, ref, "f16", f"fp8 g={g} q_len={q_len} W={window} P={P}")


@pytest.mark.parametrize("g", [1, 4])
def test_ext_scales_on_a_16bit_cache(orc, g):
    """k_scale / v_scale apply to 16-bit caches too (both kernels; the
    tensor-core one takes its masked variant for v_scale != 1)."""
    rng = np.random.default_rng(3000 + g)
    p = Paged(rng, LENS, 2 * g, 2, 128, "bf16")
    q = rand_bits(rng, (len(LENS), 1, 2 * g, 128), "bf16")
    ref = orc.paged_decode_ext(q, p.k_cache, p.v_cache, p.tables, p.lens, 0.09, "bf16", 1, 0, 2.5, 0.3)
    out = run_ext(q, p.k_cache, p.v_cache, p.tables, LENS, 0.09, "bf16", 1, 0, 0, 2.5, 0.3)
    compare(out, ref, "bf16", f"scaled g={g}")


@pytest.mark.parametrize("g", [1, 2, 4, 8, 16])
def test_ext_plain_options_equal_pa_decode_bit_for_bit(g):
    """q_len 1, no window, unit scales: the same kernels as pa_decode."""
    from paged_kv_cache_424_b200 import binding as pa
    rng = np.random.default_rng(4000 + g)
    p = Paged(rng, LENS, 2 * g, 2, 128, "f16")
    q = _dev16(p.q, "f16")
    k, v = _dev16(p.k_cache, "f16"), _dev16(p.v_cache, "f16")
    bt, cl = torch.from_numpy(p.tables).cuda(), torch.from_numpy(p.lens).cuda()
    dims = pa.dims_of(q, k, bt)
    n = pa.pa_decode_workspace_size(dims, 1100, 0)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda") if n else None
    a = torch.empty_like(q)
    pa.pa_decode(a, q, k, v, bt, cl, 0.1, 2, 1100, 0, ws)
    b = torch.empty_like(q)
    pa.pa_decode_ext(b[:, None], q[:, None], k, v, bt, cl, 0.1, 2, 1100, 1, 0, 1.0, 1.0, 0, ws)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_ext_window_one_returns_own_value():
    rng = np.random.default_rng(5000)
    p = Paged(rng, [3, 16, 17, 50], 8, 2, 128, "bf16")
    q = rand_bits(rng, (4, 3, 8, 128), "bf16")
    out = run_ext(q, p.k_cache, p.v_cache, poison_before_window(p.tables, p.lens, 3, 1), p.lens, 0.5, "bf16", 3,
                  1, 16)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    for s, L in enumerate(p.lens):
        for i in range(3):
            want = np.repeat(p.vs[s][L - 3 + i], 4, axis=0)
            assert np.array_equal(got[s, i], want), f"s={s} i={i}"


# ---------------------------------------------------------------------------
# workloads: speculative verification on the 8B shape, sliding window on the 70B shape
# ---------------------------------------------------------------------------
def test_spec8b_reduced():
    run_and_compare(W().spec8b(seed=61, num_seqs=12, num_blocks=4096))


def test_spec8b_full_sampled():
    sc = W().spec8b()
    seqs = np.sort(np.random.default_rng(62).choice(sc.dims.num_seqs, 12, replace=False))
    run_and_compare(sc, seqs=seqs)


def test_window70b_reduced():
    sc = W().window70b(seed=63, num_seqs=2, context_len=5000 + 3, window=700, num_blocks=1024)
    run_and_compare(sc)
    run_and_compare(sc, partition_tokens=16)


def test_window70b_full_sampled():
    sc = W().window70b()
    run_and_compare(sc, seqs=np.array([0, 5]))


def test_window70b_fp8_multi_token_reduced():
    sc = W().with_fp8_cache(W().window70b(seed=64, num_seqs=2, context_len=3000, window=257, q_len=2,
                                          num_blocks=1024))
    run_and_compare(sc)


# ---------------------------------------------------------------------------
# shared-prefix order (pa_prefix_order -> pa_decode_opts.seq_order)
# ---------------------------------------------------------------------------
def test_prefix8b_reduced_order_is_bit_identical_to_batch_order():
    import dataclasses
    from paged_kv_cache_424_b200.session import DeviceSession
    sc = W().prefix8b(seed=71, num_prompts=4, num_blocks=2048)
    run_and_compare(sc)                                   # in prefix order, against the oracle
    st = sc.steps[0]
    a = DeviceSession(sc).run_step(st)
    b = DeviceSession(dataclasses.replace(sc, prefix_order=False)).run_step(st)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)), "the schedule changed the results"


def test_prefix8b_full_sampled():
    sc = W().prefix8b()
    seqs = np.sort(np.random.default_rng(72).choice(sc.dims.num_seqs, 10, replace=False))
    run_and_compare(sc, seqs=seqs)


@pytest.mark.parametrize("g", [1, 4])
def test_seq_order_entry_outside_the_batch_is_skipped_and_flagged(g):
    from paged_kv_cache_424_b200 import binding as pa
    rng = np.random.default_rng(73 + g)
    p = Paged(rng, [40, 70, 300, 5], 2 * g, 2, 128, "f16")
    q = _dev16(p.q, "f16")[:, None]
    k, v = _dev16(p.k_cache, "f16"), _dev16(p.v_cache, "f16")
    bt, cl = torch.from_numpy(p.tables).cuda(), torch.from_numpy(p.lens).cuda()
    ref = torch.empty_like(q)
    pa.pa_decode_ext(ref, q, k, v, bt, cl, 0.1, 2, 300)
    order = torch.tensor([2, 0, 9, 1], dtype=torch.int32, device="cuda")   # 9 is not a sequence; 3 is missing
    out = torch.zeros_like(q)
    pa.pa_decode_ext(out, q, k, v, bt, cl, 0.1, 2, 300, seq_order=order)
    assert pa.pa_device_error() & 2, "out-of-range entry not flagged"
    for s in (0, 1, 2):
        assert torch.equal(out[s].view(torch.int16), ref[s].view(torch.int16))
    assert torch.all(out[3] == 0), "the skipped CTA row wrote something"


# ---------------------------------------------------------------------------
# several partitions per tensor-core CTA (partitions of 128-512 tokens on a
# grid of 512 (sequence, KV head) pairs, enough for the host to group them)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("P", [128, 256, 384, 512])
def test_several_partitions_per_tensor_core_cta(orc, P):
    from paged_kv_cache_424_b200 import binding as pa
    rng = np.random.default_rng(500 + P)
    S, Hk, g = 64, 8, 4
    lens = rng.integers(1, 2001, size=S)
    lens[:4] = [1, 127, 128, 129]
    p = Paged(rng, lens, Hk * g, Hk, 128, "bf16")
    scale = 0.088
    ref = p.run(orc, scale)
    q = _dev16(p.q, "bf16")
    k, v = _dev16(p.k_cache, "bf16"), _dev16(p.v_cache, "bf16")
    bt, cl = torch.from_numpy(p.tables).cuda(), torch.from_numpy(p.lens).cuda()
    maxlen = int(lens.max())
    dims = pa.dims_of(q, k, bt)
    n = pa.pa_decode_workspace_size(dims, maxlen, P)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda") if n else None
    out = torch.full_like(q, float("nan"))
    pa.pa_decode(out, q, k, v, bt, cl, scale, Hk, maxlen, P, ws)
    torch.cuda.synchronize()
    compare(out, ref, "bf16", f"P={P}")
    # masked: 2 query tokens and a window, same grouping
    q2 = rand_bits(rng, (S, 2, Hk * g, 128), "bf16")
    ref2 = orc.paged_decode_ext(q2, p.k_cache, p.v_cache, p.tables, p.lens, scale, "bf16", 2, 700)
    tables = poison_before_window(p.tables, lens, 2, 700)
    out2 = run_ext(q2, p.k_cache, p.v_cache, tables, lens, scale, "bf16", 2, 700, P)
    compare(out2, ref2, "bf16", f"masked P={P}")
