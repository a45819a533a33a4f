"""GPU parity of the FP8 E4M3 KV cache (the "FP8" reading of the pages'
KV-cache compression goal, vLLM PagedAttention 大模型推理架构深度实战 section 九
item 3): the quantising cache write bit for bit against the oracle, and
decode over E4M3 codes with per-tensor scales within the 16-bit path's
tolerances (the codes widen exactly, so the error sources are the same).
"""
import numpy as np
import pytest
import torch

from gpu_util import compare, require_gpu, run_and_compare

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


def _dev16(bits: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(TORCH[dtype])


def _is_nan16(bits: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f16":
        return ((bits & 0x7C00) == 0x7C00) & ((bits & 0x03FF) != 0)
    return ((bits & 0x7F80) == 0x7F80) & ((bits & 0x007F) != 0)


# ---------------------------------------------------------------------------
# cache write: every 16-bit input, bit for bit
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D,Hk", [(128, 1), (64, 2)])
@pytest.mark.parametrize("scales", [(1.0, 1.0), (0.0123, 0.0071), (3.7, 0.25)])
def test_cache_write_every_16bit_value(orc, dtype, D, Hk, scales):
    """All 65536 bit patterns (zeros, subnormals, ties, values past 448 x
    scale, infinities, NaNs) as keys, reversed as values, into shuffled
    slots.  Finite and infinite inputs must give the oracle's code exactly;
    NaN inputs a NaN code (0x7F or 0xFF: the sign of a NaN is not defined)."""
    from paged_kv_cache_424_b200 import binding as pa
    ks, vs = (float(np.float32(x)) for x in scales)
    rng = np.random.default_rng(41)
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    T = 65536 // (Hk * D)
    key = allbits.reshape(T, Hk, D)
    val = allbits[::-1].copy().reshape(T, Hk, D)
    NB = 2 * T // 16
    slots = rng.permutation(NB * 16)[:T].astype(np.int64)
    slots[rng.random(T) < 0.02] = -1                       # padding tokens: skipped
    kc = torch.full((NB, Hk, 16, D), 0x7F, dtype=torch.uint8, device="cuda")
    vc = torch.full_like(kc, 0x7F)
    pa.pa_reshape_and_cache_fp8(_dev16(key, dtype), _dev16(val, dtype), kc, vc,
                                torch.from_numpy(slots).cuda(), ks, vs)
    torch.cuda.synchronize()
    ek = np.full((NB, Hk, 16, D), 0x7F, np.uint8)
    ev = ek.copy()
    orc.reshape_and_cache_fp8(ek, ev, key, val, slots, dtype, ks, vs)
    for name, got, want, src in (("K", kc, ek, key), ("V", vc, ev, val)):
        got = got.cpu().numpy()
        # the input element each cache byte came from (NaN there -> any NaN code)
        nanin = np.zeros(want.shape, bool)
        live = slots >= 0
        b, o = slots[live] // 16, slots[live] % 16
        nanin[b, :, o, :] = _is_nan16(src[live], dtype)
        exact = ~nanin
        bad = np.argwhere(exact & (got != want))
        assert bad.size == 0, (f"{name}: {len(bad)} codes differ, first at {bad[0].tolist()}: "
                               f"got {got[tuple(bad[0])]:#x} want {want[tuple(bad[0])]:#x}")
        assert np.all((got[nanin] & 0x7F) == 0x7F), f"{name}: a NaN input did not give a NaN code"


# ---------------------------------------------------------------------------
# decode over FP8 caches: every built group size and head_dim
# ---------------------------------------------------------------------------
def random_codes(rng, shape, max_exp_field: int = 9) -> np.ndarray:
    """Random E4M3 codes without NaN, magnitudes below 2^(max_exp_field-6)."""
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38
    big = ((c >> 3) & 0xF) > max_exp_field
    c[big] &= 0x87
    return c


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("g", [1, 2, 4, 8, 16])
def test_fp8_group_sizes_and_head_dims(orc, dtype, D, g):
    from paged_kv_cache_424_b200 import binding as pa
    rng = np.random.default_rng(300 + g + D)
    Hk = 2
    H = Hk * g
    lens = np.array([1, 15, 16, 17, 250, 513, 1100], np.int32)
    S, MB = len(lens), 72
    NB = S * MB + 8
    kc, vc = random_codes(rng, (NB, Hk, 16, D)), random_codes(rng, (NB, Hk, 16, D))
    tables = rng.permutation(NB)[:S * MB].reshape(S, MB).astype(np.int32)
    qf = (rng.random((S, H, D), dtype=np.float32) * 2 - 1)
    q = _dev16(qf.astype(np.float16).view(np.uint16), "f16") if dtype == "f16" else \
        torch.from_numpy(qf).cuda().to(torch.bfloat16)
    qbits = q.view(torch.int16).cpu().numpy().view(np.uint16)
    ks, vs = float(np.float32(0.09)), float(np.float32(0.13))
    scale = float(np.float32(1 / np.sqrt(D)))
    ref = orc.paged_decode_fp8(qbits, kc, vc, tables, lens, scale, ks, vs, dtype)
    dk, dv = torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda()
    bt, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    for P in (0, 16, 1104):
        dims = pa.dims_of(q, dk, bt)
        n = pa.pa_decode_workspace_size(dims, 1100, P)
        ws = torch.empty(n, dtype=torch.uint8, device="cuda") if n else None
        out = torch.full_like(q, float("nan"))
        pa.pa_decode_fp8(out, q, dk, dv, bt, cl, scale, ks, vs, Hk, 1100, P, ws)
        torch.cuda.synchronize()
        compare(out, ref, dtype, f"fp8 g={g} D={D} P={P}")


@pytest.mark.parametrize("shift", [20, -30])
@pytest.mark.parametrize("g,q_len", [(4, 1), (8, 1), (16, 1), (4, 4)])
def test_fp8_bf16_q_beyond_f16_range(orc, shift, g, q_len):
    """bf16 queries whose every element lies above f16's largest finite value
    (magnitudes in [0.5, 1) x 2^20) or below its smallest normal (x 2^-30),
    with the softmax scale divided by the same power of two so the logits
    are those of O(1) queries.  The tensor-core FP8 products carry q as E4M3
    parts under a per-row power of two, so such a q must give the oracle's
    result on every row count: groups 4, 8, 16 and group 4 x 4 query tokens
    (16 columns, pa_decode_ext)."""
    from paged_kv_cache_424_b200 import binding as pa
    rng = np.random.default_rng(600 + 10 * g + q_len + shift)
    Hk, D = 2, 128
    H = Hk * g
    lens = np.array([q_len, 17, 250, 1100], np.int32)
    S, MB = len(lens), 72
    NB = S * MB + 8
    kc, vc = random_codes(rng, (NB, Hk, 16, D)), random_codes(rng, (NB, Hk, 16, D))
    tables = rng.permutation(NB)[:S * MB].reshape(S, MB).astype(np.int32)
    mag = rng.random((S, q_len, H, D), dtype=np.float32) * 0.5 + 0.5
    sign = np.where(rng.random((S, q_len, H, D)) < 0.5, -1.0, 1.0).astype(np.float32)
    q4 = torch.from_numpy(mag * sign * np.float32(2.0 ** shift)).cuda().to(torch.bfloat16)
    qa = q4.float().abs()
    assert bool((qa > 65504).all()) if shift > 0 else bool((qa < 2.0 ** -14).all() and (qa > 0).all())
    qbits = q4.view(torch.int16).cpu().numpy().view(np.uint16)
    ks, vs = float(np.float32(0.09)), float(np.float32(0.13))
    scale = float(np.float32(np.float32(1 / np.sqrt(D)) * np.float32(2.0 ** -shift)))
    dk, dv = torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda()
    bt, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    maxlen = int(lens.max())
    if q_len == 1:
        ref = orc.paged_decode_fp8(qbits[:, 0], kc, vc, tables, lens, scale, ks, vs, "bf16")
        q = q4[:, 0].contiguous()
    else:
        ref = orc.paged_decode_ext(qbits, kc, vc, tables, lens, scale, "bf16", q_len, 0, ks, vs)
        q = q4
    for P in (0, 16):
        out = torch.full_like(q, float("nan"))
        if q_len == 1:
            n = pa.pa_decode_workspace_size(pa.dims_of(q, dk, bt), maxlen, P)
            ws = torch.empty(n, dtype=torch.uint8, device="cuda") if n else None
            pa.pa_decode_fp8(out, q, dk, dv, bt, cl, scale, ks, vs, Hk, maxlen, P, ws)
        else:
            opts = pa.pa_decode_opts(q_len, 0, ks, vs)
            n = pa.pa_decode_ext_workspace_size(pa.ext_dims(q, dk, bt), opts, maxlen, P)
            ws = torch.empty(n, dtype=torch.uint8, device="cuda") if n else None
            pa.pa_decode_ext(out, q, dk, dv, bt, cl, scale, Hk, maxlen, q_len, 0, ks, vs, P, ws)
        torch.cuda.synchronize()
        compare(out, ref, "bf16", f"fp8 bf16 q x 2^{shift} g={g} q_len={q_len} P={P}")


# ---------------------------------------------------------------------------
# decode over FP8 caches: the workloads at reduced and full sizes
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("P", [0, 16, 64])
def test_tiny_fp8(P):
    run_and_compare(W().with_fp8_cache(W().tiny(0)), partition_tokens=P)


@pytest.mark.parametrize("P", [0, 16, 512, 2048])
def test_mha7b_reduced_fp8(P):
    sc = W().mha7b(seed=51, num_seqs=6, min_len=1, max_len=1500, num_blocks=1024)
    run_and_compare(W().with_fp8_cache(sc), partition_tokens=P)


def test_gqa8b_reduced_three_steps_fp8():
    sc = W().gqa8b(seed=52, num_seqs=24, num_steps=3, median=128, cap=1200, new_min=1, new_max=200,
                   num_blocks=8192)
    run_and_compare(W().with_fp8_cache(sc))


def test_long70b_reduced_fp8():
    sc = W().with_fp8_cache(W().long70b(seed=53, num_seqs=1, context_len=4096 + 7, num_blocks=512))
    run_and_compare(sc)
    run_and_compare(sc, partition_tokens=16)


def test_grouped_partitions_fp8():
    """Over an FP8 cache a CTA groups partitions up to 4096 tokens into one
    partial: 64 sequences of up to 2048 tokens at 512-token partitions."""
    sc = W().gqa8b(seed=72, num_seqs=64, num_steps=1, median=1500, cap=2048, num_blocks=16384)
    run_and_compare(W().with_fp8_cache(sc), partition_tokens=512)


def test_long70b_full_fp8_sampled():
    """The 70B long-context batch at its stated 512-token partitions over an
    FP8 cache (four partitions per CTA, one partial each): two sequences
    checked against the oracle."""
    run_and_compare(W().with_fp8_cache(W().long70b()), seqs=np.array([0, 5]))


def test_cow_reduced_fp8():
    """Copy-on-write copies move FP8 blocks (half the bytes of a 16-bit one)."""
    sc = W().with_fp8_cache(W().cow(seed=54, num_prompts=2, num_blocks=1024))
    assert sc.steps[0].block_mapping.size
    run_and_compare(sc)


def test_positive_values_fp8():
    sc = W().mha7b(seed=55, num_seqs=4, min_len=1, max_len=2048, num_blocks=1024, v_lo=0.0)
    run_and_compare(W().with_fp8_cache(sc))


def test_mha7b_full_fp8_sampled():
    """The benchmark's 64-sequence batch and launch configuration over an FP8
    cache; every written block compared, decode checked on 8 sequences."""
    sc = W().with_fp8_cache(W().mha7b())
    rng = np.random.default_rng(56)
    seqs = np.sort(rng.choice(sc.dims.num_seqs, 8, replace=False))
    run_and_compare(sc, seqs=seqs)


def test_power_of_two_scales_match_16bit_decode_of_widened_codes(orc):
    """With scales 1, decode of E4M3 codes equals the 16-bit decode of the
    same values written as fp16 (every E4M3 value is exact in fp16): the two
    GPU paths agree within the tolerance, and each agrees with the oracle."""
    from paged_kv_cache_424_b200 import binding as pa
    rng = np.random.default_rng(57)
    S, H, Hk, D, NB = 4, 8, 2, 128, 64
    codes = rng.integers(0, 256, size=(NB, Hk, 16, D), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38                     # no NaN codes (0x38 = 1.0)
    codes = np.where((codes & 0x78) > 0x48, codes & 0x87, codes).astype(np.uint8)  # keep |x| < 8
    vcodes = np.roll(codes, 1, axis=0)
    widened = orc.widen_e4m3(codes).astype(np.float16).view(np.uint16)
    vwidened = orc.widen_e4m3(vcodes).astype(np.float16).view(np.uint16)
    lens = np.array([1, 200, 513, 1000], np.int32)
    MB = 64
    tables = np.stack([rng.permutation(NB)[:MB] for _ in range(S)]).astype(np.int32)
    q = (rng.random((S, H, D), dtype=np.float32) * 2 - 1).astype(np.float16)
    dq = torch.from_numpy(q).cuda()
    bt, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    scale = 0.05
    k8, v8 = torch.from_numpy(codes).cuda(), torch.from_numpy(vcodes).cuda()
    k16, v16 = _dev16(widened, "f16"), _dev16(vwidened, "f16")
    for P in (0, 16):
        o8 = torch.empty_like(dq)
        o16 = torch.empty_like(dq)
        dims8 = pa.dims_of(dq, k8, bt)
        dims16 = pa.dims_of(dq, k16, bt)
        n8 = pa.pa_decode_workspace_size(dims8, 1000, P)
        n16 = pa.pa_decode_workspace_size(dims16, 1000, P)
        ws8 = torch.empty(max(n8, 1), dtype=torch.uint8, device="cuda")
        ws16 = torch.empty(max(n16, 1), dtype=torch.uint8, device="cuda")
        pa.pa_decode_fp8(o8, dq, k8, v8, bt, cl, scale, 1.0, 1.0, Hk, 1000, P, ws8 if n8 else None)
        pa.pa_decode(o16, dq, k16, v16, bt, cl, scale, Hk, 1000, P, ws16 if n16 else None)
        torch.cuda.synchronize()
        ref = orc.paged_decode_fp8(q.view(np.uint16), codes, vcodes, tables, lens, scale, 1.0, 1.0, "f16")
        compare(o8, ref, "f16", f"fp8 decode P={P}")
        compare(o16, ref, "f16", f"16-bit decode of the widened codes P={P}")
        assert float((o8.float() - o16.float()).abs().max()) <= 2e-3


def test_float8_dtype_tensors_accepted():
    """torch.float8_e4m3fn caches are the same bytes as uint8 ones."""
    from paged_kv_cache_424_b200 import binding as pa
    rng = np.random.default_rng(58)
    key = (rng.random((20, 2, 64), dtype=np.float32) - 0.5).astype(np.float16)
    a = torch.full((4, 2, 16, 64), 0x7F, dtype=torch.uint8, device="cuda")
    b = torch.full_like(a, 0x7F).view(torch.float8_e4m3fn)
    slots = torch.arange(20, dtype=torch.int64, device="cuda")
    dk = torch.from_numpy(key).cuda()
    pa.pa_reshape_and_cache_fp8(dk, dk, a, a.clone(), slots, 0.01, 0.01)
    pa.pa_reshape_and_cache_fp8(dk, dk, b, b.clone(), slots, 0.01, 0.01)
    torch.cuda.synchronize()
    assert torch.equal(a, b.view(torch.uint8))
    # and torch's own conversion agrees with the cache write inside E4M3's range
    ref = (dk.float() / torch.tensor(0.01, dtype=torch.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    for t in range(20):
        assert torch.equal(a[t // 16, :, t % 16, :], ref[t]), f"token {t}"


def test_swap_fp8_pools_round_trip(orc):
    from paged_kv_cache_424_b200 import binding as pa
    rng = np.random.default_rng(59)
    NBd, NBh, Hk, D = 64, 24, 8, 128
    dk = rng.integers(0, 256, (NBd, Hk, 16, D), dtype=np.uint8)
    dv = rng.integers(0, 256, (NBd, Hk, 16, D), dtype=np.uint8)
    dev_k, dev_v = torch.from_numpy(dk).cuda(), torch.from_numpy(dv).cuda()
    host_k = torch.zeros((NBh, Hk, 16, D), dtype=torch.uint8).pin_memory()
    host_v = torch.zeros((NBh, Hk, 16, D), dtype=torch.uint8).pin_memory()
    pairs = np.stack([rng.choice(NBd, 20, replace=False), rng.choice(NBh, 20, replace=False)], 1).astype(np.int64)
    pa.pa_swap_blocks(dev_k, dev_v, host_k, host_v, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    hk = np.zeros((NBh, Hk, 16, D // 2), np.uint16)
    hv = np.zeros_like(hk)
    orc.swap_blocks(hk, hv, dk.view(np.uint16).copy(), dv.view(np.uint16).copy(), pairs)
    assert np.array_equal(host_k.numpy(), hk.view(np.uint8)) and np.array_equal(host_v.numpy(), hv.view(np.uint8))
