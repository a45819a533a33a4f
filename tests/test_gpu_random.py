"""Seeded random configurations against the oracle: dtype, head_dim, group,
query tokens, window, partition size, 16-bit or FP8 cache and ragged
lengths drawn together, so combinations that no hand-written case covers
still meet the oracle within the tolerances of gpu_util."""
import numpy as np
import pytest
import torch

from gpu_util import compare, require_gpu
from pins import Paged, rand_bits

pytestmark = pytest.mark.gpu

TORCH = {"f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    from paged_kv_cache_424_b200 import build
    build.build()
    from paged_kv_cache_424_b200 import binding
    assert binding.pa_device_error() == 0
    yield
    assert binding.pa_device_error() == 0, "a kernel flagged a device error"


def _dev16(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(TORCH[dtype])


def _codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38
    c[((c >> 3) & 0xF) > 9] &= 0x87
    return c


def _config(seed):
    rng = np.random.default_rng(9000 + seed)
    dtype = ["f16", "bf16"][rng.integers(2)]
    D = [64, 128][rng.integers(2)]
    g = [1, 2, 4, 8, 16][rng.integers(5)]
    q_len = int(rng.integers(1, 16 // g + 1)) if rng.random() < 0.5 else 1
    window = [0, 0, int(rng.integers(1, 600))][rng.integers(3)]
    P = [0, 0, 16 * int(rng.integers(1, 80))][rng.integers(3)]
    fp8 = bool(rng.random() < 0.3)
    Hk = int(rng.integers(1, 4))
    S = int(rng.integers(1, 7))
    lens = rng.integers(0, 2500, size=S)
    lens[rng.random(S) < 0.2] = rng.integers(0, 20)
    return rng, dtype, D, g, q_len, window, P, fp8, Hk, lens.astype(np.int64)


@pytest.mark.parametrize("seed", range(160))
def test_random_configuration(orc, seed):
    from paged_kv_cache_424_b200 import binding as pa
    rng, dtype, D, g, q_len, window, P, fp8, Hk, lens = _config(seed)
    H = Hk * g
    what = f"{dtype} D={D} g={g} q_len={q_len} W={window} P={P} fp8={fp8} Hk={Hk} lens={lens.tolist()}"
    p = Paged(rng, lens, H, Hk, D, dtype)
    q = rand_bits(rng, (len(lens), q_len, H, D), dtype)
    scale = float(np.float32(1 / np.sqrt(D)))
    ks, vs = (float(np.float32(0.07)), float(np.float32(0.11))) if fp8 else (1.0, 1.0)
    if fp8:
        kc, vc = _codes(rng, p.k_cache.shape), _codes(rng, p.v_cache.shape)
    else:
        kc, vc = p.k_cache, p.v_cache
    ref = orc.paged_decode_ext(q, kc, vc, p.tables, p.lens, scale, dtype, q_len, window, ks, vs)
    dq = _dev16(q, dtype)
    dk = torch.from_numpy(kc).cuda() if fp8 else _dev16(kc, dtype)
    dv = torch.from_numpy(vc).cuda() if fp8 else _dev16(vc, dtype)
    bt, cl = torch.from_numpy(p.tables).cuda(), torch.from_numpy(p.lens).cuda()
    maxlen = int(lens.max())
    dims = pa.ext_dims(dq, dk, bt)
    n = pa.pa_decode_ext_workspace_size(dims, pa.pa_decode_opts(q_len, window, ks, vs), maxlen, P)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda") if n else None
    out = torch.full_like(dq, float("nan"))
    pa.pa_decode_ext(out, dq, dk, dv, bt, cl, scale, Hk, maxlen, q_len, window, ks, vs, P, ws)
    torch.cuda.synchronize()
    compare(out, ref, dtype, what)
