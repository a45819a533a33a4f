"""pa_decode_noalloc: decode attention for callers that cannot allocate.

Some callers cannot give pa_decode a workspace: an engine whose KV-cache pool
already holds nearly all device memory and forbids more allocations, a plugin
inside a framework whose memory pool it may not touch, or a path where
cudaMalloc's implicit synchronisation is not acceptable.  pa_decode_noalloc
takes no workspace and uses the library's own 64 MiB static device scratch.

These tests call it through the C ABI, on two calls in a row with different
shapes (the second call finds the first call's data still in the shared
scratch).  Each output must equal pa_decode's (with a caller workspace) bit
for bit, since both run the same plan through the same kernels and only the
scratch's address differs, so a stale partial or a wrong offset cannot hide
under a tolerance; and it must match the CPU oracle within the parity
tolerances.  A plan needing more than the scratch holds is refused before
anything is enqueued.  This file is collected last so that a
stop-at-first-failure run has run everything else.
"""
import numpy as np
import pytest
import torch

from gpu_util import compare, require_gpu
from pins import Paged

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    from paged_kv_cache_424_b200 import build
    build.build()


def _upload(p: Paged):
    dt = torch.float16 if p.dtype == "f16" else torch.bfloat16
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(dt)  # noqa: E731
    return dev(p.q), dev(p.k_cache), dev(p.v_cache), torch.from_numpy(p.tables).cuda(), \
        torch.from_numpy(p.lens).cuda()


def _both(p: Paged, scale: float, P: int):
    from paged_kv_cache_424_b200 import binding as pa
    q, k, v, bt, cl = _upload(p)
    maxlen = int(p.lens.max())
    dims = pa.dims_of(q, k, bt)
    need = pa.pa_decode_workspace_size(dims, maxlen, P)
    assert need > 0, "the case must use split-KV scratch"
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    ref = torch.full(q.shape, float("nan"), dtype=q.dtype, device="cuda")
    got = torch.full(q.shape, float("nan"), dtype=q.dtype, device="cuda")
    pa.pa_decode(ref, q, k, v, bt, cl, scale, p.Hk, maxlen, P, ws)
    pa.pa_decode_noalloc(got, q, k, v, bt, cl, scale, p.Hk, maxlen, P)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    return got, ref


def test_noalloc_matches_pa_decode_two_calls_in_a_row(orc):
    rng = np.random.default_rng(2024)
    first = Paged(rng, [3000, 17, 1200, 4097], 32, 8, 128, "bf16")
    got, ref = _both(first, 0.088, 0)
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), "call 1: differs from pa_decode"
    compare(got, first.run(orc, 0.088), "bf16", "noalloc call 1 vs the oracle")
    second = Paged(rng, [700, 2500, 33], 16, 16, 64, "f16")
    got, ref = _both(second, 0.125, 16)
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), "call 2: differs from pa_decode"
    compare(got, second.run(orc, 0.125), "f16", "noalloc call 2 vs the oracle")


def test_noalloc_refuses_a_plan_larger_than_its_scratch():
    from paged_kv_cache_424_b200 import binding as pa
    S, H, Hk, D, L = 64, 64, 8, 128, 32768
    dt = torch.bfloat16
    q = torch.zeros((S, H, D), dtype=dt, device="cuda")
    out = torch.zeros_like(q)
    k = torch.zeros((1, Hk, 16, D), dtype=dt, device="cuda")
    bt = torch.zeros((S, L // 16), dtype=torch.int32, device="cuda")
    cl = torch.full((S,), L, dtype=torch.int32, device="cuda")
    need = pa.pa_decode_workspace_size(pa.dims_of(q, k, bt), L, 512)
    assert need > 64 << 20
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_decode_noalloc(out, q, k, k, bt, cl, 0.1, Hk, L, 512)
    assert e.value.status == -5 and "scratch" in str(e.value)
    torch.cuda.synchronize()
    assert torch.all(out == 0), "a refused call must enqueue nothing"
