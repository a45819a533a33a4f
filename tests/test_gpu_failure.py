"""Failure detection on the GPU without a fault: a pipeline wait that can
never complete gives up after its bound, flags PA_DEVERR_TIMEOUT in the
device error word, and leaves the context usable (a decode right after is
still correct)."""
import time

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


def test_wait_that_never_completes_gives_up_and_reports(orc):
    from paged_kv_cache_424_b200 import binding as pa
    assert pa.pa_device_error() == 0
    t0 = time.perf_counter()
    pa.pa_check_wait_timeout(50)
    word = pa.pa_device_error()            # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert word & 16, f"PA_DEVERR_TIMEOUT not set (word {word:#x})"
    assert elapsed < 5.0, f"the bounded wait took {elapsed:.2f} s"
    assert pa.pa_device_error() == 0, "reading the word clears it"
    # the context is still usable: a decode right after matches the oracle
    rng = np.random.default_rng(91)
    p = Paged(rng, [5, 300, 1200], 16, 4, 128, "bf16")
    dt = torch.bfloat16
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(dt)  # noqa: E731
    q, k, v = dev(p.q), dev(p.k_cache), dev(p.v_cache)
    bt, cl = torch.from_numpy(p.tables).cuda(), torch.from_numpy(p.lens).cuda()
    dims = pa.dims_of(q, k, bt)
    n = pa.pa_decode_workspace_size(dims, 1200, 0)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda") if n else None
    out = torch.empty_like(q)
    pa.pa_decode(out, q, k, v, bt, cl, 0.08, 4, 1200, 0, ws)
    assert pa.pa_device_error() == 0
    compare(out, p.run(orc, 0.08), "bf16", "decode after the timeout")


def test_timeout_bound_is_checked_on_the_host():
    from paged_kv_cache_424_b200 import binding as pa
    for bad in (0, -5, 5000):
        with pytest.raises(pa.PagedAttentionError):
            pa.pa_check_wait_timeout(bad)
