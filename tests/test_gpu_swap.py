"""swap_blocks on the GPU: device <-> page-locked host block copies
(preemption), bit-exact against the oracle, through the C ABI."""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import require_gpu
from pins import rand_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    from paged_kv_cache_424_b200 import build
    build.build()


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("map_on_device", [True, False])
def test_swap_out_and_in_round_trip(orc, map_on_device):
    from paged_kv_cache_424_b200 import binding as pa
    rng = np.random.default_rng(31)
    NBd, NBh, Hk, D = 96, 40, 8, 128
    dk = rand_bits(rng, (NBd, Hk, 16, D), "bf16")
    dv = rand_bits(rng, (NBd, Hk, 16, D), "bf16")
    dev_k = torch.from_numpy(dk.view(np.int16)).cuda().view(torch.bfloat16)
    dev_v = torch.from_numpy(dv.view(np.int16)).cuda().view(torch.bfloat16)
    host_k = torch.zeros((NBh, Hk, 16, D), dtype=torch.bfloat16).pin_memory()
    host_v = torch.zeros((NBh, Hk, 16, D), dtype=torch.bfloat16).pin_memory()
    out_pairs = np.stack([rng.choice(NBd, 30, replace=False), rng.choice(NBh, 30, replace=False)], 1)
    bm = torch.from_numpy(out_pairs.astype(np.int64))
    bm = bm.cuda() if map_on_device else bm.pin_memory()
    pa.pa_swap_blocks(dev_k, dev_v, host_k, host_v, bm)
    torch.cuda.synchronize()
    hk = np.zeros((NBh, Hk, 16, D), np.uint16)
    hv = np.zeros((NBh, Hk, 16, D), np.uint16)
    orc.swap_blocks(hk, hv, dk.copy(), dv.copy(), out_pairs)
    assert np.array_equal(_bits(host_k), hk) and np.array_equal(_bits(host_v), hv), "swap-out differs from oracle"
    # swap back in to fresh destination blocks
    in_pairs = np.stack([out_pairs[:, 1], rng.choice(NBd, 30, replace=False)], 1)
    bm2 = torch.from_numpy(in_pairs.astype(np.int64))
    bm2 = bm2.cuda() if map_on_device else bm2.pin_memory()
    pa.pa_swap_blocks(host_k, host_v, dev_k, dev_v, bm2)
    torch.cuda.synchronize()
    ek, ev = dk.copy(), dv.copy()
    orc.swap_blocks(ek, ev, hk, hv, in_pairs)
    assert np.array_equal(_bits(dev_k), ek) and np.array_equal(_bits(dev_v), ev), "swap-in differs from oracle"
    assert np.array_equal(ek[in_pairs[:, 1]], dk[out_pairs[:, 0]]), "round trip lost data"
    assert pa.pa_device_error() == 0


def test_swap_flags_bad_pairs_and_refuses_pageable_memory():
    from paged_kv_cache_424_b200 import binding as pa
    dev = torch.zeros((4, 2, 16, 64), dtype=torch.float16, device="cuda")
    host = torch.zeros((4, 2, 16, 64), dtype=torch.float16).pin_memory()
    bm = torch.tensor([[0, 1], [2, 9]], dtype=torch.int64, device="cuda")  # second pair is out of range
    dev[0] = 1.0
    pa.pa_swap_blocks(dev, dev, host, host, bm)
    assert pa.pa_device_error() & 8
    assert torch.all(host[1] == 1.0) and torch.all(host[[0, 2, 3]] == 0)
    pageable = torch.zeros((4, 2, 16, 64), dtype=torch.float16)  # not page-locked
    dims = pa.cache_dims(dev)
    st = pa.LIB.pa_swap_blocks(ctypes.c_void_p(dev.data_ptr()), ctypes.c_void_p(dev.data_ptr()), 4,
                               ctypes.c_void_p(pageable.data_ptr()), ctypes.c_void_p(pageable.data_ptr()), 4,
                               ctypes.c_void_p(bm.data_ptr()), 1, ctypes.byref(dims), None)
    assert st == -8, pa.pa_last_error()
    assert pa.pa_device_error() == 0
