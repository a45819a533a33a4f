"""The library's calls capture into CUDA graphs ("vLLM 深度解析：PagedAttention
如何让大模型推理更快、更省钱", 生产环境部署的专业建议: CUDA graphs at small
batch): they allocate nothing and never synchronise, so a decode step
(cache write + decode + merge) recorded once replays with results bit-equal
to the eager calls, on both decode kernels, over FP8 caches and through
pa_decode_ext and pa_decode_noalloc."""
import numpy as np
import pytest
import torch

from gpu_util import compare, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    from paged_kv_cache_424_b200 import build
    build.build()
    from paged_kv_cache_424_b200 import binding
    assert binding.pa_device_error() == 0
    yield
    assert binding.pa_device_error() == 0


def W():
    from paged_kv_cache_424_b200 import workload
    return workload


def _scenarios():
    w = W()
    return {
        "mha-cuda-cores": w.mha7b(seed=81, num_seqs=8, min_len=100, max_len=1500, num_blocks=1024),
        "gqa-tensor-cores": w.gqa8b(seed=82, num_seqs=16, median=300, cap=2500, num_blocks=4096),
        "gqa-fp8": w.with_fp8_cache(w.gqa8b(seed=83, num_seqs=8, median=300, cap=2500, num_blocks=2048)),
        "spec-ext": w.spec8b(seed=84, num_seqs=8, num_blocks=2048),
    }


@pytest.mark.parametrize("name", ["mha-cuda-cores", "gqa-tensor-cores", "gqa-fp8", "spec-ext"])
def test_decode_step_replays_from_a_cuda_graph(name, orc):
    from oracle.harness import OracleSession
    from paged_kv_cache_424_b200.session import DeviceSession
    sc = _scenarios()[name]
    st = sc.steps[0]
    dev = DeviceSession(sc)
    dev.apply_cache_ops(st)
    inp = dev.decode_inputs(st)
    writes = dev.write_inputs(st)
    eager = dev.decode(st, 0, inputs=inp)                  # sizes and allocates the workspace
    torch.cuda.synchronize()
    out = torch.empty_like(eager)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for key, value, slots in writes:                    # idempotent: same slots, same values
            dev.write(key, value, slots)
        dev.decode(st, 0, inputs=inp, out=out)
    for _ in range(3):
        out.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16)), "graph replay differs from eager"
    ref = OracleSession(sc).run_step(st)
    compare(out, ref, sc.dims.dtype, f"{name} (graph)")


def test_noalloc_decode_replays_from_a_cuda_graph():
    from paged_kv_cache_424_b200 import binding as pa
    from paged_kv_cache_424_b200.session import DeviceSession
    sc = W().mha7b(seed=85, num_seqs=8, min_len=600, max_len=2000, num_blocks=1024)
    st = sc.steps[0]
    dev = DeviceSession(sc)
    dev.apply_cache_ops(st)
    inp = dev.decode_inputs(st)
    maxlen = st.max_context_len
    eager = torch.empty_like(inp["q"])
    args = (inp["q"], dev.k_cache, dev.v_cache, inp["block_tables"], inp["context_lens"], sc.scale,
            sc.dims.num_kv_heads, maxlen)
    pa.pa_decode_noalloc(eager, *args)                      # first call on the device: looks up the scratch
    torch.cuda.synchronize()
    out = torch.empty_like(eager)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        pa.pa_decode_noalloc(out, *args)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
