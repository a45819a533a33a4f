"""The C-ABI library: it builds, loads, exports every function include/pa.h
declares, and rejects bad arguments on the host (no GPU needed: every call
here returns before anything is enqueued)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_424_b200 import build
    build.build()
    from paged_kv_cache_424_b200 import binding
    return binding


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(pa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("pa_decode", "pa_reshape_and_cache", "pa_copy_blocks", "pa_decode_workspace_size",
              "pa_last_error", "pa_device_error"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(so, n)]
    assert not missing, f"declared but not exported: {missing}"
    assert sorted(lib.EXPORTS) == declared_functions()


def test_version(lib):
    assert lib.pa_version() >= 100


def _dims(lib, **kw):
    base = dict(num_seqs=4, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16, max_blocks_per_seq=256,
                num_blocks=1024, dtype=lib.PA_BF16)
    base.update(kw)
    return lib.pa_dims(**base)


def test_workspace_plan(lib):
    # group 1 (CUDA-core kernel): automatic 512-token partitions
    d1 = _dims(lib, num_heads=8)
    assert lib.pa_decode_num_partitions(d1, 512, 0) == 1
    assert lib.pa_decode_workspace_size(d1, 512, 0) == 0
    assert lib.pa_decode_num_partitions(d1, 513, 0) == 2
    assert lib.pa_decode_num_partitions(d1, 4096, 0) == 8
    # group 4 at head_dim 128 (tensor-core kernel): automatic 1024-token partitions
    d = _dims(lib)
    assert lib.pa_decode_num_partitions(d, 1024, 0) == 1
    assert lib.pa_decode_workspace_size(d, 1024, 0) == 0
    assert lib.pa_decode_num_partitions(d, 1025, 0) == 2
    assert lib.pa_decode_num_partitions(d, 4096, 0) == 4
    ws = lib.pa_decode_workspace_size(d, 4096, 512)
    rows = 4 * 32 * 8
    assert ws >= rows * 128 * 4 + rows * 4
    # explicit partition sizes
    assert lib.pa_decode_num_partitions(d, 4096, 16) == 256
    assert lib.pa_decode_num_partitions(d, 4096, 4096) == 1
    assert lib.pa_decode_workspace_size(d, 4096, 4096) == 0
    assert lib.pa_decode_num_partitions(d, 0, 0) == 1
    # a batch that fills two waves of resident CTAs at 2048-token partitions
    # takes them (148 SMs x 3 CTAs when no device answers)
    big = _dims(lib, num_seqs=256)
    assert lib.pa_decode_num_partitions(big, 4096, 0) == 2
    assert lib.pa_decode_num_partitions(_dims(lib, num_seqs=256, max_blocks_per_seq=512), 4097, 0) == 3
    # over an FP8 cache up to 4096 tokens
    f8 = lib.PA_FP8_E4M3
    assert lib.pa_decode_num_partitions(_dims(lib, num_seqs=256, kv_dtype=f8), 4096, 0) == 1
    assert lib.pa_decode_num_partitions(_dims(lib, num_seqs=256, kv_dtype=f8, max_blocks_per_seq=512), 8192, 0) == 2
    assert lib.pa_decode_num_partitions(_dims(lib, num_seqs=32, kv_dtype=f8, max_blocks_per_seq=512), 8192, 0) == 4
    # and for 16 query rows per KV head (two CTAs per SM)
    assert lib.pa_decode_num_partitions(_dims(lib, num_seqs=256, num_heads=128), 4096, 0) == 1
    assert lib.pa_decode_num_partitions(_dims(lib, num_seqs=16), 4096, 0) == 4  # 256 CTAs at 2048: 1024
    assert lib.pa_decode_num_partitions(_dims(lib, num_seqs=256, num_heads=8), 4096, 0) == 8  # CUDA-core: 512


def test_plan_is_consistent_over_random_shapes(lib):
    """For random batches, lengths, groups, cache types and partition
    sizes: the workspace is zero exactly when the plan has one partition,
    and otherwise holds an fp32 row of head_dim values and an lse for every
    (query row, partition); automatic partitions never split the longest
    context into more pieces than 1024-token ones would (512-token ones on
    the CUDA-core kernel)."""
    import numpy as np
    rng = np.random.default_rng(2024)
    for _ in range(400):
        g = int(rng.choice([1, 2, 4, 8, 16]))
        hk = int(rng.choice([1, 2, 4, 8]))
        d = int(rng.choice([64, 128]))
        mb = int(rng.integers(1, 600))
        kv = int(rng.choice([0, lib.PA_FP8_E4M3]))
        dims = _dims(lib, num_seqs=int(rng.integers(1, 600)), num_heads=g * hk, num_kv_heads=hk, head_dim=d,
                     max_blocks_per_seq=mb, kv_dtype=kv)
        maxlen = int(rng.integers(0, mb * 16 + 1))
        P = int(rng.choice([0, 0, 16, 128, 512, 1024, 4096]))
        parts = lib.pa_decode_num_partitions(dims, maxlen, P)
        ws = lib.pa_decode_workspace_size(dims, maxlen, P)
        assert parts >= 1
        if parts == 1:
            assert ws == 0
        else:
            rows = dims.num_seqs * dims.num_heads * parts
            assert ws >= rows * d * 4 + rows * 4
        if P == 0 and maxlen > 0:
            assert parts <= -(-maxlen // 512) if (g < 4 or d != 128) else parts <= -(-maxlen // 1024)


@pytest.mark.parametrize("kw,status", [
    (dict(block_size=32), -4), (dict(head_dim=96), -4), (dict(num_heads=24, num_kv_heads=8), -4),
    (dict(num_heads=30), -3), (dict(dtype=7), -2), (dict(num_kv_heads=0), -3), (dict(num_seqs=-1), -3),
    (dict(num_seqs=70000), -3), (dict(kv_dtype=5), -2), (dict(dtype=0, kv_dtype=1), -2),
])
def test_bad_dims_rejected(lib, kw, status):
    d = _dims(lib, **kw)
    assert lib.LIB.pa_decode_num_partitions(ctypes.byref(d), 100, 0) == status
    assert lib.pa_last_error()


def test_fp8_cache_plan_follows_the_kernel(lib):
    # groups of 4+ at head_dim 128 take the tensor-core kernel (1024-token
    # partitions) over FP8 caches too; MHA and head_dim 64 the CUDA-core one (512)
    f8 = lib.PA_FP8_E4M3
    assert lib.pa_decode_num_partitions(_dims(lib, kv_dtype=f8), 1024, 0) == 1
    assert lib.pa_decode_num_partitions(_dims(lib, kv_dtype=f8), 4096, 0) == 4
    assert lib.pa_decode_num_partitions(_dims(lib, kv_dtype=f8, num_heads=8), 1024, 0) == 2
    assert lib.pa_decode_num_partitions(_dims(lib, kv_dtype=f8, head_dim=64), 1024, 0) == 2
    assert lib.pa_decode_num_partitions(_dims(lib, kv_dtype=lib.PA_BF16), 1024, 0) == 1


def test_ext_plan_and_workspace(lib):
    """Multi-token queries multiply the partial rows; a window bounds the
    partitions by the attended span, not by the longest context."""
    d = _dims(lib, num_heads=8)                      # group 1
    O = lib.pa_decode_opts
    plain = lib.pa_decode_workspace_size(d, 4096, 512)
    assert lib.pa_decode_ext_workspace_size(d, O(1, 0, 1.0, 1.0), 4096, 512) == plain
    ws4 = lib.pa_decode_ext_workspace_size(d, O(4, 0, 1.0, 1.0), 4096, 512)
    rows4 = 4 * 4 * 8 * 8                            # S x q_len x H x partitions of 512
    assert ws4 >= rows4 * 128 * 4 + rows4 * 4 and ws4 > plain
    # window 1000 + 3 extra query tokens: at most ceil(1003 / 16) + 1 = 64 blocks -> 2 partitions of 512
    wsw = lib.pa_decode_ext_workspace_size(d, O(4, 1000, 1.0, 1.0), 4096, 512)
    rowsw = 4 * 4 * 8 * 2
    assert rowsw * 128 * 4 <= wsw < ws4
    assert lib.pa_decode_ext_workspace_size(d, O(1, 100, 1.0, 1.0), 4096, 512) == 0  # one partition
    assert lib.LIB.pa_decode_ext_workspace_size(ctypes.byref(d), None, 100, 0) == ctypes.c_size_t(-1).value


def test_bad_partition_and_context(lib):
    d = _dims(lib)
    assert lib.LIB.pa_decode_num_partitions(ctypes.byref(d), 100, 24) == -3   # not a multiple of 16
    assert lib.LIB.pa_decode_num_partitions(ctypes.byref(d), 100, -16) == -3
    assert lib.LIB.pa_decode_num_partitions(ctypes.byref(d), 100, 65536) == -3
    assert lib.LIB.pa_decode_num_partitions(ctypes.byref(d), 4097, 0) == -3   # > max_blocks_per_seq * 16
    assert lib.LIB.pa_decode_num_partitions(ctypes.byref(d), -1, 0) == -3


# The checks below hand the library fake device pointers and expect it to
# reject every call on the host.  They run in a child process with no visible
# GPU, so even a call that wrongly passed validation could not reach a device.
HOST_CHECKS = r"""
import ctypes, sys
sys.path.insert(0, %(root)r)
from paged_kv_cache_424_b200 import binding as lib

def dims(**kw):
    base = dict(num_seqs=4, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                max_blocks_per_seq=256, num_blocks=1024, dtype=lib.PA_BF16)
    base.update(kw)
    return lib.pa_dims(**base)

def decode(d, ptrs, nkv=8, maxlen=2000, part=0, ws=None, wsb=0):
    out, q, k, v, bt, cl = ptrs
    return lib.LIB.pa_decode(out, q, k, v, bt, cl, ctypes.c_float(0.1), nkv, ctypes.byref(d), maxlen, part,
                             ws, wsb, None)

d = dims()
good = [ctypes.c_void_p(0x10000)] * 6
assert decode(d, [None] + good[1:]) == -1
assert decode(d, good, nkv=4) == -3
assert decode(d, good) == -5                      # 2000 tokens: split, no workspace
assert "workspace" in lib.pa_last_error()
assert decode(d, good, ws=ctypes.c_void_p(0x20000), wsb=16) == -5
assert decode(d, [ctypes.c_void_p(0x10008)] + good[1:], maxlen=100) == -7
assert decode(dims(num_seqs=0), [None] * 6) == 0  # empty batch: nothing to do
assert lib.LIB.pa_decode_noalloc(None, None, None, None, None, None, ctypes.c_float(0.1), 8,
                                 ctypes.byref(d), 100, 0, None) == -1

p = ctypes.c_void_p(0x10000)
L = lib.LIB
assert L.pa_reshape_and_cache(None, p, p, p, p, 4, ctypes.byref(d), None) == -1
assert L.pa_reshape_and_cache(p, p, p, p, p, -1, ctypes.byref(d), None) == -3
assert L.pa_reshape_and_cache(None, None, None, None, None, 0, ctypes.byref(d), None) == 0
assert L.pa_reshape_and_cache(ctypes.c_void_p(0x10004), p, p, p, p, 4, ctypes.byref(d), None) == -7
arr = (ctypes.c_void_p * 2)(0x10000, None)
assert L.pa_copy_blocks(ctypes.cast(arr, ctypes.c_void_p), ctypes.cast(arr, ctypes.c_void_p), 2, p, 3,
                        ctypes.byref(d), None) == -1
assert L.pa_copy_blocks(None, None, 0, None, 0, ctypes.byref(d), None) == 0
assert L.pa_copy_blocks(None, None, 1, p, -1, ctypes.byref(d), None) == -3
assert L.pa_device_error(None, None) == -1
assert L.pa_check_wait_timeout(0, None) == -3
assert L.pa_check_wait_timeout(3000, None) == -3

# FP8 E4M3 caches: entry point and kv_dtype must agree; scales must be positive
f8 = dims(kv_dtype=lib.PA_FP8_E4M3)
def decode_fp8(d, ptrs=good, ks=0.5, vs=0.5, maxlen=100):
    out, q, k, v, bt, cl = ptrs
    return L.pa_decode_fp8(out, q, k, v, bt, cl, ctypes.c_float(0.1), ctypes.c_float(ks), ctypes.c_float(vs), 8,
                           ctypes.byref(d), maxlen, 0, None, 0, None)
assert decode(f8, good, maxlen=100) == -2          # pa_decode on an FP8 cache
assert "pa_decode_fp8" in lib.pa_last_error()
assert decode_fp8(d) == -2                         # pa_decode_fp8 on a 16-bit cache
assert decode_fp8(f8, ks=0.0) == -3
assert decode_fp8(f8, vs=-1.0) == -3
assert decode_fp8(f8, ks=float("inf")) == -3
assert decode_fp8(f8, ks=float("nan")) == -3
assert decode_fp8(f8, maxlen=2000) == -5           # split, no workspace
assert decode_fp8(f8, ptrs=[None] + good[1:]) == -1
assert decode_fp8(f8, ptrs=[ctypes.c_void_p(0x10008)] + good[1:]) == -7
def rc8(d, key=p, ks=0.5, vs=0.5, n=4):
    return L.pa_reshape_and_cache_fp8(key, p, p, p, p, n, ctypes.byref(d), ctypes.c_float(ks), ctypes.c_float(vs),
                                      None)
assert rc8(d) == -2                                # 16-bit cache
assert L.pa_reshape_and_cache(p, p, p, p, p, 4, ctypes.byref(f8), None) == -2
assert rc8(f8, ks=0.0) == -3
assert rc8(f8, n=-1) == -3
assert rc8(f8, key=None) == -1
assert rc8(f8, key=ctypes.c_void_p(0x10004)) == -7
assert rc8(f8, key=None, n=0) == 0

# pa_decode_ext: options are checked before anything else
def ext(d, opts, ptrs=good, maxlen=100, ws=None, wsb=0):
    out, q, k, v, bt, cl = ptrs
    return L.pa_decode_ext(out, q, k, v, bt, cl, ctypes.c_float(0.1), 8, ctypes.byref(d),
                           ctypes.byref(opts) if opts is not None else None, maxlen, 0, ws, wsb, None)
O = lib.pa_decode_opts
assert ext(d, None) == -1
assert ext(d, O(0, 0, 1.0, 1.0)) == -3                 # q_len < 1
assert ext(d, O(1, -1, 1.0, 1.0)) == -3                # window < 0
assert ext(d, O(1, 0, 0.0, 1.0)) == -3                 # scale
assert ext(d, O(1, 0, 1.0, float("nan"))) == -3
assert ext(d, O(5, 0, 1.0, 1.0)) == -4                 # group 4 x 5 query tokens > 16
assert ext(d, O(4, 0, 1.0, 1.0), ptrs=[None] + good[1:]) == -1
assert ext(d, O(4, 0, 1.0, 1.0), maxlen=2000) == -5    # split, no workspace
assert ext(dims(num_seqs=0), O(2, 64, 1.0, 1.0), ptrs=[None] * 6) == 0
print("host checks ok")
"""


def test_host_argument_errors(lib):
    import subprocess
    import sys
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", HOST_CHECKS % {"root": ROOT}], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "host checks ok" in r.stdout
