"""Error bounds of the E4M3 part splits that the tensor-core kernel uses
over FP8 caches with 4 or 8 query rows per KV head.

The kernel multiplies the E4M3 codes as stored.  It carries each query row
as three E4M3 parts under a power-of-two factor, and each softmax weight as
four parts: x = sum_k part_k / 16^k.  These tests pin the bounds that the
C header states for those splits, using E4M3 rounding alone (the oracle's
round-to-nearest-even quantiser and exact decoder), in f32 arithmetic as
in the kernel:

* q: max |q - 2^-e sum_k part_k / 16^k| <= 2^-15 max |q| for any finite
  16-bit row, with no part clamped at 448;
* w in [0, 2^8] (the lazy running max bounds a weight by 2^8):
  |w - sum_k part_k / 16^k| <= 2^-12 w + 2^-22, with no part clamped.

The GPU parity tests check the kernel itself against the oracle.
"""
import numpy as np
import pytest
import torch

E4M3_MAX = 448.0


def _parts(orc, y: np.ndarray, nparts: int):
    """Split f32 values y into nparts E4M3 values; returns (parts, sum)."""
    y = y.astype(np.float32)
    parts, total, f = [], np.zeros(y.shape, np.float64), 1.0
    for _ in range(nparts):
        d = orc.widen_e4m3(orc.quantize_e4m3(y))
        parts.append(d)
        total += d * f
        y = ((y - d.astype(np.float32)) * np.float32(16.0)).astype(np.float32)  # exact in f32
        f /= 16.0
    return parts, total


def _query_rows(dtype):
    rng = np.random.default_rng(11)
    rows = []
    for scale in (1e-6, 1e-3, 0.05, 1.0, 30.0, 3e3):
        x = rng.standard_normal((16, 128)) * scale
        rows.append(x)
        rows.append(x * rng.standard_exponential((16, 128)) ** 3)  # heavy tails
        rows.append(x * (rng.random((16, 128)) < 0.05))            # mostly zero
    if dtype == torch.bfloat16:
        rows.append(rng.standard_normal((4, 128)) * 1e6)  # past f16's range
    q = torch.tensor(np.concatenate(rows)).to(dtype).float().numpy()
    keep = np.isfinite(q).all(axis=1) & (np.abs(q).max(axis=1) > 0)  # heavy tails overflow f16
    assert keep.sum() > 200
    return q[keep]


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
def test_query_split_three_parts(orc, dtype):
    for row in _query_rows(dtype):
        mx = float(np.abs(row).max())
        _, k = np.frexp(mx)  # mx in [2^(k-1), 2^k)
        e = 8 - int(k)
        y = np.ldexp(row, e).astype(np.float32)
        assert 128.0 <= np.abs(y).max() < 256.0
        parts, total = _parts(orc, y, 3)
        assert all(np.abs(p).max() < E4M3_MAX for p in parts)  # nothing clamped
        err = np.abs(np.ldexp(total, -e) - row.astype(np.float64)).max()
        assert err <= 2.0 ** -15 * mx, (err / mx, dtype)


def test_weight_split_four_parts(orc):
    rng = np.random.default_rng(12)
    w = np.exp2(rng.uniform(-60.0, 8.0, 400000)).astype(np.float32)
    edge = [0.0, 2.0 ** -30, 2.0 ** -10, 1.0, 255.9, 256.0, 240.0, 248.0]
    w = np.concatenate([w, np.array(edge, np.float32)])
    parts, total = _parts(orc, w, 4)
    assert all(np.abs(p).max() <= 256.0 for p in parts)  # nothing near the 448 clamp
    err = np.abs(total - w.astype(np.float64))
    assert np.all(err <= 2.0 ** -12 * w + 2.0 ** -22)
    # three parts would not meet the bound on small weights
    _, total3 = _parts(orc, w, 3)
    assert np.any(np.abs(total3 - w.astype(np.float64)) > 2.0 ** -12 * w + 2.0 ** -22)
