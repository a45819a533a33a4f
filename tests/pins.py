"""Pins that tie the CPU oracle to facts fixed outside itself.

Each ``pin_*`` takes an oracle handle (``oracle.Oracle``) and raises
``AssertionError`` (or ``oracle.OracleError``) when the oracle disagrees with:

* closed forms worked by hand for two-token and block-boundary cases,
* special cases (length 1 returns V; equal keys or a zero query give the mean
  of V; constant V gives that constant; length 0 gives zeros),
* invariants the pages state for paging: the result depends only on the
  logical order of blocks ("vLLM PagedAttention 大模型推理架构深度实战" §2.2,
  page-table analogy), and equals attention over the same keys/values laid
  out contiguously (scaled-dot-product attention from torch in float64, a
  library routine with its own GQA head mapping),
* GQA == MHA with every KV head repeated (group size g),
* a position-tagged case that proves the indirection: V encodes the logical
  position, one key dominates, the output must decode to that position,
* numerical stability at logits of thousands (max-subtracted softmax),
* the bit patterns of every finite fp16 / bf16 value, widened by numpy's own
  codecs,
* the cache writes and block copies against numpy's advanced indexing and
  slice assignment, including the copy-on-write guarantee that the other
  sharers' bytes stay as they were ("…深度实战" §2.3).

They are shared by ``test_oracle_pins.py`` (real oracle) and
``test_oracle_mutants.py`` (oracle builds with a planted mistake, each of which
must fail at least one pin).
"""
from __future__ import annotations

import math

import numpy as np
import torch

NAN = {"f16": 0x7E00, "bf16": 0x7FC0}


# ---------------------------------------------------------------------------
# helpers (independent of the oracle)
# ---------------------------------------------------------------------------
def widen(bits: np.ndarray, dtype: str) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    with np.errstate(invalid="ignore"):
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def narrow(x: np.ndarray, dtype: str) -> np.ndarray:
    t = torch.from_numpy(np.asarray(x, dtype=np.float32))
    t = t.to(torch.float16 if dtype == "f16" else torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def rand_bits(rng, shape, dtype, lo=-1.0, hi=1.0):
    return narrow(rng.uniform(lo, hi, size=shape), dtype)


class Paged:
    """A paged problem built from logical per-sequence K/V by this test's own
    scatter: ``cache[table[s, j // B], h, j % B, :] = K_s[j, h, :]``."""

    def __init__(self, rng, lens, H, Hk, D, dtype, B=16, NB=None, q=None, ks=None, vs=None,
                 v_lo=-1.0):
        self.lens = np.asarray(lens, dtype=np.int32)
        S = len(lens)
        nblk = [-(-int(L) // B) for L in lens]
        MB = max(1, max(nblk) if nblk else 1)
        need = sum(nblk) + 1
        NB = NB or need + 3
        self.B, self.H, self.Hk, self.D, self.dtype = B, H, Hk, D, dtype
        perm = rng.permutation(NB - 1)
        self.pad = NB - 1
        self.tables = np.full((S, MB), self.pad, dtype=np.int32)
        pos = 0
        for s, n in enumerate(nblk):
            self.tables[s, :n] = perm[pos:pos + n]
            pos += n
        self.k_cache = np.full((NB, Hk, B, D), NAN[dtype], dtype=np.uint16)
        self.v_cache = np.full((NB, Hk, B, D), NAN[dtype], dtype=np.uint16)
        self.q = q if q is not None else rand_bits(rng, (S, H, D), dtype)
        self.ks = ks if ks is not None else [rand_bits(rng, (int(L), Hk, D), dtype) for L in lens]
        self.vs = vs if vs is not None else [rand_bits(rng, (int(L), Hk, D), dtype, lo=v_lo)
                                             for L in lens]
        for s, L in enumerate(lens):
            j = np.arange(int(L))
            self.k_cache[self.tables[s, j // B], :, j % B, :] = self.ks[s]
            self.v_cache[self.tables[s, j // B], :, j % B, :] = self.vs[s]

    def run(self, orc, scale):
        return orc.paged_decode(self.q, self.k_cache, self.v_cache, self.tables, self.lens,
                                scale, self.dtype)


def sdpa(q_bits, k_bits, v_bits, scale, dtype):
    """torch float64 SDPA for one sequence: q [H, D], k/v [L, Hk, D]."""
    q = torch.from_numpy(widen(q_bits, dtype))[None, :, None, :]
    k = torch.from_numpy(widen(k_bits, dtype)).permute(1, 0, 2)[None]
    v = torch.from_numpy(widen(v_bits, dtype)).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale,
                                                         enable_gqa=q.shape[1] != k.shape[1])
    return o[0, :, 0, :].numpy()


def assert_close(a, b, tol, what):
    a = np.asarray(a)
    b = np.asarray(b)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    assert np.all(np.isfinite(a)), f"{what}: non-finite values"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------------------
# attention pins
# ---------------------------------------------------------------------------
def pin_two_token_closed_form(orc):
    """q = (1, .5), k0 = (1, 0), k1 = (0, 1), scale s: logits s and s/2, so
    out = (e^s v0 + e^{s/2} v1) / (e^s + e^{s/2})."""
    for dtype in ("f16", "bf16"):
        for scale in (1.0, 0.5):
            q = narrow(np.array([[[1.0, 0.5]]]), dtype)
            ks = [narrow(np.array([[[1.0, 0.0]], [[0.0, 1.0]]]), dtype)]
            vs = [narrow(np.array([[[1.0, 2.0]], [[-3.0, 0.25]]]), dtype)]
            p = Paged(np.random.default_rng(0), [2], 1, 1, 2, dtype, q=q, ks=ks, vs=vs)
            out = p.run(orc, scale)[0, 0]
            a, b = math.exp(scale), math.exp(scale / 2)
            want = [(a * 1.0 + b * -3.0) / (a + b), (a * 2.0 + b * 0.25) / (a + b)]
            assert_close(out, want, 1e-14, f"two-token closed form {dtype} scale {scale}")


def pin_block_boundary_closed_form(orc):
    """17 tokens over two blocks; keys are zero except token 16 (first slot of
    the second block) whose logit is x, so
    out = (sum_{j<16} v_j + e^x v_16) / (16 + e^x)."""
    dtype, D = "f16", 2
    q = narrow(np.array([[[2.0, 0.0]]]), dtype)
    k = np.zeros((17, 1, D))
    k[16, 0, 0] = 1.5
    v = np.zeros((17, 1, D))
    v[:, 0, 0] = np.arange(17) / 8.0
    v[:, 0, 1] = -1.0
    v[16, 0, 1] = 3.0
    p = Paged(np.random.default_rng(1), [17], 1, 1, D, dtype, q=q, ks=[narrow(k, dtype)],
              vs=[narrow(v, dtype)])
    out = p.run(orc, 1.0)[0, 0]
    x = 3.0
    ex = math.exp(x)
    want0 = (sum(j / 8.0 for j in range(16)) + ex * 2.0) / (16 + ex)
    want1 = (16 * -1.0 + ex * 3.0) / (16 + ex)
    assert_close(out, [want0, want1], 1e-14, "block-boundary closed form")


def pin_length_one_returns_v(orc):
    """One token: softmax weight is exactly 1, so out == V (bit-exact)."""
    rng = np.random.default_rng(2)
    for dtype in ("f16", "bf16"):
        p = Paged(rng, [1, 1, 1], 8, 2, 64, dtype)
        out = p.run(orc, 0.125)
        for s in range(3):
            want = widen(p.vs[s][0], dtype)  # [Hk, D]
            got = out[s].reshape(2, 4, 64)
            assert np.array_equal(got, np.broadcast_to(want[:, None, :], got.shape)), \
                f"length 1 must return V exactly ({dtype})"


def pin_equal_keys_give_mean(orc):
    """All keys equal: weights are uniform, out = mean of V over the context."""
    rng = np.random.default_rng(3)
    lens = [5, 16, 31]
    ks = []
    for L in lens:
        row = rand_bits(rng, (1, 2, 32), "bf16")
        ks.append(np.repeat(row, L, axis=0))
    p = Paged(rng, lens, 4, 2, 32, "bf16", ks=ks)
    out = p.run(orc, 0.3)
    for s, L in enumerate(lens):
        mean = widen(p.vs[s], "bf16").mean(axis=0)  # [Hk, D]
        assert_close(out[s], np.repeat(mean, 2, axis=0), 1e-13, "equal keys -> mean(V)")


def pin_zero_query_gives_mean(orc):
    rng = np.random.default_rng(4)
    lens = [3, 40]
    q = np.zeros((2, 2, 16), dtype=np.uint16)  # +0.0 in both formats
    p = Paged(rng, lens, 2, 1, 16, "f16", q=q)
    out = p.run(orc, 1.0)
    for s in range(2):
        mean = widen(p.vs[s], "f16").mean(axis=0)
        assert_close(out[s], np.repeat(mean, 2, axis=0), 1e-13, "zero query -> mean(V)")


def pin_constant_v(orc):
    rng = np.random.default_rng(5)
    lens = [7, 33]
    c = narrow(np.array([0.7109375]), "bf16")[0]
    vs = [np.full((L, 2, 16), c, dtype=np.uint16) for L in lens]
    p = Paged(rng, lens, 2, 2, 16, "bf16", vs=vs)
    out = p.run(orc, 0.25)
    assert_close(out, np.full(out.shape, 0.7109375), 1e-14, "constant V")


def pin_zero_length_gives_zeros(orc):
    rng = np.random.default_rng(6)
    p = Paged(rng, [0, 4], 2, 2, 8, "f16")
    out = p.run(orc, 1.0)
    assert np.array_equal(out[0], np.zeros((2, 8))), "context_len 0 must give zeros"
    assert np.all(np.isfinite(out[1]))


def pin_matches_contiguous_sdpa(orc):
    """Paged result == torch float64 SDPA on the logical (contiguous) K/V,
    at every block-count boundary (1, 16, 17, 32, 33) and a ragged 100."""
    rng = np.random.default_rng(7)
    for dtype, H, Hk in (("f16", 4, 4), ("bf16", 8, 2)):
        lens = [1, 16, 17, 32, 33, 100]
        p = Paged(rng, lens, H, Hk, 64, dtype)
        scale = 1.0 / 8.0
        out = p.run(orc, scale)
        for s in range(len(lens)):
            ref = sdpa(p.q[s], p.ks[s], p.vs[s], scale, dtype)
            assert_close(out[s], ref, 1e-12, f"paged vs SDPA {dtype} len {lens[s]}")


def pin_physical_permutation_invariance(orc):
    """Moving blocks around the pool (and rewriting the tables) changes
    nothing: bit-identical output."""
    rng = np.random.default_rng(8)
    p = Paged(rng, [20, 50, 9], 4, 2, 32, "bf16")
    out1 = p.run(orc, 0.2)
    NB = p.k_cache.shape[0]
    perm = rng.permutation(NB)          # new position of block b is perm[b]
    k2 = np.empty_like(p.k_cache)
    v2 = np.empty_like(p.v_cache)
    k2[perm] = p.k_cache
    v2[perm] = p.v_cache
    t2 = perm[p.tables].astype(np.int32)
    out2 = orc.paged_decode(p.q, k2, v2, t2, p.lens, 0.2, "bf16")
    assert np.array_equal(out1, out2), "output must not depend on physical placement"


def pin_gqa_equals_replicated_mha(orc):
    """GQA with group g equals MHA whose KV head h is the GQA KV head h // g."""
    rng = np.random.default_rng(9)
    lens = [12, 45]
    H, Hk, D = 8, 2, 16
    g = H // Hk
    p = Paged(rng, lens, H, Hk, D, "f16")
    out = p.run(orc, 0.25)
    ks = [np.repeat(k, g, axis=1) for k in p.ks]
    vs = [np.repeat(v, g, axis=1) for v in p.vs]
    m = Paged(rng, lens, H, H, D, "f16", q=p.q, ks=ks, vs=vs)
    out2 = m.run(orc, 0.25)
    assert np.array_equal(out, out2), "GQA must equal MHA with replicated KV heads"


def pin_position_tagged(orc):
    """V[j] = (j / 128, ...) and one chosen key is 16 q: that logit beats the
    others by > 30, so the output decodes to the chosen logical position.
    Checks that position j is read from table entry j // 16, slot j % 16."""
    rng = np.random.default_rng(10)
    lens = [100, 17, 64, 33]
    chosen = [0, 16, 63, 20]
    D, H, Hk = 64, 2, 2
    q = rand_bits(rng, (4, H, D), "f16")
    ks, vs = [], []
    for s, L in enumerate(lens):
        k = rand_bits(rng, (L, Hk, D), "f16", -0.25, 0.25)
        k[chosen[s]] = narrow(16.0 * widen(q[s], "f16"), "f16")
        v = np.zeros((L, Hk, D))
        v[:, :, 0] = (np.arange(L) / 128.0)[:, None]
        ks.append(k)
        vs.append(narrow(v, "f16"))
    p = Paged(rng, lens, H, Hk, D, "f16", q=q, ks=ks, vs=vs)
    out = p.run(orc, 1.0 / 8.0)
    got = np.rint(out[:, :, 0] * 128.0)
    assert np.array_equal(got, np.repeat(np.array(chosen)[:, None], H, axis=1)), \
        f"position-tagged decode read the wrong tokens: {got.tolist()} vs {chosen}"


def pin_large_logits_are_stable(orc):
    """Logits 3600, 3598.125 and 0: exp() of the first two overflows, the
    softmax does not.  Closed form out = (v0 + e^{-d} v1 + e^{-3600} v2) /
    (1 + e^{-d} + e^{-3600}), d = x0 - x1; the last terms underflow to 0."""
    q = narrow(np.array([[[60.0]]]), "f16")
    k0, k1 = 60.0, 59.96875                  # both exact in fp16
    ks = [narrow(np.array([[[k0]], [[k1]], [[0.0]]]), "f16")]
    vs = [narrow(np.array([[[1.0]], [[-1.0]], [[0.5]]]), "f16")]
    p = Paged(np.random.default_rng(11), [3], 1, 1, 1, "f16", q=q, ks=ks, vs=vs)
    out = p.run(orc, 1.0)[0, 0, 0]
    d = 60.0 * (k0 - k1)
    want = (1.0 - math.exp(-d)) / (1.0 + math.exp(-d))
    assert math.isfinite(out) and abs(out - want) < 1e-12, f"unstable softmax: {out} vs {want}"


def pin_widen_every_finite_value(orc):
    """Length 1 returns V, so every finite fp16 / bf16 bit pattern placed in V
    must come back as numpy's own widening of that pattern."""
    for dtype in ("f16", "bf16"):
        bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
        vals = widen(bits, dtype)
        bits = bits[np.isfinite(vals)]
        D = bits.size
        k = np.zeros((1, 1, 16, D), dtype=np.uint16)
        v = np.full((1, 1, 16, D), NAN[dtype], dtype=np.uint16)
        v[0, 0, 0] = bits
        q = np.zeros((1, 1, D), dtype=np.uint16)
        out = orc.paged_decode(q, k, v, np.zeros((1, 1), np.int32), np.ones(1, np.int32), 1.0,
                               dtype)
        assert np.array_equal(out[0, 0], widen(bits, dtype)), f"{dtype} widening is wrong"


def pin_widen_query_and_key(orc):
    """Logit of a single-dim query/key pair, read back through a two-token
    softmax: weight of token 0 is 1 / (1 + e^{-x}) with x = q k (scale 1)."""
    for dtype in ("f16", "bf16"):
        rng = np.random.default_rng(12)
        for _ in range(8):
            qb = rand_bits(rng, (1, 1, 1), dtype, -3, 3)
            kb = rand_bits(rng, (1, 1, 1), dtype, -3, 3)
            ks = [np.stack([kb[0], np.zeros((1, 1), np.uint16)])]
            vs = [narrow(np.array([[[1.0]], [[0.0]]]), dtype)]
            p = Paged(rng, [2], 1, 1, 1, dtype, q=qb, ks=ks, vs=vs)
            out = p.run(orc, 1.0)[0, 0, 0]
            x = float(widen(qb, dtype).ravel()[0] * widen(kb, dtype).ravel()[0])
            want = 1.0 / (1.0 + math.exp(-x))
            assert abs(out - want) < 1e-14, f"q/k widening ({dtype}): {out} vs {want}"


# ---------------------------------------------------------------------------
# cache-write and copy pins
# ---------------------------------------------------------------------------
def pin_reshape_and_cache_matches_indexing(orc):
    rng = np.random.default_rng(13)
    NB, Hk, B, D = 12, 3, 16, 8
    kc = rand_bits(rng, (NB, Hk, B, D), "bf16")
    vc = rand_bits(rng, (NB, Hk, B, D), "bf16")
    T = 40
    slots = rng.choice(NB * B, size=T, replace=False).astype(np.int64)
    slots[[3, 17, 30]] = -1
    key = rand_bits(rng, (T, Hk, D), "bf16")
    val = rand_bits(rng, (T, Hk, D), "bf16")
    ek, ev = kc.copy(), vc.copy()
    live = slots >= 0
    ek[slots[live] // B, :, slots[live] % B, :] = key[live]
    ev[slots[live] // B, :, slots[live] % B, :] = val[live]
    orc.reshape_and_cache(kc, vc, key, val, slots)
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev), "reshape_and_cache differs"


def pin_copy_blocks_matches_slices(orc):
    rng = np.random.default_rng(14)
    NB, Hk, B, D, L = 10, 2, 16, 8, 3
    ks = [rand_bits(rng, (NB, Hk, B, D), "f16") for _ in range(L)]
    vs = [rand_bits(rng, (NB, Hk, B, D), "f16") for _ in range(L)]
    pairs = np.array([[1, 5], [2, 7], [1, 9]], dtype=np.int64)
    ek = [k.copy() for k in ks]
    ev = [v.copy() for v in vs]
    for a in ek + ev:
        a[pairs[:, 1]] = a[pairs[:, 0]]
    orc.copy_blocks(ks, vs, pairs)
    for a, b in zip(ks + vs, ek + ev):
        assert np.array_equal(a, b), "copy_blocks differs from slice assignment"


def pin_copy_on_write_keeps_sharers(orc):
    """Two sequences share a partial block; the writer copies it first and
    writes into the copy.  The other sharer's attention output and bytes are
    unchanged, and the writer sees its new token."""
    rng = np.random.default_rng(15)
    H, Hk, D, B = 2, 2, 16, 16
    NB = 6
    kc = np.full((NB, Hk, B, D), NAN["bf16"], dtype=np.uint16)
    vc = kc.copy()
    kc[0, :, :10] = rand_bits(rng, (Hk, 10, D), "bf16")
    vc[0, :, :10] = rand_bits(rng, (Hk, 10, D), "bf16")
    q = rand_bits(rng, (2, H, D), "bf16")
    tables = np.array([[0], [0]], dtype=np.int32)
    lens = np.array([10, 10], dtype=np.int32)
    before = orc.paged_decode(q, kc, vc, tables, lens, 0.25, "bf16")
    shared_k, shared_v = kc[0].copy(), vc[0].copy()
    orc.copy_blocks([kc], [vc], np.array([[0, 3]], dtype=np.int64))
    key = rand_bits(rng, (1, Hk, D), "bf16")
    val = rand_bits(rng, (1, Hk, D), "bf16")
    orc.reshape_and_cache(kc, vc, key, val, np.array([3 * B + 10], dtype=np.int64))
    tables2 = np.array([[0], [3]], dtype=np.int32)
    after = orc.paged_decode(q, kc, vc, tables2, np.array([10, 11], np.int32), 0.25, "bf16")
    assert np.array_equal(kc[0], shared_k) and np.array_equal(vc[0], shared_v), \
        "copy-on-write modified the shared block"
    assert np.array_equal(after[0], before[0]), "the other sharer's output changed"
    assert np.array_equal(kc[3, :, :10], shared_k[:, :10]), "copy lost the shared prefix"
    assert np.array_equal(kc[3, :, 10], key[0]), "the writer's token is missing"


def pin_swap_blocks_matches_slices(orc):
    """Swap out to a second (host) pool and back: numpy slice copies, and a
    round trip restores the original blocks."""
    rng = np.random.default_rng(16)
    Hk, B, D = 2, 16, 8
    dev_k = rand_bits(rng, (9, Hk, B, D), "bf16")
    dev_v = rand_bits(rng, (9, Hk, B, D), "bf16")
    host_k = np.zeros((5, Hk, B, D), np.uint16)
    host_v = np.zeros((5, Hk, B, D), np.uint16)
    out_map = np.array([[7, 0], [2, 3], [4, 1]], dtype=np.int64)
    want_k = host_k.copy()
    want_v = host_v.copy()
    want_k[out_map[:, 1]] = dev_k[out_map[:, 0]]
    want_v[out_map[:, 1]] = dev_v[out_map[:, 0]]
    orc.swap_blocks(host_k, host_v, dev_k, dev_v, out_map)
    assert np.array_equal(host_k, want_k) and np.array_equal(host_v, want_v), "swap-out differs"
    back = np.stack([out_map[:, 1], [0, 5, 6]], axis=1)
    orig_k, orig_v = dev_k.copy(), dev_v.copy()
    orc.swap_blocks(dev_k, dev_v, host_k, host_v, back)
    assert np.array_equal(dev_k[[0, 5, 6]], orig_k[[7, 2, 4]]), "swap-in did not restore the blocks"
    assert np.array_equal(dev_v[[0, 5, 6]], orig_v[[7, 2, 4]]), "swap-in did not restore the blocks"
    keep = [1, 3, 7, 8]
    assert np.array_equal(dev_k[keep], orig_k[keep]), "swap-in touched other blocks"


# ---------------------------------------------------------------------------
# FP8 E4M3 KV-cache pins
# ---------------------------------------------------------------------------
def e4m3_torch(codes) -> np.ndarray:
    """torch's own E4M3 decoding (a library routine)."""
    t = torch.from_numpy(np.asarray(codes, dtype=np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.float().numpy().astype(np.float64)


def pin_e4m3_widen_every_code(orc):
    codes = np.arange(256, dtype=np.uint8)
    got, want = orc.widen_e4m3(codes), e4m3_torch(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want)), "NaN codes differ"
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok]), "E4M3 decoding differs from torch"


def pin_e4m3_quantize_matches_torch_in_range(orc):
    """Random values, every representable value and every midpoint between
    neighbours (the tie cases) up to 448, both signs: same codes as torch's
    round-to-nearest-even conversion, the sign of zero included."""
    rng = np.random.default_rng(17)
    vals = e4m3_torch(np.arange(0, 0x7f, dtype=np.uint8))        # +0 .. 448
    mids = (vals[:-1] + vals[1:]) / 2
    y = np.concatenate([vals, mids, rng.uniform(-448, 448, 4000), rng.uniform(-1, 1, 4000),
                        rng.uniform(-2 ** -6, 2 ** -6, 2000)]).astype(np.float32)
    y = np.concatenate([y, -y])
    want = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.quantize_e4m3(y)
    # exact, zeros included: -0.0 and negatives that round to zero give -0 (0x80)
    assert np.array_equal(got, want), "quantisation differs from torch in range"
    assert got[np.signbit(y) & (y == 0)].tolist() and np.all(got[np.signbit(y) & (y == 0)] == 0x80)


def pin_e4m3_saturates_to_finite(orc):
    y = np.array([448.5, 463.9, 464.0, 500.0, 1e6, np.inf, -449.0, -1e9, np.nan], dtype=np.float32)
    got = orc.quantize_e4m3(y)
    assert got.tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F], got.tolist()


def pin_fp8_decode_equals_dequantized_decode(orc):
    """With power-of-two scales every decoded element is exact in fp16, so
    the FP8 decode must equal the (pinned) 16-bit decode of those values."""
    rng = np.random.default_rng(18)
    lens = [1, 16, 17, 70]
    H, Hk, D = 4, 2, 32
    k_scale, v_scale = 2.0 ** -6, 2.0 ** -5
    p16 = Paged(rng, lens, H, Hk, D, "f16")
    NB = p16.k_cache.shape[0]
    kc = rng.integers(0, 0x7f, size=(NB, Hk, 16, D), dtype=np.uint8) | (rng.integers(0, 2, (NB, Hk, 16, D)) << 7).astype(np.uint8)
    vc = rng.integers(0, 0x7f, size=(NB, Hk, 16, D), dtype=np.uint8) | (rng.integers(0, 2, (NB, Hk, 16, D)) << 7).astype(np.uint8)
    k16 = narrow(e4m3_torch(kc) * k_scale, "f16")
    v16 = narrow(e4m3_torch(vc) * v_scale, "f16")
    assert np.array_equal(widen(k16, "f16"), e4m3_torch(kc) * k_scale), "scaled values must be exact in fp16"
    want = orc.paged_decode(p16.q, k16, v16, p16.tables, p16.lens, 0.2, "f16")
    got = orc.paged_decode_fp8(p16.q, kc, vc, p16.tables, p16.lens, 0.2, k_scale, v_scale, "f16")
    assert np.array_equal(got, want), "FP8 decode differs from the dequantized 16-bit decode"


def pin_fp8_cache_write_matches_indexing(orc):
    rng = np.random.default_rng(19)
    NB, Hk, B, D = 6, 2, 16, 16
    kc = rng.integers(0, 255, size=(NB, Hk, B, D), dtype=np.uint8)
    vc = rng.integers(0, 255, size=(NB, Hk, B, D), dtype=np.uint8)
    T = 20
    slots = rng.choice(NB * B, size=T, replace=False).astype(np.int64)
    slots[4] = -1
    key = rand_bits(rng, (T, Hk, D), "bf16", -2, 2)
    val = rand_bits(rng, (T, Hk, D), "bf16", -2, 2)
    ks, vs = np.float32(1 / 200), np.float32(1 / 150)
    ek, ev = kc.copy(), vc.copy()
    live = slots >= 0
    qk = torch.from_numpy(widen(key, "bf16").astype(np.float32) / ks).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    qv = torch.from_numpy(widen(val, "bf16").astype(np.float32) / vs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ek[slots[live] // B, :, slots[live] % B, :] = qk[live]
    ev[slots[live] // B, :, slots[live] % B, :] = qv[live]
    orc.reshape_and_cache_fp8(kc, vc, key, val, slots, "bf16", float(ks), float(vs))
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev), "FP8 cache write differs"


def pin_brute_force_tiny(orc):
    """The first scenario (4 seqs, lengths 1/17/33/100) against the pure
    Python brute force, every (sequence, head)."""
    from oracle import brute
    from oracle.harness import OracleSession
    from paged_kv_cache_424_b200 import workload as W
    sc = W.tiny(0)
    ses = OracleSession(sc, oracle=orc)
    st = sc.steps[0]
    out = ses.run_step(st)
    k, v = ses.pool.view()
    rel = ses.pool.relabel_tables(st.block_tables, st.context_lens, 16)
    ref = np.array(brute.paged_decode(st.q, k, v, rel, st.context_lens, sc.scale, "f16"))
    assert_close(out, ref, 1e-13, "oracle vs brute force")



# ---------------------------------------------------------------------------
# multi-token / sliding-window decode pins
# ---------------------------------------------------------------------------
def ext_q(rng, S, q_len, H, D, dtype):
    return rand_bits(rng, (S, q_len, H, D), dtype)


def masked_sdpa(q_bits, k_bits, v_bits, L, q_len, window, scale, dtype):
    """torch float64 SDPA for one sequence with an explicit boolean mask:
    q [q_len, H, D], k/v [L, Hk, D]; query i sees positions
    max(0, p - W + 1) .. p with p = L - q_len + i (all up to p when W = 0).
    Rows with p < 0 are zero."""
    H = q_bits.shape[1]
    out = np.zeros((q_len, H, q_bits.shape[2]))
    pos = np.arange(L)
    mask = np.zeros((q_len, L), dtype=bool)
    for i in range(q_len):
        p = L - q_len + i
        lo = max(0, p - window + 1) if window > 0 else 0
        mask[i] = (pos <= p) & (pos >= lo)
    live = mask.any(axis=1)
    if L == 0 or not live.any():
        return out
    q = torch.from_numpy(widen(q_bits, dtype)).permute(1, 0, 2)[None]          # [1, H, q_len, D]
    k = torch.from_numpy(widen(k_bits, dtype)).permute(1, 0, 2)[None]          # [1, Hk, L, D]
    v = torch.from_numpy(widen(v_bits, dtype)).permute(1, 0, 2)[None]
    m = torch.from_numpy(mask)
    m[~torch.from_numpy(live)] = True  # keep torch finite on dead rows; they are overwritten
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale,
                                                         enable_gqa=q.shape[1] != k.shape[1])
    o = o[0].permute(1, 0, 2).numpy()
    out[live] = o[live]
    return out


def pin_ext_matches_masked_sdpa(orc):
    """Multi-token and sliding-window decode equal torch SDPA with the
    causal-window mask written out, for q_len 1-3, windows 0/1/7/16/33, GQA,
    lengths below q_len (zero rows) through 100."""
    rng = np.random.default_rng(71)
    lens = [1, 2, 5, 16, 17, 40, 100]
    for dtype in ("f16", "bf16"):
        p = Paged(rng, lens, 8, 2, 16, dtype)
        for q_len in (1, 3):
            q = ext_q(rng, len(lens), q_len, 8, 16, dtype)
            for window in (0, 1, 7, 16, 33):
                got = orc.paged_decode_ext(q, p.k_cache, p.v_cache, p.tables, p.lens, 0.3, dtype, q_len, window)
                for s, L in enumerate(lens):
                    want = masked_sdpa(q[s], p.ks[s], p.vs[s], L, q_len, window, 0.3, dtype)
                    assert_close(got[s], want, 1e-12, f"ext {dtype} q_len={q_len} W={window} L={L}")


def pin_ext_reduces_to_decode(orc):
    """q_len 1 without a window is plain decode; a window at least as long as
    the context changes nothing."""
    rng = np.random.default_rng(72)
    lens = [1, 16, 33, 300]
    p = Paged(rng, lens, 8, 4, 32, "bf16")
    base = p.run(orc, 0.2)
    for window in (0, 300, 1000):
        got = orc.paged_decode_ext(p.q[:, None], p.k_cache, p.v_cache, p.tables, p.lens, 0.2, "bf16", 1, window)
        assert np.array_equal(got[:, 0], base), f"window {window}"


def pin_ext_window_one_returns_own_value(orc):
    """A window of one token: each query returns V at its own position."""
    rng = np.random.default_rng(73)
    lens = [3, 16, 17, 50]
    p = Paged(rng, lens, 4, 2, 16, "f16")
    q = ext_q(rng, len(lens), 3, 4, 16, "f16")
    got = orc.paged_decode_ext(q, p.k_cache, p.v_cache, p.tables, p.lens, 0.5, "f16", 3, 1)
    for s, L in enumerate(lens):
        for i in range(3):
            want = widen(p.vs[s][L - 3 + i], "f16")       # [Hk, D]
            assert np.array_equal(got[s, i], np.repeat(want, 2, axis=0)), f"s={s} i={i}"


def pin_ext_query_i_is_a_truncated_decode(orc):
    """Query i of a multi-token call equals a single-query call whose context
    ends at that query's position (with and without a window)."""
    rng = np.random.default_rng(74)
    lens = [4, 20, 64, 129]
    p = Paged(rng, lens, 8, 8, 32, "bf16")
    q = ext_q(rng, len(lens), 4, 8, 32, "bf16")
    for window in (0, 10):
        got = orc.paged_decode_ext(q, p.k_cache, p.v_cache, p.tables, p.lens, 0.25, "bf16", 4, window)
        for i in range(4):
            lens_i = p.lens - 4 + i + 1
            one = orc.paged_decode_ext(np.ascontiguousarray(q[:, i:i + 1]), p.k_cache, p.v_cache, p.tables, lens_i,
                                       0.25, "bf16", 1, window)
            assert np.array_equal(got[:, i], one[:, 0]), f"query {i} window {window}"


def pin_ext_scales_and_fp8(orc):
    """K and V scales multiply the cache elements: a 16-bit cache scaled by
    powers of two equals the pre-scaled cache, and E4M3 codes equal their
    exactly widened 16-bit values."""
    rng = np.random.default_rng(75)
    lens = [5, 31, 70]
    p = Paged(rng, lens, 4, 2, 16, "f16")
    q = ext_q(rng, len(lens), 2, 4, 16, "f16")
    got = orc.paged_decode_ext(q, p.k_cache, p.v_cache, p.tables, p.lens, 0.3, "f16", 2, 9, k_scale=4.0,
                               v_scale=0.5)
    k4 = narrow(widen(p.k_cache, "f16") * 4.0, "f16")
    v5 = narrow(widen(p.v_cache, "f16") * 0.5, "f16")
    want = orc.paged_decode_ext(q, k4, v5, p.tables, p.lens, 0.3, "f16", 2, 9)
    assert np.array_equal(got, want), "scales are not applied to the elements"
    NB, Hk, B, D = p.k_cache.shape
    kc = rng.integers(0, 256, size=(NB, Hk, B, D), dtype=np.uint8)
    kc[(kc & 0x7F) == 0x7F] = 0x38
    vc = np.roll(kc, 1, axis=0)
    got8 = orc.paged_decode_ext(q, kc, vc, p.tables, p.lens, 0.01, "f16", 2, 9, k_scale=0.25, v_scale=2.0)
    k16 = narrow(e4m3_torch(kc) * 0.25, "f16")
    v16 = narrow(e4m3_torch(vc) * 2.0, "f16")
    want8 = orc.paged_decode_ext(q, k16, v16, p.tables, p.lens, 0.01, "f16", 2, 9)
    assert np.array_equal(got8, want8), "E4M3 ext decode differs from the widened 16-bit one"


def pin_ext_reads_no_block_before_the_window(orc):
    """Table entries of blocks wholly before every query's window are never
    read (they may hold anything); without the window the same entries are."""
    rng = np.random.default_rng(76)
    lens = [100, 64]
    p = Paged(rng, lens, 4, 4, 16, "f16")
    q = ext_q(rng, 2, 2, 4, 16, "f16")
    want = orc.paged_decode_ext(q, p.k_cache, p.v_cache, p.tables, p.lens, 0.3, "f16", 2, 20)
    t = p.tables.copy()
    t[0, :4] = -1      # sequence 0: window covers positions 79..99 -> blocks 4..6
    t[1, :2] = 10 ** 6  # sequence 1: positions 43..63 -> blocks 2..3
    got = orc.paged_decode_ext(q, p.k_cache, p.v_cache, t, p.lens, 0.3, "f16", 2, 20)
    assert np.array_equal(got, want)
    from oracle import OracleError
    try:
        orc.paged_decode_ext(q, p.k_cache, p.v_cache, t, p.lens, 0.3, "f16", 2, 0)
    except OracleError:
        return
    raise AssertionError("entries inside the attended range must be checked")

ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
