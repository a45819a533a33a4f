"""The seeded synthetic inputs against the recipe they are stated to follow:
shapes, length mixes, batch churn, copy-on-write pair counts, NaN-poisoned
unused slots and the write-then-attend position of the new token."""
import numpy as np
import pytest

from paged_kv_cache_424_b200 import workload as W

NAN = {"f16": W.NAN_BITS["f16"], "bf16": W.NAN_BITS["bf16"]}


def _slot_of(st, s, pos):
    return int(st.block_tables[s, pos // W.BLOCK_SIZE]) * W.BLOCK_SIZE + pos % W.BLOCK_SIZE


def test_tiny_recipe():
    sc = W.tiny(0)
    d = sc.dims
    assert (d.num_seqs, d.num_heads, d.num_kv_heads, d.head_dim, d.block_size, d.num_blocks, d.dtype) == \
        (4, 8, 8, 64, 16, 64, "f16")
    st = sc.steps[0]
    assert st.context_lens.tolist() == [1, 17, 33, 100]
    # the step writes each sequence's last position (context lengths count the new token)
    slots = st.writes[0].slot_mapping
    for s, L in enumerate(st.context_lens):
        assert slots[s] == _slot_of(st, s, int(L) - 1)
        nb = -(-int(L) // 16)
        assert np.all(st.block_tables[s, nb:] == sc.pad_block)  # padding entries name the NaN block
    # admitted contents: tokens before the new one are finite, every other slot is NaN
    pos_of = {}
    for s, L in enumerate(st.context_lens):
        for j in range(int(L)):
            pos_of[_slot_of(st, s, j)] = (s, j, int(L))
    for i, blk in enumerate(st.admit_ids):
        for t in range(16):
            k = st.admit_k[i, :, t, :]
            info = pos_of.get(int(blk) * 16 + t)
            if info is not None and info[1] < info[2] - 1:
                assert not np.any(k == NAN["f16"])
            else:
                assert np.all(k == NAN["f16"])
    assert sc.pad_block in st.admit_ids.tolist()


def test_lognormal_length_mix():
    """Median 1024, sigma 1, capped at 4096: P(capped) = P(Z > ln 4) = 0.0829."""
    L = W.lognormal_lengths(np.random.default_rng(0), 200000)
    assert L.min() >= 1 and L.max() == 4096
    assert abs(np.median(L) - 1024) < 12
    assert abs(np.mean(L == 4096) - 0.0829) < 0.003


def test_mha7b_and_long_shapes():
    m = W.mha7b(num_seqs=8)
    assert (m.dims.num_heads, m.dims.num_kv_heads, m.dims.head_dim, m.dims.dtype) == (32, 32, 128, "f16")
    assert np.all((m.steps[0].context_lens >= 128) & (m.steps[0].context_lens <= 2048))
    assert m.dims.max_blocks_per_seq == 128
    g = W.long70b(num_seqs=1, context_len=64, num_blocks=64)
    assert (g.dims.num_heads, g.dims.num_kv_heads, g.dims.dtype, g.partition_tokens) == (64, 8, "bf16", 512)
    w = W.window70b(num_seqs=1, context_len=64, window=16, num_blocks=64)
    assert (w.dims.num_heads, w.dims.num_kv_heads, w.window) == (64, 8, 16)


def test_gqa8b_churn():
    """Each later step retires round(0.1 S) sequences, admits as many with
    L ~ U{32..512} and grows every survivor by one token."""
    S = 40
    sc = W.gqa8b(seed=3, num_seqs=S, num_steps=4, median=64, cap=256, num_blocks=4096)
    assert (sc.dims.num_heads, sc.dims.num_kv_heads, sc.dims.head_dim, sc.dims.dtype) == (32, 8, 128, "bf16")
    for prev, cur in zip(sc.steps, sc.steps[1:]):
        grew = cur.context_lens == prev.context_lens + 1
        new = ~grew
        assert new.sum() == 4
        assert np.all((cur.context_lens[new] >= 32) & (cur.context_lens[new] <= 512))
        slots = cur.writes[0].slot_mapping
        for s in range(S):
            assert slots[s] == _slot_of(cur, s, int(cur.context_lens[s]) - 1)


@pytest.mark.parametrize("every", [False, True], ids=["while-shared", "per-sample"])
def test_cow_pairs_and_lengths(every):
    """A 1000-token prefix leaves an 8-token shared partial block: 7 copies
    per prompt when only a writer that still shares it copies, 8 when every
    sample copies."""
    P, n = 3, 8
    sc = W.cow(seed=4, num_prompts=P, samples=n, prefix=1000, max_tail=256, num_blocks=4096,
               cow_every_sample=every)
    st = sc.steps[0]
    assert len(st.block_mapping) == P * (n if every else n - 1)
    tails = st.context_lens - 1001
    assert np.all((tails >= 0) & (tails <= 256))
    # every sequence's first 62 blocks are its prompt's shared full blocks
    first = st.block_tables[:, :62]
    for p in range(P):
        assert np.all(first[p * n:(p + 1) * n] == first[p * n])
    assert len(np.unique(first[:, 0])) == P


def test_spec_and_prefix_recipes():
    sp = W.spec8b(num_seqs=4, median=64, cap=256, num_blocks=512)
    assert sp.q_len == 4 and sp.ext
    st = sp.steps[0]
    assert st.q.shape == (4, 4, 32, 128)
    assert len(st.writes[0].slot_mapping) == 16  # the decoded token and 3 draft tokens per sequence
    pf = W.prefix8b(num_prompts=2, prefix=100, num_blocks=512)
    assert pf.prefix_order and pf.ext and pf.dims.num_seqs == 16
    # the batch is shuffled: sharers of a prompt are not all adjacent
    firsts = pf.steps[0].block_tables[:, 0]
    assert any(firsts[i] != firsts[i + 1] for i in range(0, 7))


def test_fp8_variant_scales():
    sc = W.with_fp8_cache(W.tiny(0))
    assert sc.kv_dtype == "fp8" and sc.kv_elem_bytes == 1
    # |x| <= 1 over the scale stays inside E4M3's 448, and the scales are not powers of two
    assert 1.0 / sc.k_scale < 448 and 1.0 / sc.v_scale < 448
    for s in (sc.k_scale, sc.v_scale):
        m, _ = np.frexp(s)
        assert m != 0.5
