"""The host prefix cache (pa_prefix_cache_*) and the shared-prefix order
(pa_prefix_order) of libpa.so, on the CPU: no GPU is touched (host code).

The cache is checked against a plain Python model of automatic prefix
caching ("vLLM PagedAttention 大模型推理架构深度实战" section 7.3: requests
with an identical prefix share KV-cache blocks; section 2.3: a block's
reference count is the number of sequences mapping it): a dict from the
whole token prefix of each full block to its block id, reference counts,
and least-recently-released eviction.
"""
import collections

import numpy as np
import pytest


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_424_b200 import build
    build.build()
    from paged_kv_cache_424_b200 import binding
    return binding


class Model:
    """Prefix caching by whole-prefix keys (no hashing, no parent chain)."""

    def __init__(self):
        self.by_prefix = {}          # tuple(tokens[: 16 (i + 1)]) -> block
        self.prefix_of = {}          # block -> its key
        self.refs = collections.Counter()
        self.lru = collections.OrderedDict()

    def match(self, tokens):
        out = []
        for i in range(len(tokens) // 16):
            b = self.by_prefix.get(tuple(tokens[:16 * (i + 1)]))
            if b is None:
                break
            out.append(b)
        for b in out:
            if self.refs[b] == 0:
                self.lru.pop(b, None)
            self.refs[b] += 1
        return out

    def insert(self, tokens, blocks):
        for i in range(min(len(tokens) // 16, len(blocks))):
            key = tuple(tokens[:16 * (i + 1)])
            b = blocks[i]
            if key in self.by_prefix or b in self.prefix_of:
                continue
            self.by_prefix[key] = b
            self.prefix_of[b] = key
            self.refs[b] = 1

    def release(self, blocks):
        n = 0
        for b in blocks:
            if b in self.prefix_of and self.refs[b] > 0:
                self.refs[b] -= 1
                if self.refs[b] == 0:
                    self.lru[b] = True
                n += 1
        return n

    def evict(self, k):
        out = []
        while len(out) < k and self.lru:
            b, _ = self.lru.popitem(last=False)
            key = self.prefix_of.pop(b)
            del self.by_prefix[key]
            out.append(b)
        return out


def test_match_insert_release_evict_against_the_model(pa):
    rng = np.random.default_rng(9)
    NB = 400
    cache, model = pa.PrefixCache(NB), Model()
    free = list(rng.permutation(NB))
    prompts = [list(rng.integers(0, 50, size=int(n))) for n in rng.integers(16, 200, size=12)]
    live = []
    for step in range(300):
        op = rng.random()
        if op < 0.5 or not live:
            # a request: a known prompt plus a random continuation
            base = prompts[int(rng.integers(len(prompts)))]
            cut = int(rng.integers(0, len(base) + 1))
            toks = base[:cut] + list(rng.integers(0, 50, size=int(rng.integers(0, 60))))
            got, want = cache.match(toks), model.match(toks)
            assert got == want, f"step {step}: match"
            need = len(toks) // 16 - len(got)
            if need > len(free):
                ev = cache.evict(need - len(free) + 8)
                assert ev == model.evict(need - len(free) + 8), f"step {step}: evict"
                free.extend(ev)
            if need > len(free):
                cache.release(got)
                model.release(got)
                continue
            blocks = got + [int(free.pop()) for _ in range(need)]
            cache.insert(toks, blocks)
            model.insert(toks, blocks)
            live.append(blocks)
        else:
            blocks = live.pop(int(rng.integers(len(live))))
            assert cache.release(blocks) == model.release(blocks), f"step {step}: release"
            # blocks that are not cached go straight back to the free list
            free.extend(b for b in blocks if b not in model.prefix_of)
        st = cache.stats()
        assert st["cached"] == len(model.by_prefix)
        assert st["evictable"] == len(model.lru)
    assert cache.stats()["hits"] > 50, "the workload never reused a prefix"


def test_shared_prompt_is_found_and_divergence_stops_the_match(pa):
    cache = pa.PrefixCache(64)
    a = list(range(100, 164))                   # 4 full blocks
    cache.insert(a, [10, 11, 12, 13])
    assert cache.match(a + [1, 2, 3]) == [10, 11, 12, 13]
    b = a[:40] + [999] + a[41:]                 # differs inside block 2
    assert cache.match(b) == [10, 11]
    assert cache.match([7] + a[1:]) == []       # differs in the first token
    assert cache.match(a[:15]) == []            # no full block
    # equal blocks behind a different parent are different prefixes
    cache.insert([5] * 16 + a[16:32], [20, 21])
    assert cache.match([5] * 16 + a[16:32]) == [20, 21]
    assert cache.match(a[:32]) == [10, 11]


def test_evicted_parent_makes_children_unreachable(pa):
    cache = pa.PrefixCache(16)
    a = list(range(48))
    cache.insert(a, [1, 2, 3])
    cache.release([1, 2, 3])
    assert cache.evict(1) == [1]                # least recently released first
    assert cache.match(a) == []                 # the chain starts at the evicted block
    # block 1 reused for other content: its old children must not come back
    cache.insert([9] * 16, [1])
    assert cache.match([9] * 16 + a[16:]) == [1]
    assert cache.stats()["cached"] == 3         # 2 and 3 stay until evicted
    assert sorted(cache.evict(10)) == [2, 3]    # 1 is in use (refs 1)


def test_bad_arguments(pa):
    import ctypes
    assert not pa.LIB.pa_prefix_cache_create(0)
    assert pa.LIB.pa_prefix_cache_match(None, None, 0, None, 0) == -1
    c = pa.PrefixCache(8)
    with pytest.raises(pa.PagedAttentionError):
        c.insert(list(range(16)), [8])          # block id outside the pool
    assert pa.LIB.pa_prefix_cache_evict(c._h, -1, None) == -3


def test_prefix_order_groups_sharers(pa):
    rng = np.random.default_rng(3)
    S, MB = 40, 6
    firsts = rng.integers(0, 7, size=S)        # 7 prefixes shared by several sequences
    bt = np.zeros((S, MB), np.int32)
    bt[:, 0] = firsts * 10
    bt[:, 1:] = rng.integers(100, 1000, size=(S, MB - 1))
    cl = rng.integers(1, MB * 16, size=S).astype(np.int32)
    cl[[3, 17]] = 0
    order = pa.pa_prefix_order(bt, cl)
    assert sorted(order.tolist()) == list(range(S)), "not a permutation"
    assert order[-2:].tolist() == [3, 17], "empty contexts go last"
    keys = [bt[s, 0] for s in order[:-2]]
    assert keys == sorted(keys), "sharers of a first block must be adjacent, in block order"
    # within a group, batch order is kept
    for k in set(keys):
        members = [s for s in order[:-2] if bt[s, 0] == k]
        assert members == sorted(members)


def test_prefix8b_order_clusters_the_shuffled_batch(pa):
    """In the benchmark's shuffled batch the 8 sharers of each prompt are
    scattered; in pa_prefix_order's order they are adjacent."""
    from paged_kv_cache_424_b200 import workload as W
    sc = W.prefix8b(num_prompts=8, num_blocks=4096)
    st = sc.steps[0]
    first = st.block_tables[:, 0]
    runs_batch = 1 + int(np.count_nonzero(first[1:] != first[:-1]))
    order = pa.pa_prefix_order(st.block_tables, st.context_lens)
    f2 = first[order]
    runs_sorted = 1 + int(np.count_nonzero(f2[1:] != f2[:-1]))
    assert runs_sorted == 8 and runs_batch > 8
