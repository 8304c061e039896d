"""Prefix caching in the block allocator (host only): the C++ allocator against the reference
model after every operation of seeded scenarios with shared prompts and evictions; the model
against a brute-force longest-common-prefix rule and a hand-computed eviction sequence."""
import copy
import random

import pytest

from oracle.alloc_model import AllocatorModel, OutOfBlocks
import paged_kv_cache_428_b200 as pa
from test_allocator import same_state


def _same(a, m):
    same_state(a, m)
    assert a.prefix_stats() == m.prefix_stats()


def _prompt(rng, systems, bs):
    """A shared system prompt (sometimes cut), then a few random tokens."""
    base = list(rng.choice(systems))
    if rng.random() < 0.3:
        base = base[:rng.randint(0, len(base))]
    return base + [rng.randint(0, 5) for _ in range(rng.randint(0, 3 * bs))]


@pytest.mark.parametrize("seed", range(10))
def test_prefix_scenarios_match_model(seed):
    rng = random.Random(100 + seed)
    nb, bs = rng.choice([(24, 4), (40, 8), (16, 2)])
    systems = [[rng.randint(0, 3) for _ in range(rng.randint(bs, 4 * bs))] for _ in range(3)]
    a = pa.BlockAllocator(nb, bs, seed)
    m = AllocatorModel(nb, bs, seed)
    live = []
    for step in range(250):
        op = rng.random()
        if op < 0.35 or not live:
            toks = _prompt(rng, systems, bs)
            try:
                want = m.new_seq_prefix(toks)
            except OutOfBlocks:
                with pytest.raises(pa.PagedKVError) as e:
                    a.new_seq_prefix(toks)
                assert e.value.status == -4
            else:
                got = a.new_seq_prefix(toks)
                assert got == want
                live.append(got[0])
        elif op < 0.55:
            s = rng.choice(live)
            try:
                want = m.append_slot(s)
            except OutOfBlocks:
                with pytest.raises(pa.PagedKVError):
                    a.append_slot(s)
            else:
                assert a.append_slot(s) == want
        elif op < 0.65:
            seqs = rng.sample(live, rng.randint(1, len(live)))
            snap = copy.deepcopy(m)
            try:
                res = [m.append_slot(s) for s in seqs]
            except OutOfBlocks:
                m = snap
                with pytest.raises(pa.PagedKVError):
                    a.append_batch(seqs)
            else:
                slots, pairs = a.append_batch(seqs)
                assert slots == [r[0] for r in res]
                assert pairs == [r[1] for r in res if r[1][0] >= 0]
        elif op < 0.72:
            p = rng.choice(live)
            c = a.fork(p)
            assert c == m.fork(p)
            live.append(c)
        elif op < 0.8:
            seqs = rng.sample(live, rng.randint(1, len(live)))
            assert a.order_by_prefix(seqs) == m.order_by_prefix(seqs)
        else:
            s = rng.choice(live)
            a.free_seq(s)
            m.free_seq(s)
            live.remove(s)
        m.check_invariants()
        _same(a, m)
    assert m.hit_tokens > 0 and m.gen != [0] * nb or nb >= 40      # hits happened; small pools evicted


def _lcp(x, y):
    n = 0
    while n < min(len(x), len(y)) and x[n] == y[n]:
        n += 1
    return n


@pytest.mark.parametrize("seed", range(6))
def test_model_hits_are_longest_common_full_block_prefix(seed):
    """Without evictions, a prompt's cached tokens are the longest common prefix with any earlier
    prompt, rounded down to whole blocks of both (brute force over all earlier prompts)."""
    rng = random.Random(seed)
    bs = rng.choice([2, 4, 8])
    systems = [[rng.randint(0, 2) for _ in range(rng.randint(0, 5 * bs))] for _ in range(4)]
    m = AllocatorModel(4096, bs, seed)
    seen = []
    for _ in range(60):
        toks = _prompt(rng, systems, bs)
        want = max([(min(_lcp(toks, p), len(p)) // bs) * bs for p in seen] + [0])
        _, _, cached = m.new_seq_prefix(toks)
        assert cached == want
        seen.append(toks)


def test_hand_computed_eviction():
    """Pool of 3 blocks of 2 tokens, identity order."""
    m = AllocatorModel(3, 2, 0)
    a = pa.BlockAllocator(3, 2, 0)
    for x in (m, a):
        sA, slots, cached = x.new_seq_prefix([1, 2, 3, 4])           # blocks 0, 1, both registered
        assert (slots, cached) == ([0, 1, 2, 3], 0)
        x.free_seq(sA)                                               # queue: 1, then 0
        sC, slots, cached = x.new_seq_prefix([1, 2, 7, 7])           # hit block 0, fresh block 2
        assert (slots, cached) == ([0, 1, 4, 5], 2)
        with pytest.raises((OutOfBlocks, pa.PagedKVError)):
            x.new_seq_prefix([5, 5, 6, 6, 8])                        # needs 3, only block 1 evictable
        x.free_seq(sC)                                               # queue: 1, 2, 0
        sD, slots, cached = x.new_seq_prefix([5, 5, 6, 6, 8])        # evicts 1, 2, 0 in that order
        assert (slots, cached) == ([2, 3, 4, 5, 0], 0)
        with pytest.raises((OutOfBlocks, pa.PagedKVError)):
            x.new_seq_prefix([1, 2, 3, 4])                           # evicted: a miss, and no room
    assert m.prefix_stats() == a.prefix_stats() == {"hit_tokens": 2, "miss_tokens": 11, "cached_blocks": 2,
                                                    "evictable": 0}


def test_shared_system_prompt_memory():
    """N requests with one L-token system prompt (L a multiple of bs) and private questions hold
    L / bs shared blocks plus their own: used = L/bs + sum ceil(q_i / bs)."""
    bs, L = 16, 256
    rng = random.Random(7)
    sysp = [rng.randint(0, 1000) for _ in range(L)]
    qs = [rng.randint(1, 100) for _ in range(12)]
    a = pa.BlockAllocator(400, bs, 3)
    cached = []
    for i, q in enumerate(qs):
        _, _, c = a.new_seq_prefix(sysp + [1000 + i] * q)
        cached.append(c)
    assert cached == [0] + [L] * (len(qs) - 1)
    assert a.stats()["used"] == L // bs + sum(-(-q // bs) for q in qs)
    assert a.prefix_stats()["hit_tokens"] == L * (len(qs) - 1)


def test_order_by_prefix_groups_sharers():
    bs = 4
    a = pa.BlockAllocator(200, bs, 11)
    p1, p2 = list(range(12)), list(range(100, 108))
    sids = []
    for i in range(6):                         # interleaved: p1, p2, p1, p2 ...
        sid, _, _ = a.new_seq_prefix((p1 if i % 2 == 0 else p2) + [50 + i])
        sids.append(sid)
    order = a.order_by_prefix(sids)
    groups = [0 if i % 2 == 0 else 1 for i in order]
    assert groups in ([0, 0, 0, 1, 1, 1], [1, 1, 1, 0, 0, 0])
    assert sorted(order) == list(range(6))


def test_prefix_report_matches_closed_form_and_model():
    """System prompt (256) + one of 4 documents (1536) + a question: after the first request of
    a document, each request finds system + document cached (1792 tokens, 112 whole blocks); the
    first request of every other document finds the system prompt; changing each document's
    first tokens leaves only the system prompt to hit."""
    import workloads
    from paged_kv_cache_428_b200 import memory_report
    name = "sys256_doc1536x4_q64_n64"
    bs = workloads.PREFIX_TRACES[name]["bs"]
    prompts = workloads.make_prefix_prompts(name, 0)
    docs_seen, want = set(), 0
    for i, p in enumerate(prompts):
        doc = tuple(p[256:256 + 1536])
        want += 0 if i == 0 else (1792 if doc in docs_seen else 256)
        docs_seen.add(doc)
    rep = memory_report.run_prefix_prompts(prompts, bs)
    assert rep["cached_tokens"] == want
    m = AllocatorModel(sum(-(-len(p) // bs) for p in prompts), bs, 0)
    assert [m.new_seq_prefix(p)[2] for p in prompts] and m.hit_tokens == rep["hit_tokens"]
    assert m.stats()["used"] == rep["blocks_shared"]
    changed = memory_report.run_prefix_prompts(workloads.make_prefix_prompts(name, 0, front_changed=True), bs)
    assert changed["cached_tokens"] == 256 * (len(prompts) - 1)
    assert rep["prefill_skipped"] > 0.9 and changed["prefill_skipped"] < 0.15
