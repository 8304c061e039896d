"""Reference model of the host block allocator -- TEST INFRASTRUCTURE ONLY.

A deliberately plain Python restatement of the block-management rules the
pages describe, used to check the product's C++ allocator through its C ABI:

* fixed-size physical blocks handed out from one global free pool, the next
  block taken only when the current one is full
  ("深度解构 LLM 推理优化…" section 2.2, 动态按需分配);
* a block table per sequence mapping logical block i to a physical id
  (same page, section 2.1; "vLLM 推理原理…" section "PagedAttention 怎样整理这些缓存");
* per-block reference counts, zero-copy sharing of a parent's blocks by
  forked sequences, copy-on-write on the first divergent write into a shared
  block, release of a block when its count reaches zero
  ("KVCache技术背景与核心挑战 / PageAttention内存管理机制" sections 2.1-2.2 and 3.1;
  "深度解构…" section 2.3);
* return of all blocks of a finished sequence to the pool
  ("vLLM 推理原理…" generation flow, 结束请求并回收资源).

Policy choices the pages leave open (both this model and the C++ allocator
implement them, so block ids agree exactly):

* the free pool is a LIFO stack; its initial order is a Fisher-Yates shuffle
  of 0..N-1 driven by SplitMix64 (Vigna's published generator) from ``seed``;
  seed 0 keeps the identity order.  The first block handed out is perm[0].
* a freed sequence pushes its blocks last-to-first, so the next pops return
  them in logical order;
* copy-on-write is whole-block: a writer that finds its partially filled last
  block shared (refcount > 1) takes a fresh block, the old block's count drops
  by one and the pair (old, new) is reported for the device copy.  The last
  holder (refcount 1) writes in place, so n sharers cause n - 1 copies;
* sequence ids count up from 0.

Prefix caching ("vLLM 推理原理…" section 前缀缓存能省掉哪部分工作: requests that begin with the
same text reuse the common prefix's KV, on an exact match only):

* each full block of a prompt inserted with ``new_seq_prefix`` is registered under the key
  (predecessor block, predecessor's generation, the block's tokens); a new prompt walks its
  full blocks from the first, sharing each block whose key is registered, and stops at the
  first miss; the rest are fresh blocks, the full ones registered in turn;
* a registered block whose count drops to zero stays registered and joins the end of an
  eviction queue; when the free pool is empty a block is taken from the front of that queue,
  its key is dropped and its generation incremented (keys naming it as predecessor can no
  longer match); a hit on a queued block takes it out of the queue.
"""
from __future__ import annotations

from dataclasses import dataclass, field

MASK64 = (1 << 64) - 1


class OutOfBlocks(Exception):
    """The free pool cannot satisfy the request; the state is unchanged."""


def splitmix64_stream(seed: int):
    """SplitMix64 (S. Vigna, 2015): state += golden gamma; three xor-shift-multiply rounds."""
    state = seed & MASK64
    while True:
        state = (state + 0x9E3779B97F4A7C15) & MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        yield z ^ (z >> 31)


def seeded_block_order(n: int, seed: int) -> list[int]:
    """Initial free-pool order: identity for seed 0, else Fisher-Yates (i from n-1 down to 1,
    j = next() mod (i + 1))."""
    order = list(range(n))
    if seed == 0:
        return order
    rng = splitmix64_stream(seed)
    for i in range(n - 1, 0, -1):
        j = next(rng) % (i + 1)
        order[i], order[j] = order[j], order[i]
    return order


@dataclass
class Seq:
    blocks: list = field(default_factory=list)
    length: int = 0


class AllocatorModel:
    def __init__(self, num_blocks: int, block_size: int, seed: int = 0):
        self.num_blocks = num_blocks
        self.bs = block_size
        order = seeded_block_order(num_blocks, seed)
        self.free = list(reversed(order))       # pop() from the end yields order[0] first
        self.refcnt = [0] * num_blocks
        self.seqs: dict[int, Seq] = {}
        self.next_id = 0
        self.cache: dict = {}                   # (parent, parent_gen, tokens) -> block
        self.key_of: dict = {}                  # block -> its key
        self.gen = [0] * num_blocks
        self.evict_queue: list = []             # registered blocks with count 0, oldest first
        self.hit_tokens = 0
        self.miss_tokens = 0

    # -- pool ----------------------------------------------------------------
    def available(self) -> int:
        return len(self.free) + len(self.evict_queue)

    def _take(self) -> int:
        if self.free:
            b = self.free.pop()
        else:
            b = self.evict_queue.pop(0)
            del self.cache[self.key_of.pop(b)]
            self.gen[b] += 1
        assert self.refcnt[b] == 0
        self.refcnt[b] = 1
        return b

    def _release(self, b: int) -> None:
        self.refcnt[b] -= 1
        if self.refcnt[b] == 0:
            if b in self.key_of:
                self.evict_queue.append(b)
            else:
                self.free.append(b)

    # -- sequence operations -------------------------------------------------
    def new_seq(self) -> int:
        sid = self.next_id
        self.next_id += 1
        self.seqs[sid] = Seq()
        return sid

    def _blocks_needed(self, s: Seq, n: int) -> tuple[int, bool]:
        """Fresh blocks for n appended tokens, and whether the first write needs a CoW copy."""
        new_blocks = -(-(s.length + n) // self.bs) - len(s.blocks)
        cow = (n > 0 and s.length % self.bs != 0 and self.refcnt[s.blocks[-1]] > 1)
        return new_blocks + (1 if cow else 0), cow

    def append_n(self, sid: int, n: int):
        """Grow sequence sid by n tokens.  Returns (slots, (cow_src, cow_dst)) with (-1, -1)
        when no copy is needed."""
        s = self.seqs[sid]
        need, cow = self._blocks_needed(s, n)
        if need > self.available():
            raise OutOfBlocks()
        pair = (-1, -1)
        if cow:
            old = s.blocks[-1]
            new = self._take()
            self.refcnt[old] -= 1          # other holders keep it, so it cannot reach 0 here
            s.blocks[-1] = new
            pair = (old, new)
        slots = []
        for _ in range(n):
            pos = s.length
            if pos % self.bs == 0:
                s.blocks.append(self._take())
            slots.append(s.blocks[pos // self.bs] * self.bs + pos % self.bs)
            s.length += 1
        return slots, pair

    def append_slot(self, sid: int):
        slots, pair = self.append_n(sid, 1)
        return slots[0], pair

    def new_seq_prefix(self, tokens):
        """A sequence holding the prompt `tokens`; returns (sid, slots, cached_tokens)."""
        bs = self.bs
        n = len(tokens)
        full, total = n // bs, -(-n // bs)
        hits = []
        parent, pgen = -1, 0
        for k in range(full):
            key = (parent, pgen, tuple(tokens[k * bs:(k + 1) * bs]))
            if key not in self.cache:
                break
            b = self.cache[key]
            hits.append(b)
            parent, pgen = b, self.gen[b]
        queued_hits = sum(1 for b in hits if self.refcnt[b] == 0)
        if total - len(hits) > self.available() - queued_hits:
            raise OutOfBlocks()
        s = Seq()
        for b in hits:
            if self.refcnt[b] == 0:
                self.evict_queue.remove(b)
            self.refcnt[b] += 1
            s.blocks.append(b)
        for k in range(len(hits), total):
            b = self._take()
            s.blocks.append(b)
            if k < full:
                prev = s.blocks[k - 1] if k > 0 else -1
                key = (prev, self.gen[prev] if k > 0 else 0, tuple(tokens[k * bs:(k + 1) * bs]))
                assert key not in self.cache
                self.cache[key] = b
                self.key_of[b] = key
        s.length = n
        sid = self.next_id
        self.next_id += 1
        self.seqs[sid] = s
        cached = len(hits) * bs
        self.hit_tokens += cached
        self.miss_tokens += n - cached
        slots = [s.blocks[t // bs] * bs + t % bs for t in range(n)]
        return sid, slots, cached

    def prefix_stats(self):
        return {"hit_tokens": self.hit_tokens, "miss_tokens": self.miss_tokens, "cached_blocks": len(self.cache),
                "evictable": len(self.evict_queue)}

    def order_by_prefix(self, sids):
        """Batch order with sharers adjacent: indices sorted by block list, ties in input order."""
        return sorted(range(len(sids)), key=lambda i: (self.seqs[sids[i]].blocks, i))

    def fork(self, parent: int) -> int:
        p = self.seqs[parent]
        cid = self.new_seq()
        c = self.seqs[cid]
        c.blocks = list(p.blocks)
        c.length = p.length
        for b in c.blocks:
            self.refcnt[b] += 1
        return cid

    def free_seq(self, sid: int) -> None:
        s = self.seqs.pop(sid)
        for b in reversed(s.blocks):
            self._release(b)

    # -- views -----------------------------------------------------------------
    def block_table(self, sids, max_blocks: int):
        table = [[-1] * max_blocks for _ in sids]
        lens = []
        for r, sid in enumerate(sids):
            s = self.seqs[sid]
            if len(s.blocks) > max_blocks:
                raise ValueError("sequence %d needs %d blocks > %d" % (sid, len(s.blocks), max_blocks))
            table[r][:len(s.blocks)] = s.blocks
            lens.append(s.length)
        return table, lens

    def stats(self):
        used = sum(1 for c in self.refcnt if c > 0)
        shared = sum(1 for c in self.refcnt if c > 1)
        frag = sum(len(s.blocks) * self.bs - s.length for s in self.seqs.values())
        return {"free": self.available(), "used": used, "shared": shared, "frag_tokens": frag}

    def check_invariants(self) -> None:
        """Conservation and refcount consistency (the properties the tests assert)."""
        holders = [0] * self.num_blocks
        for s in self.seqs.values():
            assert len(s.blocks) == -(-s.length // self.bs)
            for b in s.blocks:
                holders[b] += 1
        assert holders == self.refcnt
        assert len(set(self.free)) == len(self.free)
        assert all(self.refcnt[b] == 0 for b in self.free)
        assert all(self.refcnt[b] == 0 and b in self.key_of for b in self.evict_queue)
        assert not set(self.free) & set(self.key_of)
        assert all(self.cache[k] == b for b, k in self.key_of.items()) and len(self.cache) == len(self.key_of)
        assert self.available() + sum(1 for c in self.refcnt if c > 0) == self.num_blocks
