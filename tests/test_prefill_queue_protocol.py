"""The work-queue form of the tcgen05 prefill kernel (prefill_tc.cuh), model-checked on the CPU:
one CTA processing a sequence of work items.

Beyond the one-item protocol (tests/test_prefill_protocol.py) the queue adds:
  * the K producer warp publishes items through a two-entry ring (item_full / item_empty; every
    reading warp arrives on item_empty once per item) and publishes the next item once it has
    issued the current item's last K tile;
  * the K / V rings, the S, P and O barriers are counted across items;
  * a query tile's softmax warps copy its Q rows for each item that has work for the tile and
    arrive on q_full (four arrivals); the MMA thread waits q_full before that item's first S.
    Items without work for the tile use neither side of q_full;
  * each softmax warp also writes its rows of Q's first 64 dims into tensor memory (the A
    operand of the first four k-steps of S) right before it arrives on q_full;
  * a query tile that lies wholly inside its chunk is not copied by the softmax warps: the K
    producer loads it with one TMA (landing on q_land) at the start of the item, once both query
    tiles have released the previous item's last K tile, and the softmax warps wait for q_land
    (also before the epilogue, without waiting, to announce the next item's tile early);
  * one P buffer per tile: before storing P of step g a softmax warp waits for P V of step g - 1;
  * once an item's last S product of the tile is done, each softmax warp checks (without
    waiting) whether the next item is published and, if it has work for the tile, starts
    copying its Q rows, and after the item's last P V it arrives on q_full for that next item
    before its epilogue reads O (the next item's first S product then overlaps the epilogue);
  * an item's first P V overwrites O (no accumulate), after the softmax warps read the previous
    item's O.
The model runs random interleavings and checks that every parity wait is sound (the barrier has
completed k or k + 1 phases when a wait for phase k is tried), that nothing deadlocks, that an
S product reads Q holding its own item's rows from all four warps, that no Q copy starts and
no Q row is written to tensor memory while an S product still reads the tile, that P is not
overwritten while a P V reads it, that the first P V of an item starts only after the previous
item's O was read by all four warps, and that the K / V slots hold the tile each MMA expects.
"""
import inspect
import random
import textwrap

import pytest

from test_prefill_protocol import Bar, Violation, check


def run_items(items, KST, VST, seed, rescale_p=0.2, tma_p=0.6):
    """items: list of (nkv of query tile 0, nkv of query tile 1) for one CTA.  Each query tile of
    an item is, at random (tma_p), one that lies wholly inside its chunk (its Q tile comes by TMA
    from the K producer) or a ragged one (copied by the softmax warps)."""
    rnd = random.Random(seed)
    rfull = random.Random(seed * 31 + 7)
    q_slow = rfull.random() < 0.5
    full = [(rfull.random() < tma_p, rfull.random() < tma_p) for _ in items]
    NQ = 2
    READERS = 4 * NQ + NQ + 1
    k_full = [Bar(1) for _ in range(KST)]
    k_empty = [Bar(NQ) for _ in range(KST)]
    v_full = [Bar(1) for _ in range(VST)]
    v_empty = [Bar(NQ) for _ in range(VST)]
    s_full = [Bar(1) for _ in range(NQ)]
    s_free = [Bar(4) for _ in range(NQ)]
    p_full = [Bar(4) for _ in range(2 * NQ)]
    o_done = [Bar(1) for _ in range(2 * NQ)]
    q_full = [Bar(4) for _ in range(NQ)]
    q_land = [Bar(1) for _ in range(NQ)]                   # a Q tile loaded by TMA landed
    item_full = [Bar(1) for _ in range(2)]
    item_empty = [Bar(READERS) for _ in range(2)]
    ring = [None, None]
    kslot, vslot = [None] * KST, [None] * VST
    kread, vread = [set() for _ in range(KST)], [set() for _ in range(VST)]
    inflight = []
    tc_queue = [[] for _ in range(NQ)]
    qrows = [[None] * 4 for _ in range(NQ)]                # item whose rows each warp copied last
    q_reading = [0] * NQ                                   # pending S products reading Q
    sbuf = [None] * NQ
    s_pending = [False] * NQ
    sloaded = [[-1] * 4 for _ in range(NQ)]
    pbuf = [[None] * 4 for _ in range(NQ)]               # step whose P each warp stored (one P buffer)
    pread = [0] * NQ                                       # pending P V reading the P columns
    pv_pending = [0] * NQ
    o_item = [None] * NQ                                   # item whose P V sums are in O
    o_read = [set() for _ in range(NQ)]                    # warps that read O of o_item

    def sound(bar, k):
        check(bar.done in (k, k + 1), "wait for phase %d with %d phases completed" % (k, bar.done))
        return bar.done == k + 1

    def read_item(n):
        slot = n & 1
        yield (item_full[slot], n >> 1, False)
        it = ring[slot]
        item_empty[slot].arrive()
        return it

    def k_producer():
        published = 0

        def publish(it):
            nonlocal published
            slot = published & 1
            if published >= 2:
                yield (item_empty[slot], (published >> 1) - 1, False)
            ring[slot] = it
            item_full[slot].arrive()
            published += 1
        issued = 0
        yield from publish((0,) + items[0] if items else None)
        for idx, (a, b) in enumerate(items):
            nkv = max(a, b)
            nxt = (idx + 1,) + items[idx + 1] if idx + 1 < len(items) else None
            known = False
            # the item's whole query tiles by TMA, once both tiles released the previous item's
            # last K tile (every S product of that item has finished)
            if issued > 0:
                gl = issued - 1
                yield (k_empty[gl % KST], gl // KST, True)
            for q in range(NQ):
                if (a, b)[q] > 0 and full[idx][q]:
                    check(q_reading[q] == 0, "Q tile of item %d loaded while an S product reads the tile" % idx)
                    inflight.append(("q", q, idx))
            for t in range(nkv):
                st = issued % KST
                if issued >= KST:
                    yield (k_empty[st], issued // KST - 1, True)
                check(not kread[st], "K slot %d refilled while read" % st)
                kslot[st] = None
                inflight.append((False, st, issued))
                issued += 1
                if not known and t == nkv - 1:
                    yield from publish(nxt)
                    known = True
            if not known:
                yield from publish(nxt)
        for i in range(max(0, issued - KST), issued):
            yield (k_full[i % KST], i // KST, False)

    def v_producer():
        issued = 0
        n = 0
        while True:
            it = yield from read_item(n)
            if it is None:
                break
            for t in range(max(it[1], it[2])):
                st = issued % VST
                if issued >= VST:
                    yield (v_empty[st], issued // VST - 1, True)
                check(not vread[st], "V slot %d refilled while read" % st)
                vslot[st] = None
                inflight.append((True, st, issued))
                issued += 1
            n += 1
        for i in range(max(0, issued - VST), issued):
            yield (v_full[i % VST], i // VST, False)

    def mma(q):
        gk = gs = nq = 0
        n = 0
        while True:
            it = yield from read_item(n)
            if it is None:
                break
            item, nkq, nkv = it[0], it[1 + q], max(it[1], it[2])

            def s_mma(j):
                gt, gj = gk + j, gs + j
                st = gt % KST
                yield (k_full[st], gt // KST, True)
                if gj >= 1:
                    yield (s_free[q], gj - 1, True)
                    check(all(x == gj - 1 for x in sloaded[q]), "S issued before every warp loaded the previous S")
                check(kslot[st] == gt, "S reads K slot %d holding %s, wants %d" % (st, kslot[st], gt))
                check(all(r == item for r in qrows[q]), "S of item %d reads Q rows %s" % (item, qrows[q]))
                kread[st].add((q, gj))
                q_reading[q] += 1
                s_pending[q] = True

                def done():
                    kread[st].discard((q, gj))
                    q_reading[q] -= 1
                    s_pending[q] = False
                    sbuf[q] = gj
                    s_full[q].arrive()
                    k_empty[st].arrive()
                tc_queue[q].append(done)

            def pv(i):
                gt, gi = gk + i, gs + i
                st, b = gt % VST, gi & 1
                yield (v_full[st], gt // VST, True)
                yield (p_full[2 * q + b], gi >> 1, True)
                check(vslot[st] == gt, "P V reads V slot %d holding %s, wants %d" % (st, vslot[st], gt))
                check(all(x == gi for x in pbuf[q]), "P V %d reads P holding %s" % (gi, pbuf[q]))
                if i == 0:
                    check(o_item[q] is None or len(o_read[q]) == 4,
                          "item %d overwrites O before item %s's O was read" % (item, o_item[q]))
                    o_item[q] = item
                    o_read[q] = set()
                vread[st].add((q, gi))
                pread[q] += 1
                pv_pending[q] += 1

                def done():
                    vread[st].discard((q, gi))
                    pread[q] -= 1
                    pv_pending[q] -= 1
                    o_done[2 * q + b].arrive()
                    v_empty[st].arrive()
                tc_queue[q].append(done)

            if nkq > 0:
                yield (q_full[q], nq, True)
                nq += 1
                yield from s_mma(0)
            for j in range(nkq):
                if j + 1 < nkq:
                    yield from s_mma(j + 1)
                yield from pv(j)
            for j in range(nkq, nkv):
                gt = gk + j
                yield (k_full[gt % KST], gt // KST, True)
                k_empty[gt % KST].arrive()
                yield (v_full[gt % VST], gt // VST, True)
                v_empty[gt % VST].arrive()
            gk += nkv
            gs += nkq
            n += 1
        yield ("drain", q)
        check(not tc_queue[q], "MMA thread leaves with products pending")

    def softmax(q, w):
        gs = 0
        n = 0
        copying = None                                     # item whose Q copy this warp started early
        announced = None                                   # ... and already arrived on q_full for

        def copy_q(item):
            check(q_reading[q] == 0, "Q rows of item %d copied while an S product reads the tile" % item)
            qrows[q][w] = item

        def announce_q():
            # the warp's rows of Q's first 64 dims go into tensor memory right before q_full
            check(q_reading[q] == 0, "Q written to tensor memory while an S product reads it")
            q_full[q].arrive()

        nqt = 0

        def announce_tma():
            # a whole tile: wait for its TMA load, then as announce_q
            nonlocal nqt
            yield (q_land[q], nqt, True)
            nqt += 1
            announce_q()

        while True:
            it = yield from read_item(n)
            if it is None:
                break
            item, nk = it[0], it[1 + q]
            if nk > 0 and announced != item:
                if full[item][q]:
                    yield from announce_tma()
                else:
                    if copying != item:
                        copy_q(item)
                    announce_q()
            copying = None
            announced = None
            for j in range(nk):
                gj = gs + j
                yield (s_full[q], gj, True)
                check(sbuf[q] == gj and not s_pending[q], "warp loads S %d while S holds %s" % (gj, sbuf[q]))
                sloaded[q][w] = gj
                s_free[q].arrive()
                if j > 0 and rnd.random() < rescale_p:
                    yield (o_done[2 * q + ((gj - 1) & 1)], (gj - 1) >> 1, True)
                    check(pv_pending[q] == 0, "O rescaled while a P V is pending")
                b = gj & 1
                if gj >= 1:
                    yield (o_done[2 * q + ((gj - 1) & 1)], (gj - 1) >> 1, True)
                check(pread[q] == 0, "P %d stored while a P V reads the P columns" % gj)
                pbuf[q][w] = gj
                p_full[2 * q + b].arrive()
            if nk > 0:
                ns = (n + 1) & 1
                if item_full[ns].done == ((n + 1) >> 1) + 1:        # published (test_wait, no waiting)
                    nx = ring[ns]
                    if nx is not None and nx[1 + q] > 0 and not full[nx[0]][q]:
                        copy_q(nx[0])
                        copying = nx[0]
                gl = gs + nk - 1
                yield (o_done[2 * q + (gl & 1)], gl >> 1, True)
                if copying is not None:                    # the next item's Q announced before the epilogue
                    announce_q()
                    announced = copying
                elif item_full[ns].done == ((n + 1) >> 1) + 1:     # likewise a whole tile whose load landed
                    nx = ring[ns]
                    if nx is not None and nx[1 + q] > 0 and full[nx[0]][q] and q_land[q].done == nqt + 1:
                        yield from announce_tma()
                        announced = nx[0]
                check(pv_pending[q] == 0 and o_item[q] == item, "O of item %d read too early" % item)
                o_read[q].add(w)
            gs += nk
            n += 1

    roles = [k_producer(), v_producer()] + [mma(q) for q in range(NQ)]
    roles += [softmax(q, w) for q in range(NQ) for w in range(4)]
    waiting = [None] * len(roles)
    started = [False] * len(roles)
    alive = set(range(len(roles)))

    def step(r):
        progressed = False
        while True:
            val = None
            if waiting[r] is not None:
                if waiting[r][0] == "drain":
                    if tc_queue[waiting[r][1]]:
                        return progressed
                    val = True
                else:
                    bar, k, _ = waiting[r]
                    if not sound(bar, k):
                        return progressed
                    val = True
                waiting[r] = None
                progressed = True
            try:
                waiting[r] = roles[r].send(val) if started[r] else next(roles[r])
                started[r] = True
                progressed = True
            except StopIteration:
                alive.discard(r)
                return True

    while alive or inflight or any(tc_queue):
        choices = [("role", r) for r in sorted(alive)]
        if inflight:
            choices.append(("land", None))
        choices += [("tc", q) for q in range(NQ) if tc_queue[q]]
        kind, arg = rnd.choice(choices)
        if kind == "role":
            step(arg)
        elif kind == "land":
            i = rnd.randrange(len(inflight))
            if inflight[i][0] == "q" and q_slow and rnd.random() < 0.95:
                continue                                   # in half the runs Q tiles land late
            what, st, tile = inflight.pop(i)
            if what == "q":                                # a Q tile: all four warps' rows
                qrows[st] = [tile] * 4
                q_land[st].arrive()
            else:
                (vslot if what else kslot)[st] = tile
                (v_full if what else k_full)[st].arrive()
        else:
            tc_queue[arg].pop(0)()
        if not inflight and not any(tc_queue) and alive:
            if not any(step(r) for r in sorted(alive)) and alive:
                raise Violation("deadlock: %d roles blocked" % len(alive))
    for b in k_empty + v_empty + s_free + p_full + q_full + item_empty:
        check(b.pending == b.count, "a barrier was left with partial arrivals")
    return True


def random_items(rnd, n):
    out = []
    for _ in range(n):
        a = rnd.choice([0, 1, 1, 2, 3, rnd.randint(1, 9)])
        b = rnd.choice([0, 0, a, a + 1, rnd.randint(0, 9)])
        if a == 0 and b == 0:
            a = 1
        out.append((a, b))
    return out


@pytest.mark.parametrize("KST,VST", [(4, 4), (2, 2), (3, 2)])
def test_queue_protocol_sound_race_free_and_deadlock_free(KST, VST):
    rnd = random.Random(KST * 7 + VST)
    for case in range(60):
        items = random_items(rnd, rnd.randint(1, 7))
        for seed in range(4):
            assert run_items(items, KST, VST, seed=1000 * case + seed)


def test_items_without_work_for_a_tile():
    # long runs of items that give query tile 1 nothing: its softmax warps must not run ahead
    for items in ([(1, 0)] * 6, [(2, 0), (1, 0), (3, 1), (1, 0), (1, 0)], [(1, 1)] * 5, [(0, 2), (1, 0)] * 3):
        for seed in range(40):
            assert run_items(list(items), 4, 4, seed)


def _mutant(old, new):
    text = textwrap.dedent(inspect.getsource(run_items))
    assert text.count(old) == 1, old
    ns = {}
    exec(compile(text.replace(old, new), "<mutant>", "exec"), run_items.__globals__, ns)
    return ns["run_items"]


@pytest.mark.parametrize("old,new", [
    # q_full used for every item (also without work): idle softmax warps run phases ahead
    ("            if nk > 0 and announced != item:\n                if full[item][q]:",
     "            if announced != item:\n                if full[item][q] and nk > 0:"),
    # the next item's Q copy started before this item's S products are done
    ("            if nk > 0:\n                ns = (n + 1) & 1\n",
     "            if True:\n                ns = (n + 1) & 1\n"),
    # the next item published before the slot's previous item was read by every warp
    ("            if published >= 2:\n                yield (item_empty[slot], (published >> 1) - 1, False)\n",
     "            if False:\n                yield (item_empty[slot], (published >> 1) - 1, False)\n"),
    # P stored without waiting for the previous step's P V, which may still read the P columns
    ("                if gj >= 1:\n                    yield (o_done[2 * q + ((gj - 1) & 1)], (gj - 1) >> 1, True)\n                check(pread",
     "                check(pread"),
    # the two-buffer rule (wait for P V of step g - 2) with one buffer
    ("                if gj >= 1:\n                    yield (o_done[2 * q + ((gj - 1) & 1)], (gj - 1) >> 1, True)\n                check(pread",
     "                if gj >= 2:\n                    yield (o_done[2 * q + b], (gj - 2) >> 1, True)\n                check(pread"),
    # a whole Q tile loaded by the K producer before the previous item's S products finished
    ("            if issued > 0:\n                gl = issued - 1\n                yield (k_empty[gl % KST], gl // KST, True)\n", ""),
    # a whole Q tile announced without waiting for its load to land
    ("            yield (q_land[q], nqt, True)\n", "            if False:\n                yield\n"),
    # the epilogue reads O (and the next item's Q is announced) without waiting for the item's
    # last P V
    ("                gl = gs + nk - 1\n                yield (o_done[2 * q + (gl & 1)], gl >> 1, True)\n                if copying is not None:",
     "                gl = gs + nk - 1\n                if copying is not None:"),
])
def test_model_catches_planted_mistakes(old, new):
    bad = _mutant(old, new)
    rnd = random.Random(5)
    with pytest.raises(Violation):
        for seed in range(300):
            bad([(1, 0), (2, 0), (1, 0), (3, 2), (1, 0), (2, 2)] if seed % 2 else random_items(rnd, 6), 4, 4, seed)
