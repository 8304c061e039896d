"""The tcgen05 prefill kernel's barrier protocol (prefill_tc.cuh), model-checked on the CPU.

Roles, as the kernel runs them for one CTA (two 128-row query tiles q = 0, 1):
  * K producer / V producer warps: tile it goes to slot it % ST after the slot's empty barrier
    completed phase it / ST - 1; its data lands later (the full barrier completes then);
  * one MMA thread per query tile: S_j needs K_j and (j > 0) s_free phase j - 1; P V_j needs V_j
    and p_full phase j >> 1 of barrier j & 1 (two barriers, one P buffer); completions arrive on s_full / k_empty and o_done /
    v_empty in issue order (tcgen05.commit); past its KV range the thread releases each K and V
    slot as its data lands;
  * four softmax warps per query tile: first write the tile's Q rows to shared memory (and the
    first 64 dims of them to tensor memory) and arrive q_full (the MMA thread waits for it before
    S_0); then wait s_full phase j, load S_j, arrive s_free; sometimes
    rescale O (wait o_done of P V_{j-1}); on the context's last tile wait V_j (zeroing rows);
    before storing P_j wait o_done of P V_{j-1}; arrive p_full; at the end wait o_done of the
    last P V and read O.
An mbarrier parity wait for phase k passes when the number of completed phases has a parity
other than k's, so it is only sound if that number is k or k + 1 whenever the wait is tried:
k - 1 would pass early, k + 2 would never pass.  The model runs random interleavings and checks
that every wait respects this, that every role finishes without deadlock, and that no shared
buffer is overwritten while an operation still reads it or read before it holds the right tile
(K / V slots, S, the P buffer, O).

The wait before storing P_j (for P V_{j-1}) is not implied by the others: S_j's commit is issued
before P V_{j-1} on the MMA thread (S_j overlaps softmax j - 1), so a softmax that has S_j knows
nothing of P V_{j-1}; a planted mistake that drops the wait is caught.  (With two P buffers the
wait was for P V_{j-2}, which S_j's commit did imply.)
"""
import inspect
import random
import textwrap

import pytest


class Violation(AssertionError):
    pass


def check(cond, msg):
    if not cond:
        raise Violation(msg)


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, count, 0

    def arrive(self):
        self.pending -= 1
        check(self.pending >= 0, "more arrivals than the barrier's count in one phase")
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


def run(nkv_q, KST, VST, seed, ctx_last_tile=True, rescale_p=0.2, abort_p=0.0, bad=None):
    """One CTA; nkv_q[q] = KV tiles of query tile q (as the kernel's nkv_of computes them).
    abort_p: chance per scheduling step that some role raises the CTA's abort flag (a timeout);
    bad = (is_v, tile): that producer finds a bad block-table entry there."""
    rnd = random.Random(seed)
    NQ = len(nkv_q)
    nkv = max(nkv_q)
    abort = [False]
    k_full = [Bar(1) for _ in range(KST)]
    k_empty = [Bar(NQ) for _ in range(KST)]
    v_full = [Bar(1) for _ in range(VST)]
    v_empty = [Bar(NQ) for _ in range(VST)]
    s_full = [Bar(1) for _ in range(NQ)]
    s_free = [Bar(4) for _ in range(NQ)]
    p_full = [Bar(4) for _ in range(2 * NQ)]
    o_done = [Bar(1) for _ in range(2 * NQ)]
    q_full = [Bar(4) for _ in range(NQ)]
    # data state
    kslot, vslot = [None] * KST, [None] * VST              # tile whose data sits in the slot
    kread, vread = [set() for _ in range(KST)], [set() for _ in range(VST)]   # pending MMA readers
    qrows = [set() for _ in range(NQ)]                     # softmax warps whose Q rows are written
    sbuf = [None] * NQ                                     # tile of the completed S product
    s_pending = [False] * NQ                               # an S product is writing S
    sloaded = [[-1] * 4 for _ in range(NQ)]                # last S tile each softmax warp loaded
    pbuf = [[None] * 4 for _ in range(NQ)]                 # tile of P each warp stored (one buffer)
    pread = [0] * NQ                                       # pending P V reading the P buffer
    pv_pending = [0] * NQ                                  # pending P V (writes O)
    inflight = []                                          # (kind, slot, tile) still landing
    tc_queue = [[] for _ in range(NQ)]                     # per MMA thread: completions in order

    def sound(bar, k):
        check(bar.done in (k, k + 1), "wait for phase %d with %d phases completed" % (k, bar.done))
        return bar.done == k + 1

    # a role yields (barrier, phase, ends_on_abort) and gets back True (passed) or False (the
    # abort flag ended the wait); ("drain", q) waits until MMA thread q has nothing pending
    def producer(is_v, ST):
        full, empty = (v_full, v_empty) if is_v else (k_full, k_empty)
        slot, readers = (vslot, vread) if is_v else (kslot, kread)
        issued = 0
        for it in range(nkv):
            st = it % ST
            if it >= ST and not (yield (empty[st], it // ST - 1, True)):
                break
            if abort[0]:
                break
            if bad == (is_v, it):
                abort[0] = True                            # record, stop; no copy for this tile
                break
            check(not readers[st], "slot %d refilled while an MMA still reads tile %s" % (st, slot[st]))
            slot[st] = None                                # being overwritten
            inflight.append((is_v, st, it))
            issued += 1
        # the kernel waits for its last ring's worth of tiles before leaving
        for i in range(max(0, issued - ST), issued):
            yield (full[i % ST], i // ST, False)
        check(all(x[0] != is_v for x in inflight), "producer leaves with copies in flight")

    def mma(q):
        nkq = nkv_q[q]

        def s_mma(j):
            st = j % KST
            if not (yield (k_full[st], j // KST, True)) or abort[0]:
                return False
            if j >= 1:
                if not (yield (s_free[q], j - 1, True)) or abort[0]:
                    return False
                check(all(x == j - 1 for x in sloaded[q]), "S_%d issued before every warp loaded S_%d" % (j, j - 1))
            check(len(qrows[q]) == 4, "S_%d reads Q before every warp wrote its rows" % j)
            check(kslot[st] == j, "S_%d reads slot %d holding %s" % (j, st, kslot[st]))
            kread[st].add((q, j))
            s_pending[q] = True

            def done():
                kread[st].discard((q, j))
                s_pending[q] = False
                sbuf[q] = j
                s_full[q].arrive()
                k_empty[st].arrive()
            tc_queue[q].append(done)
            return True

        def pv(i):
            st, b = i % VST, i & 1
            if not (yield (v_full[st], i // VST, True)) or abort[0]:
                return False
            if not (yield (p_full[2 * q + b], i >> 1, True)) or abort[0]:
                return False
            check(vslot[st] == i, "P V_%d reads V slot %d holding %s" % (i, st, vslot[st]))
            check(all(x == i for x in pbuf[q]), "P V_%d reads P holding %s" % (i, pbuf[q]))
            vread[st].add((q, i))
            pread[q] += 1
            pv_pending[q] += 1

            def done():
                vread[st].discard((q, i))
                pread[q] -= 1
                pv_pending[q] -= 1
                o_done[2 * q + b].arrive()
                v_empty[st].arrive()
            tc_queue[q].append(done)
            return True

        ok = True
        if nkq > 0:
            ok = (yield (q_full[q], 0, True)) and not abort[0]
            if ok:
                ok = yield from s_mma(0)
        for j in range(nkq):
            if not ok:
                break
            if j + 1 < nkq:
                ok = yield from s_mma(j + 1)
            if ok:
                ok = yield from pv(j)
        for j in range(nkq, nkv):
            if not ok:
                break
            ok = (yield (k_full[j % KST], j // KST, True)) and not abort[0]
            if ok:
                k_empty[j % KST].arrive()
                ok = (yield (v_full[j % VST], j // VST, True)) and not abort[0]
            if ok:
                v_empty[j % VST].arrive()
        if not ok:
            abort[0] = True
        yield ("drain", q)                                 # every MMA this thread issued finished
        check(not tc_queue[q], "MMA thread leaves with products pending")

    def softmax(q, w):
        n = nkv_q[q]
        qrows[q].add(w)
        q_full[q].arrive()
        for j in range(n):
            if not (yield (s_full[q], j, True)) or abort[0]:
                return
            check(sbuf[q] == j and not s_pending[q], "warp loads S_%d while S holds %s" % (j, sbuf[q]))
            sloaded[q][w] = j
            s_free[q].arrive()
            if j > 0 and rnd.random() < rescale_p:
                if not (yield (o_done[2 * q + ((j - 1) & 1)], (j - 1) >> 1, True)) or abort[0]:
                    return
                check(pv_pending[q] == 0, "O rescaled while a P V is pending")
            if ctx_last_tile and j == nkv - 1:
                if not (yield (v_full[j % VST], j // VST, True)):
                    return
                check(vslot[j % VST] == j, "zeroing rows of V_%d in the wrong slot contents" % j)
            b = j & 1
            if j >= 1:
                if not (yield (o_done[2 * q + ((j - 1) & 1)], (j - 1) >> 1, True)) or abort[0]:
                    return
            check(pread[q] == 0, "P_%d stored while a P V reads the P buffer" % j)
            pbuf[q][w] = j
            p_full[2 * q + b].arrive()
        if n > 0:
            if (yield (o_done[2 * q + ((n - 1) & 1)], (n - 1) >> 1, True)) and not abort[0]:
                check(pv_pending[q] == 0, "O read while a P V is pending")

    roles = [producer(False, KST), producer(True, VST)]
    roles += [mma(q) for q in range(NQ)]
    roles += [softmax(q, w) for q in range(NQ) for w in range(4)]
    waiting = [None] * len(roles)
    started = [False] * len(roles)
    alive = set(range(len(roles)))

    def step(r):
        """Advance role r until it blocks or ends; True if it made progress."""
        progressed = False
        while True:
            val = None
            if waiting[r] is not None:
                if waiting[r][0] == "drain":
                    if tc_queue[waiting[r][1]]:
                        return progressed
                    val = True
                else:
                    bar, k, ends_on_abort = waiting[r]
                    if sound(bar, k):
                        val = True
                    elif ends_on_abort and abort[0]:
                        val = False
                    else:
                        return progressed
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
        if abort_p and not abort[0] and rnd.random() < abort_p:
            abort[0] = True
        choices = [("role", r) for r in sorted(alive)]
        if inflight:
            choices.append(("land", None))
        choices += [("tc", q) for q in range(NQ) if tc_queue[q]]
        kind, arg = rnd.choice(choices)
        if kind == "role":
            step(arg)
        elif kind == "land":
            is_v, st, it = inflight.pop(rnd.randrange(len(inflight)))
            (vslot if is_v else kslot)[st] = it
            (v_full if is_v else k_full)[st].arrive()
        else:
            tc_queue[arg].pop(0)()                          # one thread's completions in issue order
        if not inflight and not any(tc_queue) and alive:
            if not any(step(r) for r in sorted(alive)) and alive:
                raise Violation("deadlock: %d roles blocked" % len(alive))
    if not abort[0]:
        for b in k_empty + v_empty + s_free + p_full + q_full:
            check(b.pending == b.count, "a barrier was left with partial arrivals")
    return True


def tile_counts(ctx, chunk, pair, TQ=32, BN=64, NQ=2):
    """nkv_of(q) as the kernel computes it."""
    out = []
    for q in range(NQ):
        t0 = (pair * NQ + q) * TQ
        out.append(0 if t0 >= chunk else -(-(ctx - chunk + min(chunk, t0 + TQ)) // BN))
    return out


@pytest.mark.parametrize("KST,VST", [(4, 4), (3, 3), (2, 2), (5, 5), (4, 2)])
def test_protocol_sound_race_free_and_deadlock_free(KST, VST):
    rnd = random.Random(KST * 10 + VST)
    cases = 0
    while cases < 50:
        chunk = rnd.randint(1, 300)
        ctx = chunk + rnd.randint(0, 400)
        npairs = (-(-chunk // 32) + 1) // 2
        n = tile_counts(ctx, chunk, rnd.randrange(npairs))
        if max(n) == 0:
            continue
        for seed in range(4):
            assert run(n, KST, VST, seed=1000 * cases + seed)
        cases += 1


def test_second_tile_missing_and_short_ranges():
    # an odd number of query tiles leaves the last pair with one tile (nkv_of(1) == 0)
    for n in ([1, 0], [3, 0], [1, 1], [1, 2], [7, 8], [9, 9]):
        for seed in range(20):
            assert run(list(n), 4, 4, seed)


def _mutant(old, new):
    text = textwrap.dedent(inspect.getsource(run))
    assert text.count(old) == 1, old
    ns = {}
    exec(compile(text.replace(old, new), "<mutant>", "exec"), run.__globals__, ns)
    return ns["run"]


@pytest.mark.parametrize("old,new", [
    # the softmax stores P_j without waiting for P V_{j-1}, which may still read the P buffer
    ("            if j >= 1:\n                if not (yield (o_done[2 * q + ((j - 1) & 1)], (j - 1) >> 1, True)) or abort[0]:\n                    return\n            check(pread",
     "            check(pread"),
    # ... or after P V_{j-2} only (the rule for two P buffers)
    ("            if j >= 1:\n                if not (yield (o_done[2 * q + ((j - 1) & 1)], (j - 1) >> 1, True)) or abort[0]:\n                    return\n            check(pread",
     "            if j >= 2:\n                if not (yield (o_done[2 * q + b], (j - 2) >> 1, True)) or abort[0]:\n                    return\n            check(pread"),
    # O rescaled after waiting for P V_{j-2} instead of P V_{j-1} (P V_{j-1} may still be adding)
    ("            if j > 0 and rnd.random() < rescale_p:\n                if not (yield (o_done[2 * q + ((j - 1) & 1)], (j - 1) >> 1, True)) or abort[0]:",
     "            if j > 0 and rnd.random() < rescale_p:\n                if not (yield (o_done[2 * q + (j & 1)], max(j - 2, 0) >> 1, True)) or abort[0]:"),
    # a K slot is released after one query tile's S instead of both
    ("k_empty = [Bar(NQ) for _ in range(KST)]", "k_empty = [Bar(1) for _ in range(KST)]"),
    # S_0 issued without waiting for the softmax warps' Q rows
    ("            ok = (yield (q_full[q], 0, True)) and not abort[0]\n", "            ok = True\n"),
    # S_{j+1} issued without waiting for the softmax to have loaded S_j
    ("            if j >= 1:\n                if not (yield (s_free[q], j - 1, True)) or abort[0]:\n                    return False\n",
     "            if False:\n                pass\n"),
])
def test_model_catches_planted_mistakes(old, new):
    bad = _mutant(old, new)
    with pytest.raises(Violation):
        for seed in range(200):
            bad([6, 7], 4, 4, seed)


@pytest.mark.parametrize("KST,VST", [(4, 4), (3, 3), (2, 2)])
def test_abort_paths_drain_and_end(KST, VST):
    # a timeout raised at a random moment, or a bad block-table entry met by either producer at
    # any tile: every role still finishes, the drains' parity waits are sound, no copy is in
    # flight when a producer leaves and no MMA is pending when an MMA thread leaves
    rnd = random.Random(7 * KST + VST)
    for case in range(40):
        chunk = rnd.randint(1, 300)
        ctx = chunk + rnd.randint(0, 400)
        npairs = (-(-chunk // 32) + 1) // 2
        n = tile_counts(ctx, chunk, rnd.randrange(npairs))
        if max(n) == 0:
            continue
        for seed in range(3):
            assert run(n, KST, VST, seed=100 * case + seed, abort_p=0.01)
            bad = (rnd.random() < 0.5, rnd.randrange(max(n)))
            assert run(n, KST, VST, seed=100 * case + seed + 50, bad=bad)


def test_model_catches_a_missing_drain():
    # the producer leaves without waiting for its last tiles: copies may still be landing
    bad = _mutant("        for i in range(max(0, issued - ST), issued):\n            yield (full[i % ST], i // ST, False)\n", "")
    with pytest.raises(Violation):
        for seed in range(300):
            bad([6, 7], 4, 4, seed, abort_p=0.02)
