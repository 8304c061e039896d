"""The decode kernels' shared-memory stage ring (CPU only).

A producer warp fills stage i % STAGES for block i; consumer warp w takes blocks
i = w (mod NW) and waits with mbarrier parity waits.  A parity wait passes when the
barrier's current phase parity differs from the awaited one, so it is only sound when the
barrier cannot still be in the previous phase: i.e. when block i - STAGES (same stage)
belongs to the same consumer warp, i.e. STAGES % NW == 0.  This test (1) model-checks the
protocol under random interleavings, showing early passes for a non-multiple and none for
multiples, and (2) checks every stage count the library's kernel configurations produce."""
import os
import random
import subprocess
import tempfile
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent


def _ring(stages, nw, nblk, seed):
    rnd = random.Random(seed)
    full_done, empty_done = [0] * stages, [0] * stages
    landed, consumed, inflight = set(), set(), []
    prod, nxt = 0, list(range(nw))
    passes = lambda done, k: (done & 1) != (k & 1)          # mbarrier try_wait.parity
    for _ in range(200000):
        if len(consumed) == nblk:
            return "ok"
        a = rnd.randrange(nw + 2)
        if a == nw and prod < nblk:
            s = prod % stages
            if prod < stages or passes(empty_done[s], prod // stages - 1):
                inflight.append(prod)
                prod += 1
        elif a == nw + 1 and inflight:
            b = inflight.pop(rnd.randrange(len(inflight)))
            landed.add(b)
            full_done[b % stages] += 1
        elif a < nw:
            i = nxt[a]
            if i < nblk and passes(full_done[i % stages], i // stages):
                if i not in landed:
                    return "early"
                consumed.add(i)
                empty_done[i % stages] += 1
                nxt[a] += nw
    return "stuck"


def test_protocol_model():
    assert any(_ring(6, 4, 40, s) == "early" for s in range(200))       # the hazard exists
    for stages, nw in [(4, 4), (8, 4), (12, 4), (16, 4), (8, 2), (8, 8)]:
        assert all(_ring(stages, nw, 40, s) == "ok" for s in range(200)), (stages, nw)


PROBE = r'''
#include <cstdio>
#include "decode.cuh"
#include "decode_mma.cuh"
using namespace pa;
template <int D, int BS, int G, bool F> void simt() { using C = DecodeConfig<D, BS, G, F>; printf("%d %d\n", C::STAGES, C::NW); }
template <int D, int BS, int G> void mma() { using C = MmaDecodeConfig<D, BS, G>; printf("%d %d\n", C::STAGES, C::NW); }
template <int D, int BS> void all() {
  simt<D, BS, 1, false>(); simt<D, BS, 4, false>(); simt<D, BS, 8, true>(); simt<D, BS, 1, true>();
  mma<D, BS, 1>(); mma<D, BS, 4>(); mma<D, BS, 8>(); }
int main() { all<64, 16>(); all<64, 32>(); all<64, 64>(); all<128, 16>(); all<128, 32>(); all<128, 64>(); }
'''


def test_library_stage_counts_are_multiples_of_consumer_warps():
    with tempfile.TemporaryDirectory() as tmp:
        src = Path(tmp) / "probe.cu"
        src.write_text(PROBE)
        exe = Path(tmp) / "probe"
        nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
        subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", str(ROOT / "include"), "-I",
                        str(ROOT / "paged_kv_cache_428_b200" / "csrc"), str(src), "-o", str(exe)],
                       check=True, capture_output=True)
        rows = [tuple(map(int, l.split())) for l in subprocess.run([str(exe)], capture_output=True, text=True,
                                                                    check=True).stdout.split("\n") if l.strip()]
    assert len(rows) == 6 * 7
    for stages, nw in rows:
        assert stages % nw == 0 and stages >= nw, (stages, nw)


def _ring_all_heads(stages, nw, nunits, seed, count=None):
    """The whole-block kernel's ring: unit k's K goes to use j = 2k and its V to j = 2k + 1,
    stage j % stages; every consumer warp consumes every use in order and the stage's empty
    barrier completes a phase after `count` (all nw) warps arrived."""
    count = nw if count is None else count
    rnd = random.Random(seed)
    nuse = 2 * nunits
    full_done, empty_done, arrivals = [0] * stages, [0] * stages, [0] * stages
    landed, inflight = set(), []
    prod, nxt = 0, [0] * nw
    passes = lambda done, k: (done & 1) != (k & 1)
    for _ in range(400000):
        if all(n == nuse for n in nxt):
            return "ok"
        a = rnd.randrange(nw + 2)
        if a == nw and prod < nuse:
            s = prod % stages
            if prod < stages or passes(empty_done[s], prod // stages - 1):
                if any(n <= prod - stages for n in nxt):
                    return "overwrite"                      # a warp still reads the stage's last use
                inflight.append(prod)
                prod += 1
        elif a == nw + 1 and inflight:
            j = inflight.pop(rnd.randrange(len(inflight)))
            landed.add(j)
            full_done[j % stages] += 1
        elif a < nw:
            j = nxt[a]
            if j < nuse and passes(full_done[j % stages], j // stages):
                if j not in landed:
                    return "early"
                s = j % stages
                arrivals[s] += 1
                if arrivals[s] == count:
                    arrivals[s] = 0
                    empty_done[s] += 1
                nxt[a] += 1
    return "stuck"


def test_whole_block_ring_protocol_model():
    """Every stage count the whole-block kernel instantiates (3, 6, 12: 64, 32 and 16 KB
    stages in a 192 KB ring), with its 8 consumer warps: no early pass, no deadlock.  An
    empty barrier initialised for one arrival instead of eight lets the producer refill a
    stage a slower warp still reads, and the model sees it (an overwrite or an early pass)."""
    assert any(_ring_all_heads(6, 8, 30, s, count=1) in ("early", "overwrite") for s in range(200))
    for stages in (3, 6, 12):
        assert all(_ring_all_heads(stages, 8, 30, s) == "ok" for s in range(60)), stages
