"""The whole-block decode kernel's schedule (CPU only).

The kernel cuts the step's T units (one block of one sequence, every KV head) into per-CTA
ranges, each into a static segment and tail chunks that any CTA may claim; a piece (the part of
one sequence inside one segment) that is not its whole sequence writes a partial into slot
2 g + (0 if the piece starts the segment else 1), and the merge kernel reads, for each split
sequence, the slots of the non-empty segments it overlaps.  This test compiles the library's
own segment arithmetic (AllHeadsSegs, decode_allheads.cuh) into a host program and checks, for
many sizes: the segments partition [0, T) in id order, seg_of agrees with the bounds, chunks
hold at most U units and the tail about 15 % of a range; and for random sequence layouts:
partial pieces never share a slot, and the pieces the merge reads are exactly the pieces the
decode writes (whatever CTA claims which chunk)."""
import os
import random
import subprocess
import tempfile
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent

PROBE = r'''
#include <cstdio>
#include "decode_allheads.cuh"
using namespace pa;
int main(int argc, char **argv) {
  int T, C;
  while (scanf("%d %d", &T, &C) == 2) {
    const AllHeadsSegs sg = AllHeadsSegs::make(T, C);
    printf("case %d %d %d %d %d\n", T, C, sg.Ce, sg.U, kTailChunks);
    for (int g = 0; g < sg.Ce * (1 + kTailChunks); ++g) {
      int lo, hi; sg.bounds(g, lo, hi);
      printf("seg %d %d %d\n", g, lo, hi);
    }
    printf("segof");
    for (int x = 0; x < T; ++x) printf(" %d", sg.seg_of(x));
    printf("\n");
  }
  return 0;
}
'''

CASES = [(1, 148), (5, 148), (147, 148), (148, 148), (149, 148), (300, 148), (592, 148), (1000, 148),
         (9216, 148), (9300, 148), (45000, 148), (12, 3), (100, 7), (64, 160), (2000, 160)]


@pytest.fixture(scope="module")
def segs():
    with tempfile.TemporaryDirectory() as tmp:
        src = Path(tmp) / "probe.cu"
        src.write_text(PROBE)
        exe = Path(tmp) / "probe"
        nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
        subprocess.run([nvcc, "-std=c++17", "--expt-relaxed-constexpr", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-I", str(ROOT / "include"), "-I", str(ROOT / "paged_kv_cache_428_b200" / "csrc"), str(src),
                        "-o", str(exe)], check=True, capture_output=True)
        inp = "".join("%d %d\n" % c for c in CASES)
        out = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, check=True).stdout
    cases, cur = [], None
    for line in out.splitlines():
        f = line.split()
        if f[0] == "case":
            cur = dict(T=int(f[1]), C=int(f[2]), Ce=int(f[3]), U=int(f[4]), NCH=int(f[5]), segs=[])
            cases.append(cur)
        elif f[0] == "seg":
            cur["segs"].append((int(f[2]), int(f[3])))
        else:
            cur["segof"] = [int(v) for v in f[1:]]
    assert len(cases) == len(CASES)
    return cases


def test_segments_partition_the_units(segs):
    for c in segs:
        T, Ce, U, NCH = c["T"], c["Ce"], c["U"], c["NCH"]
        assert Ce == min(T, c["C"])
        pos = 0
        for g, (lo, hi) in enumerate(c["segs"]):
            assert lo <= hi
            if lo < hi:
                assert lo == pos, (T, g)                     # contiguous, in id order
                pos = hi
            if g % (1 + NCH):
                assert hi - lo <= U                          # chunks hold at most U units
        assert pos == T
        for x, g in enumerate(c["segof"]):
            lo, hi = c["segs"][g]
            assert lo <= x < hi, (T, x, g)
        per = T // Ce
        if per >= 40:                                        # tails of about 15 % of a range
            for r in range(Ce):
                tail = sum(hi - lo for lo, hi in c["segs"][r * (1 + NCH) + 1:(r + 1) * (1 + NCH)])
                assert 0.12 * per <= tail <= 0.15 * per + NCH, (T, r, tail, per)


def _layout(T, rnd):
    """Random sequence sizes (in units) summing to T, with some one-unit sequences."""
    sizes = []
    while sum(sizes) < T:
        sizes.append(rnd.choice([1, 1, 2, 3, rnd.randint(1, 40), rnd.randint(1, max(1, T // 3))]))
    sizes[-1] -= sum(sizes) - T
    if sizes[-1] <= 0:
        sizes.pop()
    prefix = [0]
    for n in sizes:
        prefix.append(prefix[-1] + n)
    assert prefix[-1] == T
    return prefix


def test_partial_slots_unique_and_counts_match(segs):
    rnd = random.Random(7)
    for c in segs:
        T, S = c["T"], c["segs"]
        seg_of = c["segof"]
        for _ in range(20):
            prefix = _layout(T, rnd)
            used = {}
            for s in range(len(prefix) - 1):
                gs, ge = prefix[s], prefix[s + 1]
                g0, g1 = seg_of[gs], seg_of[ge - 1]
                target = sum(1 for g in range(g0, g1 + 1) if S[g][0] < S[g][1])
                pieces = 0
                for g in range(g0, g1 + 1):
                    lo, hi = S[g]
                    if lo >= hi:
                        continue
                    a, b = max(gs, lo), min(ge, hi)
                    assert a < b                             # every non-empty segment in between overlaps
                    pieces += 1
                    if g0 == g1:
                        continue                             # the whole sequence: no partial
                    slot = 2 * g + (0 if gs <= lo else 1)
                    assert slot not in used, (T, s, g, used.get(slot))
                    used[slot] = (s, g)
                assert pieces == target
                assert (g0 == g1) == (pieces == 1)
            assert all(slot < 2 * c["Ce"] * (1 + c["NCH"]) for slot in used)
