"""The C-ABI library loads, exports every symbol include/pa.h declares, and rejects bad
arguments on the host before any launch (CPU only: no call here reaches a kernel)."""
import ctypes
import json
import re
from pathlib import Path

import pytest

import paged_kv_cache_428_b200 as pa

ROOT = Path(__file__).resolve().parent.parent


def declared_functions():
    text = (ROOT / "include" / "pa.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("pa_reshape_and_cache", "pa_decode", "pa_copy_blocks", "pa_decode_workspace_size",
                 "pa_alloc_create", "pa_alloc_append_slot", "pa_alloc_fork", "pa_alloc_free_seq",
                 "pa_alloc_block_table", "pa_kv_bytes_per_token"):
        assert must in names


@pytest.mark.parametrize("name", declared_functions())
def test_symbol_exported(name):
    assert hasattr(pa.lib(), name), "libpa.so does not export %s" % name


def test_status_strings_and_version():
    assert pa.pa_status_str(0) == "ok"
    for code in (-1, -2, -3, -4, -5, -6):
        assert pa.pa_status_str(code) != "unknown status"
    assert pa.pa_version() >= 100


def test_kv_bytes_closed_forms():
    g = json.loads((ROOT / "tests" / "golden" / "kv_size_closed_forms.json").read_text())
    for e in g["per_token"]:
        assert pa.pa_kv_bytes_per_token(e["layers"], e["h_kv"], e["head_dim"], e["elem_bytes"]) == e["bytes"]
    for e in g["per_sequence"]:
        assert e["tokens"] * pa.pa_kv_bytes_per_token(e["layers"], e["h_kv"], e["head_dim"],
                                                      e["elem_bytes"]) == e["bytes"]


def test_workspace_size():
    assert pa.pa_decode_workspace_size(64, 32, 128, 4096, 0) == 0
    assert pa.pa_decode_workspace_size(64, 32, 128, 512, 512) == 0        # one partition: no partials
    n = pa.pa_decode_workspace_size(64, 32, 128, 4096, 512)
    counters = (64 * 32 * 4 + 255) // 256 * 256              # one int per (sequence, query head)
    ml = (64 * 32 * 8 * 2 * 4 + 255) // 256 * 256
    assert n == counters + ml + 64 * 32 * 8 * 128 * 4


L = pa.lib()
FAKE = 1 << 20            # an aligned non-null address; never dereferenced on these paths


def _decode(**kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, maxblk=8, ctx=FAKE, B=2, maxctx=100, hq=4, hkv=2, d=64,
             bs=16, nb=16, scale=0.125, dt=0, ks=1.0, vs=1.0, P=0, ws=0, wsb=0)
    a.update(kw)
    return L.pa_decode(a["out"], a["q"], a["k"], a["v"], a["bt"], a["maxblk"], a["ctx"], a["B"], a["maxctx"],
                       a["hq"], a["hkv"], a["d"], a["bs"], a["nb"], a["scale"], a["dt"], a["ks"], a["vs"], a["P"],
                       a["ws"], a["wsb"], None)


def test_decode_host_checks():
    assert _decode(hq=6, hkv=4) == -1                       # h_q % h_kv != 0
    assert _decode(d=96) == -2                              # unsupported head dim
    assert _decode(bs=8) == -2                              # unsupported block size
    assert _decode(hq=48, hkv=2) == -2                      # group 24 unsupported
    assert _decode(dt=7) == -1                              # bad cache dtype
    assert _decode(dt=1, ks=0.0) == -1                      # E4M3 needs positive scales
    assert _decode(dt=1, vs=float("nan")) == -1
    assert _decode(P=24) == -1                              # partition not a multiple of bs
    assert _decode(P=16, maxctx=1000) == -3                 # partials need a workspace
    assert _decode(P=16, maxctx=1000, ws=FAKE, wsb=64) == -3
    assert _decode(P=16, maxctx=1000, ws=FAKE + 4, wsb=1 << 30) == -3   # misaligned workspace
    assert _decode(q=0) == -1                               # null pointer
    assert _decode(out=FAKE + 2) == -1                      # misaligned output
    assert _decode(scale=float("inf")) == -1
    assert _decode(B=0) == 0                                # nothing to do, nothing launched


def test_cache_write_and_copy_host_checks():
    def rc(**kw):
        a = dict(key=FAKE, val=FAKE, ks_=0, vs_=0, kc=FAKE, vc=FAKE, slots=FAKE, T=4, hkv=2, d=64, bs=16, nb=8,
                 dt=0, ksc=1.0, vsc=1.0)
        a.update(kw)
        return L.pa_reshape_and_cache(a["key"], a["val"], a["ks_"], a["vs_"], a["kc"], a["vc"], a["slots"], a["T"],
                                      a["hkv"], a["d"], a["bs"], a["nb"], a["dt"], a["ksc"], a["vsc"], None)
    assert rc(T=0) == 0
    assert rc(d=80) == -2
    assert rc(ks_=100) == -1                                # stride shorter than a row
    assert rc(ks_=132) == -1                                # stride not a multiple of 8 elements
    assert rc(dt=1, ksc=-1.0) == -1
    assert rc(kc=0) == -1
    assert rc(key=FAKE + 8) == -1                           # misaligned rows
    ptrs = (ctypes.c_void_p * 1)(FAKE)
    assert L.pa_copy_blocks(ptrs, ptrs, 1, FAKE, 3, 24, 8, None) == -1      # block bytes not /16
    assert L.pa_copy_blocks(ptrs, ptrs, 1, FAKE, 0, 4096, 8, None) == 0     # no pairs
    nul = (ctypes.c_void_p * 1)(0)
    assert L.pa_copy_blocks(nul, ptrs, 1, FAKE, 3, 4096, 8, None) == -1


def test_host_validators():
    import torch
    bt = torch.tensor([[2, 5, 1, -1], [0, 3, -1, -1]], dtype=torch.int32)
    assert pa.pa_validate_block_tables(bt, torch.tensor([37, 20], dtype=torch.int32), 16, 6) == 0
    assert pa.pa_validate_block_tables(bt, torch.tensor([37, 40], dtype=torch.int32), 16, 6) == -1  # reads a -1
    assert pa.pa_validate_block_tables(bt, torch.tensor([37, 20], dtype=torch.int32), 16, 5) == -1  # id 5 >= 5
    assert pa.pa_validate_block_tables(bt, torch.tensor([65, 20], dtype=torch.int32), 16, 6) == -1  # row too short
    assert pa.pa_validate_slots(torch.tensor([0, -1, 95]), 16, 6) == 0
    assert pa.pa_validate_slots(torch.tensor([96]), 16, 6) == -1


def test_prefill_host_checks():
    def rc(**kw):
        a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, maxblk=8, qs=FAKE, ctx=FAKE, B=2, mql=64, hq=8, hkv=2,
                 d=128, bs=16, nb=16, scale=0.088, dt=0)
        a.update(kw)
        return L.pa_prefill(a["out"], a["q"], a["k"], a["v"], a["bt"], a["maxblk"], a["qs"], a["ctx"], a["B"],
                            a["mql"], a["hq"], a["hkv"], a["d"], a["bs"], a["nb"], a["scale"], a["dt"], None)
    assert rc(hq=6, hkv=4) == -1                            # h_q % h_kv != 0
    assert rc(d=96) == -2                                   # unsupported head dim
    assert rc(bs=8) == -2                                   # unsupported block size
    assert rc(hq=32, hkv=2) == -2                           # group 16 unsupported
    assert rc(dt=1) == -2                                   # quantised caches: bf16 only
    assert rc(dt=9) == -1                                   # not a cache type
    assert rc(scale=float("nan")) == -1
    assert rc(scale=-0.1) == -1                             # the kernel needs scale >= 0
    assert rc(B=-1) == -1 and rc(mql=-1) == -1 and rc(nb=0) == -1
    assert rc(qs=0) == -1 and rc(out=0) == -1               # null pointers
    assert rc(q=FAKE + 4) == -1                             # misaligned rows
    assert rc(B=0) == 0 and rc(mql=0) == 0                  # nothing to do, nothing launched


def test_prefill_ws_host_checks():
    def rc(ws=FAKE, wsb=256, **kw):
        a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, maxblk=8, qs=FAKE, ctx=FAKE, B=2, mql=64, hq=8, hkv=2,
                 d=128, bs=16, nb=16, scale=0.088, dt=0)
        a.update(kw)
        return L.pa_prefill_ws(a["out"], a["q"], a["k"], a["v"], a["bt"], a["maxblk"], a["qs"], a["ctx"], a["B"],
                               a["mql"], a["hq"], a["hkv"], a["d"], a["bs"], a["nb"], a["scale"], a["dt"], ws, wsb,
                               None)
    need = L.pa_prefill_workspace_size()
    assert 8 <= need <= 4096
    assert rc(ws=0) == -3                                   # no workspace
    assert rc(wsb=need - 1) == -3                           # too small
    assert rc(ws=FAKE + 8) == -3                            # misaligned
    assert rc(ws=0, B=0) == -3                              # the workspace is checked first
    assert rc(wsb=need, d=96) == -2                         # then pa_prefill's own checks
    assert rc(wsb=need, hq=6, hkv=4) == -1
    assert rc(wsb=need, B=0) == 0                           # nothing to do, nothing launched


def test_decode_step_host_checks():
    def rc(**kw):
        a = dict(key=FAKE, val=FAKE, kst=0, vst=0, slots=FAKE, out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, maxblk=8,
                 ctx=FAKE, B=2, maxctx=100, hq=4, hkv=2, d=64, bs=16, nb=16, scale=0.125, dt=0, ks=1.0, vs=1.0, P=0,
                 ws=0, wsb=0)
        a.update(kw)
        return L.pa_decode_step(a["key"], a["val"], a["kst"], a["vst"], a["slots"], a["out"], a["q"], a["kc"], a["vc"],
                                a["bt"], a["maxblk"], a["ctx"], a["B"], a["maxctx"], a["hq"], a["hkv"], a["d"],
                                a["bs"], a["nb"], a["scale"], a["dt"], a["ks"], a["vs"], a["P"], a["ws"], a["wsb"],
                                None)
    # every rejection happens before the cache write is launched
    assert rc(B=-1) == -1
    assert rc(B=0) == 0
    assert rc(hq=6, hkv=4) == -1
    assert rc(d=96) == -2
    assert rc(dt=1, ks=0.0) == -1                           # quantised caches need positive scales
    assert rc(P=16, maxctx=1000) == -3                      # partials need a workspace
    assert rc(q=0) == -1
    assert rc(kst=100) == -1                                # key rows shorter than h_kv * d
    assert rc(slots=0) == -1
