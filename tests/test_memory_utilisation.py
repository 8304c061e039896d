"""Memory utilisation of contiguous reservation vs paged allocation (host only): the oracle's
model pinned to the pages' numbers and to brute force, and the product's report (the C++
allocator driven through serving traces) equal to the model at every step."""
import json
from pathlib import Path

import pytest

import workloads
import paged_kv_cache_428_b200 as pa
from paged_kv_cache_428_b200 import memory_report
from oracle import memory_model as mm

GOLDEN = Path(__file__).resolve().parent / "golden"


# ------------------------------------------------------------------------------ oracle pins
def test_worked_fragmentation_example():
    """A 1024-token window holding 500 tokens: contiguous reservation wastes 524 slots; paged
    allocation wastes only the unfilled part of the last block."""
    g = json.loads((GOLDEN / "fragmentation_example.json").read_text())
    assert mm.contiguous_reserved(1, g["window"]) - g["generated"] == g["wasted"]
    for bs, waste in ((16, 12), (32, 12), (64, 12), (128, 12), (256, 12)):
        assert mm.paged_reserved([g["generated"]], bs) - g["generated"] == waste


@pytest.mark.parametrize("bs", [1, 16, 32, 64])
def test_paged_reserved_brute_force_and_bound(bs):
    for n in range(0, 300):
        r = mm.paged_reserved([n], bs)
        assert r == mm.paged_reserved_brute_force([n], bs)
        assert 0 <= r - n <= bs - 1
    lens = list(range(0, 200, 7))
    assert mm.paged_reserved(lens, bs) == mm.paged_reserved_brute_force(lens, bs)


def test_capacity_example():
    g = json.loads((GOLDEN / "capacity_example.json").read_text())
    args = (g["budget_bytes"], g["layers"], g["h_kv"], g["head_dim"])
    assert mm.capacity_tokens(*args, 2) == g["tokens_fp16"]
    assert mm.capacity_tokens(*args, 1) == g["tokens_fp8"]
    assert pa.pa_kv_capacity_tokens(*args, 2) == g["tokens_fp16"]
    assert pa.pa_kv_capacity_tokens(*args, 1) == g["tokens_fp8"]
    for b in (0, 1, 131071, 131072, 10 ** 12):
        for e in (1, 2):
            assert pa.pa_kv_capacity_tokens(b, 32, 8, 128, e) == mm.capacity_tokens(b, 32, 8, 128, e)
    assert pa.pa_kv_capacity_tokens(10 ** 9, 0, 8, 128, 2) == 0


def test_simulate_hand_computed():
    """Two requests, one slot, window 8, bs 4: request 0 (prompt 3, 2 outputs), then request 1
    (prompt 5, 1 output).  Step 0: lengths [4] -> 4 slots; step 1: [5] -> 8; step 2: request 1
    admitted, [6] -> 8; then done."""
    rec = mm.simulate([3, 5], [2, 1], 1, 8, 4)
    assert [(r["active"], r["live"], r["contiguous"], r["paged"], r["paged_waste"]) for r in rec] == \
        [(1, 4, 8, 4, 0), (1, 5, 8, 8, 3), (1, 6, 8, 8, 2)]
    s = mm.summary(rec)
    assert s["live_token_steps"] == 15 and s["contiguous_slot_steps"] == 24 and s["paged_slot_steps"] == 20


# ------------------------------------------------------------------------ product vs model
@pytest.mark.parametrize("name,max_steps", [("chat_w2048_b8", None), ("chat_w2048_b64", 400),
                                            ("long_w4096_b32", 300)])
def test_report_equals_model_every_step(name, max_steps):
    t = workloads.make_trace(name, 3)
    got = memory_report.run_trace(t.prompts, t.outputs, t.slots, t.window, t.bs, seed=5, max_steps=max_steps)
    want = mm.simulate(t.prompts, t.outputs, t.slots, t.window, t.bs, max_steps=max_steps)
    assert len(got) == len(want)
    for a, b in zip(got, want):
        for k in ("step", "active", "live", "contiguous", "paged", "paged_waste"):
            assert a[k] == b[k], (k, a, b)
        assert a["worst_seq_waste"] <= t.bs - 1


def test_paged_utilisation_shape():
    """Paging keeps utilisation above 96 % on every trace (the pages' '60 % -> above 96 %'),
    while whole-window reservation stays far below it."""
    for name in workloads.TRACES:
        t = workloads.make_trace(name, 0)
        s = mm.summary(mm.simulate(t.prompts, t.outputs, t.slots, t.window, t.bs))
        assert s["paged_utilisation"] > 0.96 and s["contiguous_utilisation"] < 0.6, (name, s)
        assert s["waste_reduction"] > 0.9


def test_report_cli_runs(capsys):
    assert memory_report.main(["--trace", "chat_w2048_b8"]) == 0
    out = json.loads(capsys.readouterr().out)
    assert out["paged_utilisation"] > 0.96 and out["max_seq_waste"] <= out["block_size"] - 1
    assert out["capacity_llama3_8b_9000MiB"]["tokens_bf16"] == 72000
