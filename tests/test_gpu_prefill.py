"""Chunked-prefill attention through the C ABI against the fp64 oracle, on both schedules:
pa_prefill (one CTA per work item) and pa_prefill_ws (one CTA per SM claiming items from a
counter, sequences longest first, the next item prepared while the current one ends): every
template instance on ragged chunks, whole prompts, one-token chunks, the full-size workloads on
sampled rows, more sequences than the claim order keeps in shared memory, the workspace left
zero, and the guards."""
import numpy as np
import pytest
import torch

import workloads
import paged_kv_cache_428_b200 as pa
from paritylib import check_close, u16

pytestmark = pytest.mark.gpu
DEV = "cuda"


QUEUE = [pytest.param(False, id="grid"), pytest.param(True, id="queue")]


def _run(queue, out, case, kc, vc, tables=None, ctx=None, ws=None):
    args = (out, case.q.to(DEV), kc, vc, (case.block_tables if tables is None else tables).to(DEV),
            case.query_start.to(DEV), (case.context_lens if ctx is None else ctx).to(DEV), case.max_query_len)
    if queue:
        ws = pa.make_prefill_workspace(DEV) if ws is None else ws
        pa.pa_prefill_ws(*args, ws, case.scale)
        torch.cuda.synchronize()
        assert int(ws.count_nonzero()) == 0                       # left zero for the next call
    else:
        pa.pa_prefill(*args, case.scale)
        torch.cuda.synchronize()


def _gpu(case, queue):
    kc, vc = case.k_cache.to(DEV).clone(), case.v_cache.to(DEV).clone()
    if case.slot_mapping.numel():
        pa.pa_reshape_and_cache(case.key_new.to(DEV), case.value_new.to(DEV), kc, vc, case.slot_mapping.to(DEV))
    out = torch.empty_like(case.q, device=DEV)
    _run(queue, out, case, kc, vc)
    return out, kc, vc


def _oracle(case, orc, rows=None):
    kc, vc = u16(case.k_cache).copy(), u16(case.v_cache).copy()
    if case.slot_mapping.numel():
        orc.reshape_and_cache(u16(case.key_new), u16(case.value_new), kc, vc, case.slot_mapping.cpu().numpy(),
                              h_kv=case.h_kv, d=case.d, bs=case.bs, num_blocks=case.num_blocks)
    ref = orc.paged_prefill(u16(case.q), kc, vc, case.block_tables.cpu().numpy(), case.query_start.cpu().numpy(),
                            case.context_lens.cpu().numpy(), h_kv=case.h_kv, bs=case.bs, scale=case.scale, rows=rows)
    return ref, kc, vc


def _parity(orc, case, queue, rows=None):
    out, kc, vc = _gpu(case, queue)
    ref, okc, ovc = _oracle(case, orc, rows)
    assert np.array_equal(u16(kc), okc) and np.array_equal(u16(vc), ovc)   # the chunk's writes
    got = out if rows is None else torch.stack([out[r, h] for r, h in rows])
    assert pa.pa_device_errors() == 0
    return check_close(got, ref, False, case.name)


@pytest.mark.parametrize("queue", QUEUE)
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_every_prefill_variant(orc, d, bs, g, queue):
    """Ragged chunks (1..150 rows) after ragged cached prefixes (0..200 tokens)."""
    h_kv = 2
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", 5 * d + bs + g, B=4, h_q=h_kv * g,
                                       h_kv=h_kv, d=d, bs=bs, cached=(0, 200), chunk=(1, 150), pool_factor=1.3)
    _parity(orc, case, queue)


@pytest.mark.parametrize("queue", QUEUE)
@pytest.mark.parametrize("g", [1, 4, 8])
def test_whole_prompts_and_single_rows(orc, g, queue):
    h_kv = 2
    # whole prompts (nothing cached): plain causal attention
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_prompt", 3 + g, B=3, h_q=h_kv * g, h_kv=h_kv,
                                       chunk=(1, 200))
    _parity(orc, case, queue)
    # one-row chunks: a decode step through the prefill kernel
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", 4 + g, B=5, h_q=h_kv * g, h_kv=h_kv,
                                       cached=(0, 300), chunk=(1, 1))
    _parity(orc, case, queue)


@pytest.mark.parametrize("queue", QUEUE)
def test_chunk_lengths_on_tile_edges(orc, queue):
    """Chunks of exactly one, two and a fraction of a query tile (16 tokens at g = 4), and a
    context that ends exactly on a 64-token KV tile."""
    for chunk, cached in ((16, 48), (32, 0), (17, 47), (15, 113)):
        case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", chunk + cached, B=2, h_q=8, h_kv=2,
                                           cached=(cached, cached), chunk=(chunk, chunk))
        _parity(orc, case, queue)


@pytest.mark.parametrize("queue", QUEUE)
@pytest.mark.parametrize("name", ["prefill_llama3_8b_b8_chunk512", "prefill_llama3_8b_b8_prompt"])
def test_full_size_sampled(orc, name, queue):
    case = workloads.make_prefill_case(name, 0)
    g = torch.Generator().manual_seed(11)
    T = case.q.shape[0]
    qs = case.query_start.tolist()
    rows = [(int(r), int(h)) for r, h in zip(torch.randint(0, T, (40,), generator=g),
                                             torch.randint(0, case.h_q, (40,), generator=g))]
    rows += [(qs[s + 1] - 1, 5) for s in range(case.B)]          # the last row of every chunk
    _parity(orc, case, queue, rows=rows)


@pytest.mark.parametrize("queue", QUEUE)
def test_empty_chunks_between_sequences(orc, queue):
    """Sequences with no query rows (query_start repeats a value) among others: they have no work
    items and their neighbours' rows are unaffected; also sequences with no tokens at all."""
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", 45, B=9, h_q=8, h_kv=2, cached=(0, 100),
                                       chunk=(0, 5))
    assert case.meta["chunk"].count(0) >= 2
    _parity(orc, case, queue)
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", 59, B=7, h_q=8, h_kv=2, cached=(0, 0),
                                       chunk=(0, 40))
    assert 0 in case.meta["chunk"]
    _parity(orc, case, queue)


def test_queue_with_more_sequences_than_kept_in_shared_memory(orc):
    """1100 sequences (beyond the 1024 whose tables and claim order the kernel keeps in shared
    memory: it reads them from global memory and claims in sequence order), short chunks after
    short prefixes, two calls in a row on one workspace."""
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", 31, B=1100, h_q=8, h_kv=2,
                                       cached=(0, 40), chunk=(1, 6), pool_factor=1.2)
    ref, _, _ = _oracle(case, orc)
    kc, vc = case.k_cache.to(DEV).clone(), case.v_cache.to(DEV).clone()
    pa.pa_reshape_and_cache(case.key_new.to(DEV), case.value_new.to(DEV), kc, vc, case.slot_mapping.to(DEV))
    ws = pa.make_prefill_workspace(DEV)
    for _ in range(2):
        out = torch.full_like(case.q, float("nan"), device=DEV)
        _run(True, out, case, kc, vc, ws=ws)
        check_close(out, ref, False, "1100 sequences")
    assert pa.pa_device_errors() == 0


def test_queue_matches_grid_bit_for_bit():
    """Both schedules run the same per-item arithmetic: identical outputs (full-size chunk
    workload, seed 3)."""
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", 3)
    kc, vc = case.k_cache.to(DEV).clone(), case.v_cache.to(DEV).clone()
    pa.pa_reshape_and_cache(case.key_new.to(DEV), case.value_new.to(DEV), kc, vc, case.slot_mapping.to(DEV))
    a, b = torch.empty_like(case.q, device=DEV), torch.empty_like(case.q, device=DEV)
    _run(False, a, case, kc, vc)
    _run(True, b, case, kc, vc)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("queue", QUEUE)
def test_bad_block_and_bad_chunk_are_flagged(queue):
    """A block-table entry outside the pool stops the CTA that meets it; every row of the
    sequence that holds it comes out NaN.  A context shorter than its chunk leaves that
    sequence's rows unwritten.  Both set their error bit."""
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", 1, B=3, h_q=8, h_kv=2, cached=(40, 80),
                                       chunk=(10, 30))
    pa.pa_device_errors(clear=True)
    tab = case.block_tables.clone()
    tab[1, 0] = case.num_blocks + 5                              # outside the pool
    kc, vc = case.k_cache.to(DEV), case.v_cache.to(DEV)
    out = torch.zeros_like(case.q, device=DEV)
    _run(queue, out, case, kc, vc, tables=tab)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_BAD_BLOCK
    qs = case.query_start.tolist()
    assert torch.isnan(out[qs[1]:qs[2]].float()).all()
    ctx = case.context_lens.clone()
    ctx[2] = 1                                                   # shorter than its chunk
    out2 = torch.zeros_like(case.q, device=DEV)
    _run(queue, out2, case, kc, vc, ctx=ctx)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_BAD_CHUNK
    assert (out2[qs[2]:qs[3]].float() == 0).all()
