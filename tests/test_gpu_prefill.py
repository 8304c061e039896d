"""Chunked-prefill attention (pa_prefill, through the C ABI) against the fp64 oracle: every
template instance on ragged chunks, whole prompts, one-token chunks, the full-size workloads on
sampled rows, and the guards."""
import numpy as np
import pytest
import torch

import workloads
import paged_kv_cache_428_b200 as pa
from paritylib import check_close, u16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gpu(case):
    kc, vc = case.k_cache.to(DEV).clone(), case.v_cache.to(DEV).clone()
    if case.slot_mapping.numel():
        pa.pa_reshape_and_cache(case.key_new.to(DEV), case.value_new.to(DEV), kc, vc, case.slot_mapping.to(DEV))
    out = torch.empty_like(case.q, device=DEV)
    pa.pa_prefill(out, case.q.to(DEV), kc, vc, case.block_tables.to(DEV), case.query_start.to(DEV),
                  case.context_lens.to(DEV), case.max_query_len, case.scale)
    torch.cuda.synchronize()
    return out, kc, vc


def _oracle(case, orc, rows=None):
    kc, vc = u16(case.k_cache).copy(), u16(case.v_cache).copy()
    if case.slot_mapping.numel():
        orc.reshape_and_cache(u16(case.key_new), u16(case.value_new), kc, vc, case.slot_mapping.cpu().numpy(),
                              h_kv=case.h_kv, d=case.d, bs=case.bs, num_blocks=case.num_blocks)
    ref = orc.paged_prefill(u16(case.q), kc, vc, case.block_tables.cpu().numpy(), case.query_start.cpu().numpy(),
                            case.context_lens.cpu().numpy(), h_kv=case.h_kv, bs=case.bs, scale=case.scale, rows=rows)
    return ref, kc, vc


def _parity(orc, case, rows=None):
    out, kc, vc = _gpu(case)
    ref, okc, ovc = _oracle(case, orc, rows)
    assert np.array_equal(u16(kc), okc) and np.array_equal(u16(vc), ovc)   # the chunk's writes
    got = out if rows is None else torch.stack([out[r, h] for r, h in rows])
    assert pa.pa_device_errors() == 0
    return check_close(got, ref, False, case.name)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_every_prefill_variant(orc, d, bs, g):
    """Ragged chunks (1..150 rows) after ragged cached prefixes (0..200 tokens)."""
    h_kv = 2
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", 5 * d + bs + g, B=4, h_q=h_kv * g,
                                       h_kv=h_kv, d=d, bs=bs, cached=(0, 200), chunk=(1, 150), pool_factor=1.3)
    _parity(orc, case)


@pytest.mark.parametrize("g", [1, 4, 8])
def test_whole_prompts_and_single_rows(orc, g):
    h_kv = 2
    # whole prompts (nothing cached): plain causal attention
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_prompt", 3 + g, B=3, h_q=h_kv * g, h_kv=h_kv,
                                       chunk=(1, 200))
    _parity(orc, case)
    # one-row chunks: a decode step through the prefill kernel
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", 4 + g, B=5, h_q=h_kv * g, h_kv=h_kv,
                                       cached=(0, 300), chunk=(1, 1))
    _parity(orc, case)


def test_chunk_lengths_on_tile_edges(orc):
    """Chunks of exactly one, two and a fraction of a query tile (16 tokens at g = 4), and a
    context that ends exactly on a 64-token KV tile."""
    for chunk, cached in ((16, 48), (32, 0), (17, 47), (15, 113)):
        case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", chunk + cached, B=2, h_q=8, h_kv=2,
                                           cached=(cached, cached), chunk=(chunk, chunk))
        _parity(orc, case)


@pytest.mark.parametrize("name", ["prefill_llama3_8b_b8_chunk512", "prefill_llama3_8b_b8_prompt"])
def test_full_size_sampled(orc, name):
    case = workloads.make_prefill_case(name, 0)
    g = torch.Generator().manual_seed(11)
    T = case.q.shape[0]
    qs = case.query_start.tolist()
    rows = [(int(r), int(h)) for r, h in zip(torch.randint(0, T, (40,), generator=g),
                                             torch.randint(0, case.h_q, (40,), generator=g))]
    rows += [(qs[s + 1] - 1, 5) for s in range(case.B)]          # the last row of every chunk
    _parity(orc, case, rows=rows)


def test_bad_block_and_bad_chunk_are_flagged():
    case = workloads.make_prefill_case("prefill_llama3_8b_b8_chunk512", 1, B=3, h_q=8, h_kv=2, cached=(40, 80),
                                       chunk=(10, 30))
    pa.pa_device_errors()
    tab = case.block_tables.clone()
    tab[1, 0] = case.num_blocks + 5                              # outside the pool
    kc, vc = case.k_cache.to(DEV), case.v_cache.to(DEV)
    out = torch.zeros_like(case.q, device=DEV)
    pa.pa_prefill(out, case.q.to(DEV), kc, vc, tab.to(DEV), case.query_start.to(DEV), case.context_lens.to(DEV),
                  case.max_query_len, case.scale)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() & pa.PA_DEVERR_BAD_BLOCK
    qs = case.query_start.tolist()
    assert torch.isnan(out[qs[1]:qs[2]].float()).all()
    ctx = case.context_lens.clone()
    ctx[2] = 1                                                   # shorter than its chunk
    out2 = torch.zeros_like(case.q, device=DEV)
    pa.pa_prefill(out2, case.q.to(DEV), kc, vc, case.block_tables.to(DEV), case.query_start.to(DEV), ctx.to(DEV),
                  case.max_query_len, case.scale)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() & pa.PA_DEVERR_BAD_CHUNK
    assert (out2[qs[2]:qs[3]].float() == 0).all()
