"""Decode over sequences built with the allocator's prefix cache (through the C ABI): each
request writes K/V only for the tokens the cache did not hold, and every output row still
equals the fp64 oracle on that request's own logical rows."""
import math
import zlib

import numpy as np
import pytest
import torch

import paged_kv_cache_428_b200 as pa
from paritylib import check_close, u16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _rows(tokens, h_kv, d):
    """K and V rows of every position: a function of the whole prefix up to that position (as a
    model's would be), drawn from a generator seeded by the prefix's CRC."""
    ks, vs = [], []
    for t in range(len(tokens)):
        g = torch.Generator().manual_seed(zlib.crc32(np.asarray(tokens[:t + 1], np.int32).tobytes()))
        ks.append(torch.randn(h_kv, d, generator=g).to(torch.bfloat16))
        vs.append(torch.randn(h_kv, d, generator=g).to(torch.bfloat16))
    return torch.stack(ks), torch.stack(vs)


def _oracle_row(orc, q, krows, vrows, bs, scale):
    """fp64 attention of one sequence over its contiguous rows (identity block table)."""
    n, h_kv, d = krows.shape
    nb = max(1, -(-n // bs))
    kp = torch.zeros(nb * bs, h_kv, d, dtype=torch.bfloat16)
    vp = torch.zeros_like(kp)
    kp[:n], vp[:n] = krows, vrows
    kp = kp.reshape(nb, bs, h_kv, d).transpose(1, 2).contiguous()
    vp = vp.reshape(nb, bs, h_kv, d).transpose(1, 2).contiguous()
    tab = np.arange(nb, dtype=np.int32)[None]
    return orc.paged_decode(u16(q[None]), u16(kp), u16(vp), tab, np.array([n], np.int32), h_kv=h_kv, bs=bs,
                            scale=scale)[0]


@pytest.mark.parametrize("d,bs", [(128, 16), (64, 32)])
def test_prefix_cached_decode_matches_oracle(orc, d, bs):
    h_q, h_kv, nb = 8, 2, 256
    g = torch.Generator().manual_seed(d + bs)
    systems = [torch.randint(0, 500, (n,), generator=g).tolist() for n in (3 * bs + 5, 2 * bs)]
    prompts = []
    for i in range(8):
        q = torch.randint(0, 500, (int(torch.randint(1, 40, (1,), generator=g)),), generator=g).tolist()
        prompts.append(systems[i % 2] + q)
    prompts.append(list(prompts[2]))                      # an identical prompt: fully cached blocks
    a = pa.BlockAllocator(nb, bs, 9)
    kc = torch.full((nb, h_kv, bs, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    vc = torch.full_like(kc, float("nan"))
    sids, toks, cached_all = [], [], []
    for p in prompts:
        sid, slots, cached = a.new_seq_prefix(p)
        k, v = _rows(p, h_kv, d)
        if cached < len(p):                               # write only what the cache lacks
            pa.pa_reshape_and_cache(k[cached:].to(DEV), v[cached:].to(DEV), kc, vc,
                                    torch.tensor(slots[cached:], dtype=torch.int64, device=DEV))
        sids.append(sid)
        toks.append(list(p))
        cached_all.append(cached)
    assert cached_all[0] == 0 and min(cached_all[2:]) >= 2 * bs and cached_all[-1] == len(prompts[2]) // bs * bs
    # one decode step: append a token to every sequence, write its K/V, attend
    new_tok = torch.randint(0, 500, (len(sids),), generator=g).tolist()
    slots, pairs = a.append_batch(sids)
    assert pairs == []                                    # cached blocks are full: no copy-on-write
    kn, vn = [], []
    for i, t in enumerate(new_tok):
        toks[i].append(t)
        k, v = _rows(toks[i], h_kv, d)
        kn.append(k[-1])
        vn.append(v[-1])
    pa.pa_reshape_and_cache(torch.stack(kn).to(DEV), torch.stack(vn).to(DEV), kc, vc,
                            torch.tensor(slots, dtype=torch.int64, device=DEV))
    maxb = max(-(-len(t) // bs) for t in toks)
    tab, lens = a.block_table(sids, maxb)
    q = torch.randn(len(sids), h_q, d, generator=g).to(torch.bfloat16)
    out = torch.empty((len(sids), h_q, d), dtype=torch.bfloat16, device=DEV)
    scale = 1.0 / math.sqrt(d)
    pa.pa_decode(out, q.to(DEV), kc, vc, tab.to(DEV), lens.to(DEV), int(lens.max()), scale, 2 * bs)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    ref = np.stack([_oracle_row(orc, q[i], *_rows(toks[i], h_kv, d), bs, scale) for i in range(len(sids))])
    check_close(out, ref, False, "prefix-cached decode")
