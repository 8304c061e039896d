"""KV memory utilisation of a serving trace under the library's block allocator, next to a
contiguous scheme that reserves the whole context window per request.

    python -m paged_kv_cache_428_b200.memory_report --trace chat_w2048_b64 [--seed 0] [--per-step]
    python -m paged_kv_cache_428_b200.memory_report --prefix sys256_doc1536x4_q64_n64

Contiguous pre-allocation keeps the window reserved for every request for its whole life
("深度解构 LLM 推理优化…" section 1.2, Internal Fragmentation / Reservation Gap; intelliparadigm
section 1: a 1024-token window with 500 generated tokens leaves 524 slots unused).  The paged
figures come from the C++ allocator itself (pa_alloc_* through the binding): blocks are taken
only when a sequence's last block is full and returned when it finishes ("深度解构…" section
2.2), so each sequence wastes at most block_size - 1 slots.

The trace runs continuous batching over `slots` request slots: at the start of a step, empty
slots take the next requests in order; an admitted request's prompt is appended at once
(pa_alloc_append_n), then every step appends one generated token per active request
(pa_alloc_append_batch); the allocator's state is read after the step's appends
(pa_alloc_stats: blocks in use, slots allocated but not filled); a request that has produced
its output length is released at the end of the step (pa_alloc_free_seq).
"""
from __future__ import annotations

import argparse
import json
import sys

from . import BlockAllocator, pa_kv_capacity_tokens


def run_trace(prompts, outputs, slots: int, window: int, bs: int, seed: int = 0, max_steps=None):
    """Per-step records: step, active requests, live tokens, contiguous reserved slots
    (active x window), paged reserved slots (blocks in use x bs), paged waste (allocator's
    unfilled slots), largest per-sequence waste."""
    pool = slots * (-(-window // bs))                # enough blocks for every slot at full window
    alloc = BlockAllocator(pool, bs, seed)
    queue = list(range(len(prompts)))
    seq_of = [None] * slots                          # allocator sequence id per slot
    req_of = [None] * slots                          # request index per slot
    done = [0] * len(prompts)                        # tokens generated per request
    records = []
    step = 0
    try:
        while (queue or any(r is not None for r in req_of)) and (max_steps is None or step < max_steps):
            for j in range(slots):
                if req_of[j] is None and queue:
                    r = queue.pop(0)
                    req_of[j], seq_of[j] = r, alloc.new_seq()
                    alloc.append_n(seq_of[j], prompts[r])
            active = [j for j in range(slots) if req_of[j] is not None]
            alloc.append_batch([seq_of[j] for j in active])
            for j in active:
                done[req_of[j]] += 1
            st = alloc.stats()
            lens = [alloc.seq_len(seq_of[j]) for j in active]
            worst = max((-(-n // bs) * bs - n for n in lens), default=0)
            records.append(dict(step=step, active=len(active), live=sum(lens), contiguous=len(active) * window,
                                paged=st["used"] * bs, paged_waste=st["frag_tokens"], worst_seq_waste=worst))
            for j in active:
                if done[req_of[j]] >= outputs[req_of[j]]:
                    alloc.free_seq(seq_of[j])
                    req_of[j] = seq_of[j] = None
            step += 1
        assert alloc.stats()["used"] == 0 or max_steps is not None
    finally:
        alloc.close()
    return records


def summarise(records) -> dict:
    live = sum(r["live"] for r in records)
    cont = sum(r["contiguous"] for r in records)
    paged = sum(r["paged"] for r in records)
    return {"steps": len(records), "live_token_steps": live, "contiguous_slot_steps": cont,
            "paged_slot_steps": paged,
            "contiguous_utilisation": round(live / cont, 6) if cont else 0.0,
            "paged_utilisation": round(live / paged, 6) if paged else 0.0,
            "waste_reduction": round(1.0 - (paged - live) / (cont - live), 6) if cont > live else 0.0,
            "concurrency_gain": round(cont / paged, 3) if paged else 0.0,
            "max_seq_waste": max((r["worst_seq_waste"] for r in records), default=0)}


def run_prefix_prompts(prompts, bs: int, seed: int = 0) -> dict:
    """Insert every prompt with prefix caching (all requests alive together) and report the
    prompt tokens found cached (prefill skipped), and the blocks held against the blocks the
    same requests would hold without sharing (sum of ceil(len / bs))."""
    pool = sum(-(-len(p) // bs) for p in prompts)
    alloc = BlockAllocator(pool, bs, seed)
    try:
        cached = [alloc.new_seq_prefix(p)[2] for p in prompts]
        used, ps = alloc.stats()["used"], alloc.prefix_stats()
    finally:
        alloc.close()
    total = sum(len(p) for p in prompts)
    return {"requests": len(prompts), "prompt_tokens": total, "cached_tokens": sum(cached),
            "prefill_skipped": round(sum(cached) / total, 6), "blocks_shared": used, "blocks_private": pool,
            "memory_saving": round(1.0 - used / pool, 6), "hit_tokens": ps["hit_tokens"],
            "miss_tokens": ps["miss_tokens"]}


def capacity_report(budget_bytes: int, layers: int, h_kv: int, head_dim: int) -> dict:
    return {"budget_bytes": budget_bytes,
            "tokens_bf16": pa_kv_capacity_tokens(budget_bytes, layers, h_kv, head_dim, 2),
            "tokens_one_byte_codes": pa_kv_capacity_tokens(budget_bytes, layers, h_kv, head_dim, 1)}


def main(argv=None) -> int:
    import workloads
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--trace", default="chat_w2048_b64", choices=sorted(workloads.TRACES))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--per-step", action="store_true")
    ap.add_argument("--prefix", default=None, choices=sorted(workloads.PREFIX_TRACES),
                    help="report prefix caching on prompts sharing a system prompt and documents")
    a = ap.parse_args(argv)
    if a.prefix:
        bs = workloads.PREFIX_TRACES[a.prefix]["bs"]
        out = {"prefix_trace": a.prefix, "seed": a.seed, "block_size": bs,
               "same_document_front": run_prefix_prompts(workloads.make_prefix_prompts(a.prefix, a.seed), bs, a.seed),
               "document_front_changed": run_prefix_prompts(
                   workloads.make_prefix_prompts(a.prefix, a.seed, front_changed=True), bs, a.seed)}
        print(json.dumps(out))
        return 0
    t = workloads.make_trace(a.trace, a.seed)
    rec = run_trace(t.prompts, t.outputs, t.slots, t.window, t.bs, a.seed)
    out = {"trace": a.trace, "seed": a.seed, "requests": len(t.prompts), "slots": t.slots, "window": t.window,
           "block_size": t.bs, **summarise(rec),
           "capacity_llama3_8b_9000MiB": capacity_report(9000 * 2 ** 20, 32, 8, 128)}
    if a.per_step:
        out["per_step"] = rec
    print(json.dumps(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
