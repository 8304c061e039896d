"""Memory-utilisation model of contiguous reservation vs paged allocation -- TEST
INFRASTRUCTURE ONLY (the tests import it; the product never does).

Plain Python restatement of the arithmetic the pages give:

* contiguous pre-allocation reserves the maximum length for every request for its whole
  life, so the unused remainder of the window is wasted and cannot serve other requests
  ("深度解构 LLM 推理优化…" section 1.2, Internal Fragmentation and Reservation Gap;
  intelliparadigm section 1: a 1024-token window with 500 generated tokens wastes 524);
* paged allocation takes a new fixed-size block only when the current one is full, so a
  sequence holds ceil(n / bs) blocks and wastes at most bs - 1 slots of its last block
  ("深度解构…" section 2.2, utilisation ~60 % -> above 96 %);
* KV capacity of a memory budget: budget // (2 x layers x H_kv x d_h x b)
  ("深度解构…" sections 1.1 and 3.2: ~72k tokens in ~9 GB for Llama-3-8B at FP16, doubled
  with an FP8 cache).

The serving trace (what requests exist, when they start and end) is the measurement's
setup, not the method: continuous batching over ``slots`` request slots, slots filled in index
order from the request queue at the start of a step; an admitted request first holds its
prompt, then every step (its first included) adds one generated token; measurements are taken
after the step's tokens are added; a request that has generated its output length is released
at the end of that step.
"""
from __future__ import annotations


def contiguous_reserved(active_requests: int, window: int) -> int:
    """Slots a contiguous scheme holds: the whole window for every active request."""
    return active_requests * window


def paged_reserved(lengths, bs: int) -> int:
    """Slots a paged scheme holds: ceil(n / bs) whole blocks per sequence."""
    return sum(-(-n // bs) * bs for n in lengths)


def paged_reserved_brute_force(lengths, bs: int) -> int:
    """The same count by simulating token by token: a sequence takes a block whenever a token
    lands on a block boundary (independent of the closed form above)."""
    slots = 0
    for n in lengths:
        for t in range(n):
            if t % bs == 0:
                slots += bs
    return slots


def capacity_tokens(budget_bytes: int, layers: int, h_kv: int, head_dim: int, elem_bytes: int) -> int:
    """Whole tokens whose KV fits in the budget."""
    return budget_bytes // (2 * layers * h_kv * head_dim * elem_bytes)


def simulate(prompts, outputs, slots: int, window: int, bs: int, max_steps: int | None = None) -> list:
    """Per-step records of the continuous-batching trace described in the module docstring:
    dicts with the step, the active requests, the live tokens, the contiguous and paged
    reserved slots and the paged waste.  Runs until every request is done (or max_steps)."""
    queue = list(range(len(prompts)))
    slot_req = [None] * slots            # request index in each slot
    generated = [0] * len(prompts)
    out = []
    step = 0
    while (queue or any(r is not None for r in slot_req)) and (max_steps is None or step < max_steps):
        for j in range(slots):
            if slot_req[j] is None and queue:
                slot_req[j] = queue.pop(0)
        active = [r for r in slot_req if r is not None]
        for r in active:
            generated[r] += 1
        lengths = [prompts[r] + generated[r] for r in active]
        paged = paged_reserved(lengths, bs)
        out.append(dict(step=step, active=len(active), live=sum(lengths),
                        contiguous=contiguous_reserved(len(active), window), paged=paged,
                        paged_waste=paged - sum(lengths)))
        for j in range(slots):
            r = slot_req[j]
            if r is not None and generated[r] >= outputs[r]:
                slot_req[j] = None
        step += 1
    return out


def summary(records) -> dict:
    """Time-averaged utilisation (live / reserved, summed over steps) of both schemes."""
    live = sum(r["live"] for r in records)
    cont = sum(r["contiguous"] for r in records)
    paged = sum(r["paged"] for r in records)
    return dict(steps=len(records), live_token_steps=live, contiguous_slot_steps=cont, paged_slot_steps=paged,
                contiguous_utilisation=live / cont if cont else 0.0,
                paged_utilisation=live / paged if paged else 0.0,
                waste_reduction=1.0 - (paged - live) / (cont - live) if cont > live else 0.0)
