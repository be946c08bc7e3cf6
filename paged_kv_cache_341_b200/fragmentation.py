"""KV-memory fragmentation simulator: contiguous reservation against paged blocks.

The pages contrast two ways of holding a batch's KV cache in a fixed budget
of token slots:

* contiguous: each request gets one contiguous buffer.  Sized to the maximum
  context, most of it is never written ("internal fragmentation": a buffer for
  2,048 tokens holding 200 wastes the rest); and buffers of different sizes
  coming and going leave holes too small for the next request although the
  free total would fit it ("external fragmentation") -- "PagedAttention
  Explained: Managing KV Cache Efficiently" (agentechip.com), section "The
  Memory Fragmentation Problem", and the 60-80 % waste figure there and in
  the "Paged Attention" glossary entry (aidolsgroup.com), "Full definition".
* paged: fixed-size blocks from one pool, taken one at a time as a sequence
  grows, so the only slack is the unfilled tail of each sequence's last block
  ("PagedAttention Explained: Managing KV Cache Efficiently", section
  "Implementing a Simplified Paged KV Cache").

``simulate`` replays one synthetic serving trace (arrivals, prompt and output
lengths) step by step under one allocator and reports how much of the held
memory holds no KV, how many requests ran at once, and how long the trace
took.  The paged allocator is the library's block pool (``pa.Pool``, C++);
the contiguous ones are a first-fit arena written here.  Everything runs on
the host.

Model of a step: first admit waiting requests in arrival order (first come,
first served; the queue head blocks the rest), allocating the prompt; then
every running request writes one token; requests that reach their final
length release their memory.  Paged: a token at offset 0 of a block takes a
fresh block; if the pool is empty the youngest running request is preempted
(its blocks released, it rejoins the front of the queue and starts over).
"""

import dataclasses

import numpy as np


@dataclasses.dataclass
class Request:
    arrival: int        # step at which it may be admitted
    prompt: int         # tokens present at admission
    output: int         # tokens generated afterwards (one per step)

    @property
    def final(self):
        return self.prompt + self.output


def synthetic_trace(n, max_context, seed, rate=4.0, prompt=(32, 512), output_median=192, output_sigma=1.0):
    """Seeded trace: Poisson arrivals (``rate`` per step), uniform prompt
    lengths, log-normal output lengths, every request within ``max_context``."""
    rng = np.random.default_rng(seed)
    gaps = rng.exponential(1.0 / rate, size=n)
    arrivals = np.floor(np.cumsum(gaps)).astype(np.int64)
    prompts = rng.integers(prompt[0], prompt[1] + 1, size=n)
    outs = np.exp(rng.normal(np.log(output_median), output_sigma, size=n))
    outs = np.clip(np.floor(outs), 1, max_context - prompts).astype(np.int64)
    return [Request(int(a), int(p), int(o)) for a, p, o in zip(arrivals, prompts, outs)]


class ContiguousArena:
    """First-fit allocator of contiguous slot ranges in [0, capacity)."""

    def __init__(self, capacity):
        self.capacity = int(capacity)
        self.holes = [(0, self.capacity)]      # sorted, disjoint, non-adjacent (start, size)

    def free_total(self):
        return sum(size for _, size in self.holes)

    def largest_hole(self):
        return max((size for _, size in self.holes), default=0)

    def alloc(self, n):
        for i, (start, size) in enumerate(self.holes):
            if size >= n:
                if size == n:
                    del self.holes[i]
                else:
                    self.holes[i] = (start + n, size - n)
                return start
        return None

    def free(self, start, n):
        self.holes.append((start, n))
        self.holes.sort()
        merged = []
        for s, z in self.holes:
            if merged and merged[-1][0] + merged[-1][1] == s:
                merged[-1] = (merged[-1][0], merged[-1][1] + z)
            else:
                merged.append((s, z))
        self.holes = merged


@dataclasses.dataclass
class Result:
    allocator: str
    steps: int = 0                   # steps until the last request finished
    finished: int = 0
    preemptions: int = 0             # paged: requests restarted for lack of blocks
    external_failures: int = 0       # contiguous: admissions refused although the free total would fit
    held_slot_steps: int = 0         # sum over steps of slots held by running requests
    used_slot_steps: int = 0         # sum over steps of slots holding KV
    running_steps: int = 0           # sum over steps of running requests

    @property
    def waste(self):
        """Fraction of held memory that holds no KV, averaged over the trace."""
        return 1.0 - self.used_slot_steps / self.held_slot_steps if self.held_slot_steps else 0.0

    @property
    def mean_batch(self):
        return self.running_steps / self.steps if self.steps else 0.0


def simulate(trace, capacity_tokens, allocator, block_size=16, max_context=2048, pool_factory=None,
             max_steps=1_000_000):
    """Replay ``trace`` in a budget of ``capacity_tokens`` slots.

    allocator: "paged" (blocks of ``block_size`` from ``pool_factory(num_blocks,
    block_size)``, default the library pool), "contiguous-max" (one buffer of
    ``max_context`` slots per request) or "contiguous-exact" (one buffer of
    exactly the final length, the best a contiguous scheme can do).
    """
    res = Result(allocator)
    queue = []                      # waiting requests (index into trace), front first
    nxt = 0                         # next trace entry not yet arrived
    running = []                    # [index, length, state]; state: list of block ids or (start, size)
    if allocator == "paged":
        if pool_factory is None:
            from . import pa
            pool_factory = pa.Pool
        nb = capacity_tokens // block_size
        pool = pool_factory(nb, block_size)
        alloc = pool.alloc if hasattr(pool, "alloc") else pool.pa_pool_alloc
        free = pool.free if hasattr(pool, "free") else pool.pa_pool_free
        nfree = pool.num_free if hasattr(pool, "num_free") else pool.pa_pool_num_free
    elif allocator in ("contiguous-max", "contiguous-exact"):
        arena = ContiguousArena(capacity_tokens)
    else:
        raise ValueError("unknown allocator %r" % allocator)

    def release(entry):
        if allocator == "paged":
            free(list(entry[2]))
        else:
            arena.free(*entry[2])

    step = 0
    while (nxt < len(trace) or queue or running) and step < max_steps:
        while nxt < len(trace) and trace[nxt].arrival <= step:
            queue.append(nxt)
            nxt += 1
        # admission, first come first served
        while queue:
            r = trace[queue[0]]
            if allocator == "paged":
                need = -(-r.prompt // block_size)
                if need > nfree():
                    break
                state = [int(b) for b in alloc(need)]
            else:
                size = max_context if allocator == "contiguous-max" else r.final
                if size > capacity_tokens:
                    raise ValueError("request larger than the whole budget")
                start = arena.alloc(size)
                if start is None:
                    if arena.free_total() >= size:
                        res.external_failures += 1
                    break
                state = (start, size)
            running.append([queue.pop(0), r.prompt, state])
        # one token per running request, oldest first
        i = 0
        while i < len(running):
            entry = running[i]
            if allocator == "paged" and entry[1] % block_size == 0:
                # a fresh block is needed: preempt the youngest running
                # requests until one is free; they restart later
                preempted_self = False
                while nfree() == 0:
                    victim = running.pop()
                    release(victim)
                    queue.insert(0, victim[0])
                    res.preemptions += 1
                    if victim is entry:
                        preempted_self = True
                        break
                if preempted_self:
                    break                       # entry was the youngest: nobody after it is left
                entry[2].extend(int(b) for b in alloc(1))
            entry[1] += 1
            i += 1
        step += 1
        held = used = 0
        for entry in running:
            used += entry[1]
            held += len(entry[2]) * block_size if allocator == "paged" else entry[2][1]
        res.held_slot_steps += held
        res.used_slot_steps += used
        res.running_steps += len(running)
        done = [e for e in running if e[1] >= trace[e[0]].final]
        for entry in done:
            release(entry)
            running.remove(entry)
            res.finished += 1
    res.steps = step
    return res


def static_waste(lengths, reserved):
    """Waste of reserving ``reserved`` slots for each of ``lengths`` at one instant (closed form)."""
    lengths = np.asarray(lengths, np.float64)
    return 1.0 - lengths.sum() / (len(lengths) * float(reserved))


def report(seed=3414, n=600, max_context=2048, capacity_tokens=64 * 2048):
    """Markdown table of the three allocators on one synthetic trace."""
    trace = synthetic_trace(n, max_context, seed)
    rows = []
    for alloc, bs in (("contiguous-max", 0), ("contiguous-exact", 0), ("paged", 8), ("paged", 16), ("paged", 32)):
        r = simulate(trace, capacity_tokens, alloc, block_size=bs or 16, max_context=max_context)
        rows.append("| %s%s | %.1f %% | %.1f | %d | %d | %d |" % (
            alloc, " bs=%d" % bs if bs else "", 100 * r.waste, r.mean_batch, r.steps, r.preemptions,
            r.external_failures))
    mean_final = float(np.mean([t.final for t in trace]))
    head = ["trace: %d requests, prompts U[32, 512], outputs log-normal (median 192, sigma 1), mean final "
            "length %.0f tokens, max context %d, budget %d token slots (seed %d)" % (
                n, mean_final, max_context, capacity_tokens, seed), "",
            "| allocator | held memory without KV | mean running requests | steps | preemptions | "
            "external-fragmentation refusals |", "|---|---|---|---|---|---|"]
    return "\n".join(head + rows)


if __name__ == "__main__":
    print(report())
