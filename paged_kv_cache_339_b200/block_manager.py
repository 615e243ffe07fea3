"""Host-side block bookkeeping for the paged KV cache.

Free list, per-sequence block tables, reference counts, fork and the
copy-on-write decision. Nothing here touches the GPU: it produces the int32
block tables, int64 slot mapping and (src, dst) copy pairs that the three
C-ABI calls consume.

Passages followed:
  * fixed-size blocks and a per-sequence ordered block table; blocks can sit
    anywhere, in any order ("Paged Attention: Virtual Memory for the KV Cache",
    "The fix borrowed from operating systems");
  * incremental allocation: a sequence gets a block, fills it, and asks for the
    next only when it needs one; a finished sequence returns its blocks to the
    shared pool at once (same section; glossary "Paged attention", "What is
    Paged Attention?");
  * prefill assigns logical block indices in order and takes physical blocks
    from a free list ("Paged Attention as a Memory Manager", "How the Kernel
    Executes Paged Attention");
  * several tables may point at one physical block (prefix sharing, parallel
    samples); a sequence about to write into a shared block first gets a
    private copy of it ("Paged Attention: Virtual Memory for the KV Cache",
    "Sharing comes almost for free").
"""

from __future__ import annotations

from collections import deque
from typing import Dict, List, Optional, Tuple


class OutOfBlocks(RuntimeError):
    """The free list is empty. The caller decides what to preempt ("What it
    does not fix": paging pushes the ceiling out but does not remove it)."""


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self._free = deque(range(num_blocks))
        self.refcount = [0] * num_blocks
        self.tables: Dict[int, List[int]] = {}
        self.lengths: Dict[int, int] = {}

    # -- pool ---------------------------------------------------------------
    @property
    def num_free_blocks(self) -> int:
        return len(self._free)

    def _pop(self) -> int:
        if not self._free:
            raise OutOfBlocks("no free KV block")
        b = self._free.popleft()
        assert self.refcount[b] == 0
        self.refcount[b] = 1
        return b

    def _release(self, b: int) -> None:
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            self._free.append(b)

    # -- sequences ----------------------------------------------------------
    def add_sequence(self, seq_id: int, num_tokens: int) -> List[int]:
        """Prefill: logical blocks in order, physical ones from the free list.
        Returns the slot of every prompt token (for a multi-token write)."""
        if seq_id in self.tables:
            raise KeyError(f"sequence {seq_id} exists")
        nb = -(-num_tokens // self.block_size)
        if nb > len(self._free):
            raise OutOfBlocks(f"need {nb} blocks, {len(self._free)} free")
        self.tables[seq_id] = [self._pop() for _ in range(nb)]
        self.lengths[seq_id] = num_tokens
        return [self.slot(seq_id, p) for p in range(num_tokens)]

    def slot(self, seq_id: int, pos: int) -> int:
        """Physical slot of logical position pos: block table[pos // BS],
        offset pos % BS."""
        t = self.tables[seq_id]
        return t[pos // self.block_size] * self.block_size + pos % self.block_size

    def append_token(self, seq_id: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        """Reserve the slot of the next token of seq_id.

        Returns (slot, cow) where cow is a (src, dst) block copy that must run
        before the token is written, or None. A new block is taken only when
        the last one is full; a shared last block is copied first."""
        t = self.tables[seq_id]
        pos = self.lengths[seq_id]
        cow = None
        if pos % self.block_size == 0:
            t.append(self._pop())
        else:
            last = t[-1]
            if self.refcount[last] > 1:
                dst = self._pop()
                self.refcount[last] -= 1
                t[-1] = dst
                cow = (last, dst)
        self.lengths[seq_id] = pos + 1
        return self.slot(seq_id, pos), cow

    def fork(self, parent: int, child: int) -> None:
        """The child shares every block of the parent (parallel sampling)."""
        if child in self.tables:
            raise KeyError(f"sequence {child} exists")
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        for b in self.tables[child]:
            self.refcount[b] += 1

    def free(self, seq_id: int) -> None:
        """Return a finished sequence's blocks; unshared ones go back on the
        free list immediately."""
        for b in self.tables.pop(seq_id):
            self._release(b)
        del self.lengths[seq_id]

    # -- views ----------------------------------------------------------------
    def block_tables(self, seq_ids, stride: Optional[int] = None):
        """int32 [len(seq_ids), stride] table rows padded with 0, as a list of
        lists (the caller turns it into a tensor)."""
        rows = [self.tables[s] for s in seq_ids]
        stride = stride or max([len(r) for r in rows] + [1])
        return [r + [0] * (stride - len(r)) for r in rows]

    def reserved_unused_tokens(self, seq_id: int) -> int:
        """Slots held but not used by seq_id: at most block_size - 1 (only a
        sequence's last block can be partly used, P1 "The fix borrowed from
        operating systems")."""
        return len(self.tables[seq_id]) * self.block_size - self.lengths[seq_id]

    def check_invariants(self) -> None:
        """Every block is either free (refcount 0) or referenced exactly
        refcount times by the tables; nothing is lost or double-owned."""
        counts = [0] * self.num_blocks
        for t in self.tables.values():
            for b in t:
                counts[b] += 1
        free = set(self._free)
        assert len(free) == len(self._free), "block on the free list twice"
        for b in range(self.num_blocks):
            assert counts[b] == self.refcount[b], (b, counts[b], self.refcount[b])
            assert (b in free) == (self.refcount[b] == 0), b


def contiguous_reservation_waste(max_context: int, lengths) -> float:
    """Fraction of a max-length contiguous reservation left untouched when
    requests stop at `lengths` (internal fragmentation of the scheme paging
    replaces; "Paged Attention as a Memory Manager", "The KV-Cache
    Fragmentation Problem")."""
    lengths = list(lengths)
    reserved = max_context * len(lengths)
    return 1.0 - sum(lengths) / reserved


def paged_waste(block_size: int, lengths) -> float:
    """Fraction of allocated slots left untouched under paging: only the last,
    partly filled block of each request wastes anything."""
    lengths = list(lengths)
    reserved = sum(-(-L // block_size) * block_size for L in lengths)
    return 1.0 - sum(lengths) / reserved if reserved else 0.0


def lifetime_trace(num_requests: int, max_context: int, seed: int, mean_prompt: int = 256,
                   mean_completion: int = 512, sigma: float = 1.0, arrivals_per_step: float = 0.5):
    """A seeded request trace: (arrival step, prompt tokens, completion tokens)
    per request. Prompt and completion lengths are log-normal with the given
    means (mu = ln(mean) - sigma^2 / 2), prompts clipped to [1, max_context / 2]
    and completions to [1, max_context - prompt], so every request fits one
    maximum-length reservation; arrivals are Poisson with the given rate.
    The pages give only the maximum context (4096) and the average completion
    (512) of their worked example; the distributions are a plain choice."""
    import math
    import random
    rnd = random.Random(seed)

    def lognormal(mean):
        return math.exp(math.log(mean) - sigma * sigma / 2.0 + sigma * rnd.gauss(0.0, 1.0))

    trace, t = [], 0.0
    for _ in range(num_requests):
        t += rnd.expovariate(arrivals_per_step)
        p = min(max(1, round(lognormal(mean_prompt))), max_context // 2)
        c = min(max(1, round(lognormal(mean_completion))), max_context - p)
        trace.append((int(t), p, c))
    return trace


def simulate_lifetimes(trace, max_context: int, block_size: int, max_live: int):
    """Run a request trace through both allocation schemes, step by step.

    A request is admitted (first come, first served) once it has arrived and
    fewer than `max_live` requests are live; it is prefilled with its prompt,
    then generates one token per step until its completion length is reached,
    and is freed. Both schemes see the same admissions, so they hold the same
    tokens at every step and differ only in what they reserve:
      * contiguous: a slab of `max_context` slots per live request, reserved
        at admission ("Paged Attention as a Memory Manager", "The KV-Cache
        Fragmentation Problem"; "Paged Attention: Virtual Memory for the KV
        Cache", first section);
      * paged: this module's BlockManager, a block at a time as tokens arrive
        ("The fix borrowed from operating systems").
    Returns the reserved-but-unused fraction of each scheme, summed over all
    steps (time-averaged) and at each request's completion, the largest
    number of unused slots one live paged request ever held, and whether the
    pool got every block back."""
    import math
    total_tokens = sum(p + c for _, p, c in trace)
    bm = BlockManager(num_blocks=max(1, min(max_live, len(trace)) *
                                     math.ceil(max_context / block_size)),
                      block_size=block_size)
    pending = sorted(range(len(trace)), key=lambda i: (trace[i][0], i))
    live = {}            # request -> tokens still to generate
    nxt, step = 0, 0
    used_sum = contig_sum = paged_sum = 0
    fin_used = fin_contig = fin_paged = 0
    max_unused = 0
    while nxt < len(pending) or live:
        while nxt < len(pending) and len(live) < max_live and trace[pending[nxt]][0] <= step:
            r = pending[nxt]
            bm.add_sequence(r, trace[r][1])
            live[r] = trace[r][2]
            nxt += 1
        done = []
        for r in live:
            bm.append_token(r)
            live[r] -= 1
            if live[r] == 0:
                done.append(r)
        used = sum(bm.lengths[r] for r in live)
        held = sum(len(bm.tables[r]) for r in live) * block_size
        used_sum += used
        contig_sum += len(live) * max_context
        paged_sum += held
        max_unused = max([max_unused] + [bm.reserved_unused_tokens(r) for r in live])
        for r in done:
            fin_used += bm.lengths[r]
            fin_contig += max_context
            fin_paged += len(bm.tables[r]) * block_size
            bm.free(r)
            del live[r]
        step += 1
    bm.check_invariants()
    assert fin_used == total_tokens
    return {
        "requests": len(trace), "steps": step, "max_context": max_context,
        "block_size": block_size, "max_live": max_live,
        "contiguous_waste": 1.0 - used_sum / contig_sum if contig_sum else 0.0,
        "paged_waste": 1.0 - used_sum / paged_sum if paged_sum else 0.0,
        "contiguous_waste_at_completion": 1.0 - fin_used / fin_contig if fin_contig else 0.0,
        "paged_waste_at_completion": 1.0 - fin_used / fin_paged if fin_paged else 0.0,
        "paged_max_unused_slots_per_request": max_unused,
        "all_blocks_returned": bm.num_free_blocks == bm.num_blocks,
    }
