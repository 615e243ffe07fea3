"""Host bookkeeping: free list, tables, refcounts, fork, copy-on-write."""

import json
import random
from pathlib import Path

import pytest

from paged_kv_cache_339_b200.block_manager import (BlockManager, OutOfBlocks,
                                                   contiguous_reservation_waste,
                                                   lifetime_trace, paged_waste,
                                                   simulate_lifetimes)

GOLDEN = Path(__file__).parent / "golden"


def test_incremental_allocation_and_slots():
    bm = BlockManager(num_blocks=8, block_size=4)
    slots = bm.add_sequence(0, 6)                  # 2 blocks, second half full
    t = bm.tables[0]
    assert len(t) == 2 and bm.num_free_blocks == 6
    assert slots == [t[p // 4] * 4 + p % 4 for p in range(6)]
    s6, cow = bm.append_token(0)                   # fills block 1
    s7, _ = bm.append_token(0)
    assert cow is None and bm.num_free_blocks == 6
    assert (s6, s7) == (t[1] * 4 + 2, t[1] * 4 + 3)
    s8, _ = bm.append_token(0)                     # asks for a new block only now
    assert bm.num_free_blocks == 5 and s8 == bm.tables[0][2] * 4
    bm.check_invariants()


def test_waste_at_most_one_partial_block():
    """Only a sequence's last block can be partly used, so its unused slots
    stay below one block (P1, 'The fix borrowed from operating systems')."""
    rnd = random.Random(0)
    bm = BlockManager(num_blocks=4000, block_size=16)
    for s in range(50):
        bm.add_sequence(s, rnd.randint(1, 300))
        for _ in range(rnd.randint(0, 40)):
            bm.append_token(s)
        assert 0 <= bm.reserved_unused_tokens(s) < 16
    bm.check_invariants()


def test_free_returns_blocks_immediately():
    bm = BlockManager(num_blocks=10, block_size=4)
    bm.add_sequence(0, 9)
    bm.add_sequence(1, 12)
    assert bm.num_free_blocks == 4
    bm.free(0)
    assert bm.num_free_blocks == 7
    bm.add_sequence(2, 28)                          # reuses the returned blocks
    assert bm.num_free_blocks == 0
    with pytest.raises(OutOfBlocks):
        bm.append_token(2)                         # 28 % 4 == 0: needs a block
    bm.check_invariants()


def test_out_of_blocks_leaves_state_intact():
    bm = BlockManager(num_blocks=3, block_size=4)
    bm.add_sequence(0, 8)
    with pytest.raises(OutOfBlocks):
        bm.add_sequence(1, 8)
    assert 1 not in bm.tables and bm.num_free_blocks == 1
    bm.check_invariants()


def test_fork_and_copy_on_write():
    """Siblings share every block; the first to write into the shared partly
    filled block gets a copy, the other then writes in place."""
    bm = BlockManager(num_blocks=20, block_size=4)
    bm.add_sequence(0, 10)                          # blocks a, b, c (c has 2 rows)
    bm.fork(0, 1)
    a, b, c = bm.tables[0]
    assert bm.refcount[c] == 2
    slot0, cow0 = bm.append_token(0)
    assert cow0 is not None and cow0[0] == c and cow0[1] != c
    assert bm.tables[0] == [a, b, cow0[1]] and slot0 == cow0[1] * 4 + 2
    assert bm.refcount[c] == 1
    slot1, cow1 = bm.append_token(1)                # sole owner now
    assert cow1 is None and slot1 == c * 4 + 2
    assert bm.refcount[a] == 2 and bm.refcount[b] == 2
    bm.check_invariants()
    bm.free(0)
    assert bm.refcount[a] == 1 and bm.refcount[cow0[1]] == 0
    bm.free(1)
    assert bm.num_free_blocks == 20
    bm.check_invariants()


def test_fork_on_block_boundary_needs_no_copy():
    bm = BlockManager(num_blocks=10, block_size=4)
    bm.add_sequence(0, 8)                           # both blocks full
    bm.fork(0, 1)
    _, cow = bm.append_token(1)
    assert cow is None and bm.tables[1][:2] == bm.tables[0]
    bm.check_invariants()


def test_prefix_sharing_pays_once():
    """Ten requests with one long prompt point at one physical copy."""
    bm = BlockManager(num_blocks=200, block_size=16)
    bm.add_sequence(0, 512)
    for s in range(1, 10):
        bm.fork(0, s)
    assert bm.num_free_blocks == 200 - 32
    assert all(bm.refcount[b] == 10 for b in bm.tables[0])
    bm.check_invariants()


def test_random_lifecycle_conserves_blocks():
    rnd = random.Random(7)
    bm = BlockManager(num_blocks=300, block_size=8)
    live, nxt = [], 0
    for _ in range(2000):
        op = rnd.random()
        try:
            if op < 0.2 or not live:
                bm.add_sequence(nxt, rnd.randint(1, 60)); live.append(nxt); nxt += 1
            elif op < 0.3:
                bm.fork(rnd.choice(live), nxt); live.append(nxt); nxt += 1
            elif op < 0.45:
                s = live.pop(rnd.randrange(len(live))); bm.free(s)
            else:
                bm.append_token(rnd.choice(live))
        except OutOfBlocks:
            pass
        bm.check_invariants()


def test_worked_example_internal_fragmentation():
    """Max context 4096, average completion 512: ~87% of each contiguous
    reservation is never touched; paging wastes under one block per request."""
    g = json.loads((GOLDEN / "fragmentation_worked_example.json").read_text())
    lens = [g["average_len"]] * 8
    w = contiguous_reservation_waste(g["max_context"], lens)
    assert w == pytest.approx(g["exact_untouched_fraction"], abs=1e-12)
    assert abs(w - g["page_says_untouched_fraction_approx"]) <= 0.0051   # "roughly 87%"
    assert paged_waste(16, lens) == 0.0
    assert paged_waste(16, [513]) == pytest.approx(1 - 513 / 528)


def test_lifetime_simulation_reproduces_the_worked_example():
    """Requests that all end at 512 tokens under a 4096-token maximum: each
    contiguous reservation is 87.5 % untouched at completion ('Paged
    Attention as a Memory Manager', 'The KV-Cache Fragmentation Problem'),
    while 512 = 32 whole blocks of 16 leaves paging nothing unused."""
    g = json.loads((GOLDEN / "fragmentation_worked_example.json").read_text())
    M, L = g["max_context"], g["average_len"]
    # prompt L - 1, one generated token: a single step at length L
    r = simulate_lifetimes([(0, L - 1, 1)] * 10, M, 16, max_live=4)
    assert r["contiguous_waste"] == g["exact_untouched_fraction"]
    assert r["contiguous_waste_at_completion"] == g["exact_untouched_fraction"]
    assert r["paged_waste"] == 0.0 and r["paged_max_unused_slots_per_request"] == 0
    # prompt 1, 511 generated tokens: lengths 2..512 over the lifetime
    r = simulate_lifetimes([(0, 1, L - 1)] * 10, M, 16, max_live=4)
    assert r["contiguous_waste_at_completion"] == g["exact_untouched_fraction"]
    lens = range(2, L + 1)
    assert r["contiguous_waste"] == pytest.approx(1 - sum(lens) / (len(lens) * M), abs=1e-15)
    held = sum(-(-n // 16) * 16 for n in lens)
    assert r["paged_waste"] == pytest.approx(1 - sum(lens) / held, abs=1e-15)
    assert r["paged_waste_at_completion"] == 0.0


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_lifetime_simulation_paged_waste_below_one_block_per_request(bs):
    """A seeded trace of arrivals and completions: every live paged request
    holds fewer than one block of unused slots at every step ('The fix
    borrowed from operating systems'), every block comes back, and paging
    wastes a small fraction of what max-length contiguous slabs do."""
    trace = lifetime_trace(400, 4096, seed=11)
    r = simulate_lifetimes(trace, 4096, bs, max_live=32)
    assert r["all_blocks_returned"]
    assert r["paged_max_unused_slots_per_request"] < bs
    assert r["paged_waste"] < bs / 2 / 256          # mean prompt alone is 256 tokens
    assert r["contiguous_waste"] > 0.6
    assert r["paged_waste"] < r["contiguous_waste"] / 20
    # the two schemes hold the same tokens; only reservations differ
    assert 0.0 <= r["paged_waste_at_completion"] < 1.0


def test_lifetime_trace_is_seeded_and_fits_the_maximum():
    a, b = lifetime_trace(200, 4096, seed=3), lifetime_trace(200, 4096, seed=3)
    assert a == b and a != lifetime_trace(200, 4096, seed=4)
    assert all(1 <= p and 1 <= c and p + c <= 4096 for _, p, c in a)
    assert all(a[i][0] <= a[i + 1][0] for i in range(len(a) - 1))
