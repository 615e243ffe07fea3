"""Several decode steps driven by the host block manager, on the GPU, against
the oracle replaying the same host-side operations.

Parallel samples of one prompt share its blocks; when one sibling is about to
write into a shared, partly filled block it first gets its own copy of it
("Paged Attention: Virtual Memory for the KV Cache", "Sharing comes almost for
free"). Here BlockManager decides everything (slots, new blocks, copy-on-write
pairs, freed and reused blocks, tables) and the three C-ABI calls carry it
out, step after step: pa_copy_blocks, then pa_write_kv, then pa_decode.

Per pair of siblings a third sequence (the observer) shares the pair's blocks
and never steps: every sibling write into a block it shares must go to a copy,
so the K/V the observer's table reaches stays bit-identical at every step. After each step the
sibling that diverged first is freed and forked again from its partner, so the
next step diverges again inside a shared partial block, and its private blocks
go back to the free list to be reused.
"""

import numpy as np
import pytest
import torch

from oracle import ORACLE
from paged_kv_cache_339_b200 import build as pa_build
from paged_kv_cache_339_b200 import ops
from paged_kv_cache_339_b200.block_manager import BlockManager
from tests.gpu_helpers import TOL, bits, max_abs_err, pool_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pa_build.build()
    ops.library()


def _f64(logical_bits):
    """fp16 bit patterns (int16) to fp64 values, exactly."""
    return logical_bits.view(np.float16).astype(np.float64)


class Mirror:
    """The device pools and their host copy, kept in step: every operation is
    applied to the device through the C-ABI and to the host copy through the
    oracle (raw fp16 bit patterns in the logical layout, so both are data
    movement only and compare bit for bit)."""

    def __init__(self, NB, H, BS, D, gen):
        self.k = torch.randn((NB, H, BS, D), generator=gen).to(torch.float16).cuda()
        self.v = torch.randn((NB, H, BS, D), generator=gen).to(torch.float16).cuda()
        self.kb, self.vb = pool_bits(self.k), pool_bits(self.v)
        self.H, self.D, self.gen = H, D, gen

    def copy(self, pairs):
        if not pairs:
            return
        t = torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2)
        ops.pa_copy_blocks(self.k, self.v, t.cuda())
        self.kb, self.vb = ORACLE.copy_blocks(self.kb, self.vb, t.numpy())

    def write(self, slots):
        T = len(slots)
        key = torch.randn((T, self.H, self.D), generator=self.gen).to(torch.float16)
        val = torch.randn((T, self.H, self.D), generator=self.gen).to(torch.float16)
        s = torch.tensor(slots, dtype=torch.int64)
        ops.pa_write_kv(self.k, self.v, key.cuda(), val.cuda(), s.cuda())
        self.kb, self.vb = ORACLE.write_kv(self.kb, self.vb, bits(key), bits(val), s.numpy())

    def check_bit_exact(self):
        torch.cuda.synchronize()
        assert np.array_equal(pool_bits(self.k), self.kb)
        assert np.array_equal(pool_bits(self.v), self.vb)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2)], ids=["mha_simt", "gqa4_tc"])
def test_allocator_driven_decode_steps(Hq, Hkv):
    BS, D, NB = 16, 128, 160
    num_pairs, prefix_len, steps = 3, 64, 6
    gen = torch.Generator().manual_seed(339)
    rng = np.random.default_rng(339)
    bm = BlockManager(NB, BS)
    m = Mirror(NB, Hkv, BS, D, gen)

    # prompt: one prefix, written as a multi-token write
    root = 100
    m.write(bm.add_sequence(root, prefix_len))
    # per pair: a sibling A with its own suffix (not a whole number of
    # blocks), then B and the observer O forked from A
    seqs = []                      # [A, B, O] ids per pair
    for j in range(num_pairs):
        a, b, o = 3 * j, 3 * j + 1, 3 * j + 2
        bm.fork(root, a)
        s = int(rng.integers(1, 60))
        while s % BS == 0:
            s = int(rng.integers(1, 60))
        slots, pairs = [], []
        for _ in range(s):
            slot, cow = bm.append_token(a)
            slots.append(slot)
            if cow:
                pairs.append(cow)
        m.copy(pairs)
        m.write(slots)
        bm.fork(a, b)
        bm.fork(a, o)
        seqs.append([a, b, o])
    bm.free(root)                  # the prefix stays: the pairs still hold it
    bm.check_invariants()
    m.check_bit_exact()

    order = [x for p in seqs for x in p]
    scale = 1.0 / np.sqrt(D)
    q = torch.randn((len(order), Hq, D), generator=gen).to(torch.float16)
    ws = ops.decode_workspace(len(order), Hq, D, 4096, BS)
    observer_out = None
    for step in range(steps):
        # one sibling of each pair (seeded coin) writes first: it copies the
        # shared partial block; the other then writes in place or, where the
        # observer still shares that block with it, copies too
        slots, pairs, first = [], [], []
        # a partly filled last block held by r sequences is copied by each
        # sibling that still shares it when it writes: twice while the
        # observer holds it too (r = 3), once when only the siblings do; a
        # full last block is never copied (both siblings take new blocks)
        expect = 0
        for a, _, _ in seqs:
            if bm.lengths[a] % BS != 0:
                r = bm.refcount[bm.tables[a][-1]]
                expect += (r > 1) + (r > 2)
        for a, b, o in seqs:
            d, k = (a, b) if rng.integers(0, 2) == 0 else (b, a)
            first.append((d, k))
            for sid in (d, k):
                slot, cow = bm.append_token(sid)
                slots.append(slot)
                if cow:
                    pairs.append(cow)
        assert len(pairs) == expect, step
        m.copy(pairs)
        m.write(slots)
        bm.check_invariants()
        lens = [bm.lengths[s] for s in order]
        bt = torch.tensor(bm.block_tables(order), dtype=torch.int32)
        out = torch.full((len(order), Hq, D), float("nan"), device="cuda")
        ops.pa_decode(out, q.cuda(), m.k, m.v, bt.cuda(),
                      torch.tensor(lens, dtype=torch.int32).cuda(), max(lens), scale, ws)
        torch.cuda.synchronize()
        assert ops.pa_decode_status(ws) == ops.PA_OK
        m.check_bit_exact()
        ref = ORACLE.decode(_f64(bits(q)), _f64(m.kb), _f64(m.vb), bt.numpy(),
                            np.asarray(lens), float(np.float32(scale)))
        assert max_abs_err(out, ref) <= TOL[torch.float16], step
        # the observers never stepped: the K/V their tables reach is bit for
        # bit what it was at the first step (the device pools equal the
        # mirror, checked above), and their rows stay what they were to
        # within the tolerance (the work plan may cut them differently as
        # the batch around them grows, which changes only fp32 rounding)
        obs_kv = []
        for _, _, o in seqs:
            tab = bm.tables[o]
            obs_kv.append((m.kb[tab].copy(), m.vb[tab].copy()))
        obs = out[[order.index(o) for _, _, o in seqs]].cpu()
        if observer_out is None:
            observer_out, observer_kv = obs, obs_kv
        for (k0, v0), (k1, v1) in zip(observer_kv, obs_kv):
            assert np.array_equal(k0, k1) and np.array_equal(v0, v1), step
        assert (obs - observer_out).abs().max().item() <= TOL[torch.float16], step
        # re-fork: the sibling that diverged first drops its private blocks
        # and shares its partner's table again
        for d, k in first:
            bm.free(d)
            bm.fork(k, d)
        bm.check_invariants()
    for p in seqs:
        for s in p:
            bm.free(s)
    bm.check_invariants()
    assert bm.num_free_blocks == NB
