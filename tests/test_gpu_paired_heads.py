"""Paired KV heads on the tensor-core path (block size 8).

A block stores its KV heads one after the other ("Paged Attention as a Memory
Manager", "Virtual Memory as the Blueprint": a block holds the keys and
values of a fixed number of tokens), so at block size 8 the tensor-core
kernel loads the pages of KV heads 2j and 2j + 1 of a block with one copy and
treats the pair as one head of 2G query heads (G = 4 or 8), each score kept
for its own KV head's query heads only. pa_decode pairs heads with at least
two pairs per item stream, or with fewer pairs than streams when the longest
context allowed leaves the halved pieces above the workspace's smallest
split. The output must match the fp64 oracle element by element within the
decode tolerance, whatever the lengths, pieces and head layouts, and the
plan must count the work in pairs exactly when the kernel pairs.
"""

import numpy as np
import pytest
import torch

from oracle import ORACLE
from paged_kv_cache_339_b200 import build as pa_build
from paged_kv_cache_339_b200 import ops
from paged_kv_cache_339_b200 import workloads as W
from tests.gpu_helpers import (TOL, f64, max_abs_err, oracle_step, pool_f64, reference_rows,
                               run_step)

pytestmark = pytest.mark.gpu

H_NUM_ITEMS, H_NUM_PAIRS = 2, 3   # header words: items, (sequence, piece) pairs


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pa_build.build()
    ops.library()


def batch(lens, dtype, Hq, Hkv, BS=8, seed=31):
    gen = torch.Generator().manual_seed(seed)
    NB = sum((L + BS - 1) // BS for L in lens) + 6
    tables = W._place(lens, BS, NB, gen)
    return W._assemble("paired", dtype, BS, Hq, Hkv, 128, lens, tables, NB, gen, seed, "cuda")


def streams():
    """Item streams of the tensor-core kernel: two per SM."""
    return 2 * torch.cuda.get_device_properties(0).multi_processor_count


def auto_min_split(max_ctx):
    """The workspace's smallest automatic split (pa_workspace.h)."""
    return max(256, -(-(-(-max_ctx // 64)) // 128) * 128)


def expect_paired(B, Hkv, G, BS, max_ctx):
    """pa_decode's choice to read KV heads in pairs (without shared prefixes)."""
    if BS != 8 or Hkv % 2 or G not in (4, 8):
        return False
    units = B * (Hkv // 2)
    if units >= 2 * streams():
        return True
    if units >= streams():
        return False
    return B * max_ctx * Hkv // streams() // 4 >= auto_min_split(max_ctx)


def paired_lens(lens, Hkv):
    """`lens` repeated until the batch has at least two KV-head pairs per
    item stream (the fewest for which pa_decode pairs heads)."""
    reps = -(-2 * streams() // (len(lens) * (Hkv // 2)))
    return lens * reps


def decode(b, split):
    """Decode only; returns the output and the plan's (items, pairs)."""
    B, Hq, D = b.q.shape
    max_ctx = max(b.max_context_len, 1)
    ws = ops.decode_workspace(B, Hq, D, max_ctx, b.block_size, split)
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    ops.pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, max_ctx,
                  b.scale, ws, split_tokens=split, path=ops.PA_PATH_TCGEN05)
    torch.cuda.synchronize()
    assert ops.pa_decode_status(ws) == ops.PA_OK
    words = ws[:64].cpu().numpy().view(np.int32)
    return out, int(words[H_NUM_ITEMS]), int(words[H_NUM_PAIRS])


LENS = [0, 1, 2, 7, 8, 9, 31, 32, 33, 63, 64, 65, 127, 128, 129, 300, 1000, 1, 4099]

# (dtype, query heads, KV heads, with at least two KV-head pairs per stream)
LAYOUTS = [
    (torch.bfloat16, 16, 4, True),    # G = 4: two KV heads fill the 8-row tile
    (torch.float16, 16, 4, True),
    (torch.bfloat16, 8, 2, True),     # one pair
    (torch.bfloat16, 32, 8, True),    # four pairs
    (torch.bfloat16, 32, 4, True),    # G = 8: two KV heads fill the 16-row tile
    (torch.float16, 32, 4, True),
    (torch.bfloat16, 12, 3, False),   # odd KV heads: one head per item
    (torch.float16, 64, 4, False),    # G = 16: one head per item
]


_REF = {}


@pytest.mark.parametrize("dtype,Hq,Hkv,paired", LAYOUTS)
@pytest.mark.parametrize("split", [0, 32, 64, 200])
def test_matches_oracle(dtype, Hq, Hkv, paired, split):
    b = batch(paired_lens(LENS, Hkv) if paired else LENS, dtype, Hq, Hkv)
    assert expect_paired(b.q.shape[0], Hkv, Hq // Hkv, 8, b.max_context_len) == paired
    bc = b.to("cpu")
    out, items, pairs = decode(b, split)
    # the plan counts (sequence, piece) pairs x KV heads, halved when paired
    assert items == pairs * (Hkv // 2 if paired else Hkv)
    o = out.cpu()
    key = (dtype, Hq, Hkv, paired)
    if key not in _REF:   # the batch is seeded: one oracle run per layout
        _REF[key] = ORACLE.decode(*oracle_inputs(bc))
    ref = _REF[key]
    assert max_abs_err(out, ref) <= TOL[dtype]
    assert torch.count_nonzero(o[0]) == 0
    G = Hq // Hkv
    # one token: its stored value, exactly (the pair's other head adds zeros)
    vp = pool_f64(bc.v_cache)
    blk = int(bc.block_tables[1, 0])
    for h in range(Hq):
        assert np.array_equal(o[1, h].numpy().astype(np.float64), vp[blk, h // G, 0])


def test_few_short_sequences_are_not_paired():
    """Fewer than two KV-head pairs per item stream, and contexts too short
    for halved pieces: one head per item."""
    lens = [L for L in LENS if L <= 1000]
    b = batch(lens, torch.bfloat16, 16, 4)
    assert not expect_paired(len(lens), 4, 4, 8, max(lens))
    _, items, pairs = decode(b, 0)
    assert items == pairs * 4


@pytest.mark.parametrize("Hq", [32, 64])
def test_few_long_sequences_are_paired(Hq):
    """Four long sequences (8 KV heads, 4 or 8 query heads each): fewer pairs
    than streams, but long enough contexts: paired, split into pieces and
    merged. Every query head of each sequence's first KV pair against the
    oracle, every row against the CUDA-core path."""
    lens = [20000, 33001, 47007, 60000]
    b = batch(lens, torch.bfloat16, Hq, 8, seed=37)
    G = Hq // 8
    assert expect_paired(4, 8, G, 8, max(lens))
    out, items, pairs = decode(b, 0)
    assert items == pairs * 4
    simt = run_step(b, path=ops.PA_PATH_SIMT, write=False)
    assert float((out - simt).abs().max()) <= 2e-3
    for seq in range(4):
        heads = list(range(2 * G))
        ref = reference_rows(b, seq, heads)
        for h in heads:
            row = out[seq, h].cpu().numpy().astype(np.float64)
            assert np.max(np.abs(row - ref[h])) <= 2e-3, (seq, h)


def oracle_inputs(bc):
    return (f64(bc.q), pool_f64(bc.k_cache), pool_f64(bc.v_cache), bc.block_tables.numpy(),
            bc.context_lens.numpy(), float(np.float32(bc.scale)))


def test_nan_in_unread_slots_does_not_leak():
    """Slots past each sequence's end (inside its last block, which the paired
    copy loads whole for both heads) and unused blocks are NaN."""
    lens = paired_lens([5, 33, 100, 250, 8, 9], 8)
    b = batch(lens, torch.bfloat16, 32, 8)
    used = torch.zeros(b.num_blocks, b.block_size, dtype=torch.bool)
    bt = b.block_tables.cpu()
    for i, L in enumerate(lens):
        for j in range(L):
            used[bt[i, j // b.block_size], j % b.block_size] = True
    logical = (~used)[:, None, :, None].expand(b.k_cache.shape).numpy()
    mask = torch.from_numpy(ORACLE.physical_pool(np.ascontiguousarray(logical))).cuda()
    b.k_cache[mask] = float("nan")
    b.v_cache[mask] = float("nan")
    bc = b.to("cpu")
    for split in (0, 64):
        out, items, pairs = decode(b, split)
        assert items == pairs * 4
        assert max_abs_err(out, ORACLE.decode(*oracle_inputs(bc))) <= 2e-3


def test_step_with_write():
    """The whole step (KV write, then decode) of a GQA batch at block size 8
    (32 / 8 heads) against the oracle's step."""
    b = W.gqa("cuda", num_seqs=streams() // 2, max_len=700, block_size=8)
    bc = b.to("cpu")
    out = run_step(b, path=ops.PA_PATH_TCGEN05)
    assert max_abs_err(out, oracle_step(bc)) <= 2e-3


def mixed_long(BS=8, seed=41):
    """A GQA batch (32 / 8 heads) of log-normal lengths with four long
    sequences among them, whose many pieces are merged."""
    gen = torch.Generator().manual_seed(seed)
    lens = W.lognormal_lens(streams() // 2, 512, 1.0, 16, 4096, gen)
    lens[3], lens[40], lens[77], lens[100] = 20000, 33001, 47007, 65536
    NB = sum((L + BS - 1) // BS for L in lens) + 8
    tables = W._place(lens, BS, NB, gen)
    return W._assemble("mixed_long", torch.bfloat16, BS, 32, 8, 128, lens, tables, NB, gen, seed,
                       "cuda")


@pytest.mark.parametrize("name", ["gqa_bs8", "mixed_long"])
def test_full_size(name):
    """Full-size GQA (256 sequences, 32 / 8 heads) and a batch with four long
    sequences among short ones, at block size 8: every row against the
    CUDA-core path, sampled rows against the oracle (the long sequences'
    first KV pair in full)."""
    b = W.gqa("cuda", block_size=8) if name == "gqa_bs8" else mixed_long()
    B, Hq, D = b.q.shape
    outs = {}
    for path in (ops.PA_PATH_TCGEN05, ops.PA_PATH_SIMT):
        outs[path] = run_step(b, path=path, write=False)
    assert float((outs[ops.PA_PATH_TCGEN05] - outs[ops.PA_PATH_SIMT]).abs().max()) <= 2e-3
    got = outs[ops.PA_PATH_TCGEN05]
    rng = np.random.default_rng(17)
    G = Hq // b.num_kv_heads
    picks = [(int(s), list(range(2 * G))) for s in rng.choice(B, 4, replace=False)]
    if name == "mixed_long":
        picks += [(s, list(range(2 * G))) for s in (3, 40, 77, 100)]
    for seq, heads in picks:
        ref = reference_rows(b, seq, heads)
        for h in heads:
            row = got[seq, h].cpu().numpy().astype(np.float64)
            assert np.max(np.abs(row - ref[h])) <= 2e-3, (seq, h)
