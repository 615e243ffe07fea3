"""The work plan a decode call leaves in its workspace.

The planning kernel cuts every sequence into pieces (work pairs) and lists
them longest first. Whatever the cut, the pieces of a sequence must tile its
context exactly once, carry split indices 0..n-1 with n = the recorded split
count (at most the workspace's split capacity), and the list must be sorted
by 128-token chunk count, longest first. Checked on the workspace after real
calls, at full size and with explicit split sizes.
"""

import numpy as np
import pytest
import torch

from paged_kv_cache_339_b200 import build as pa_build
from paged_kv_cache_339_b200 import ops
from paged_kv_cache_339_b200 import workloads as W
from tests.gpu_helpers import run_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pa_build.build()
    ops.library()


def _align256(x):
    return (x + 255) // 256 * 256


def read_plan(ws, num_seqs):
    raw = ws.cpu().numpy()
    hdr = raw[:256].view(np.int32)
    status, num_items, num_pairs, split_tokens, max_splits = (int(hdr[0]), int(hdr[2]),
                                                              int(hdr[3]), int(hdr[4]), int(hdr[5]))
    pairs = raw[256:256 + 16 * num_pairs].view(np.int32).reshape(num_pairs, 4)
    nsplit_off = 256 + _align256(num_seqs * max_splits * 16)
    nsplit = raw[nsplit_off:nsplit_off + 4 * num_seqs].view(np.int32)
    return dict(status=status, num_items=num_items, split_tokens=split_tokens,
                max_splits=max_splits, pairs=pairs, nsplit=nsplit)


def check_plan(plan, lens, num_kv_heads, explicit_split=0):
    assert plan["status"] == 0
    pairs, nsplit, ms, S = plan["pairs"], plan["nsplit"], plan["max_splits"], plan["split_tokens"]
    assert plan["num_items"] == len(pairs) * num_kv_heads
    if explicit_split:
        assert S == explicit_split
    seq, splitix, n, tb, te = (pairs[:, 0], pairs[:, 1] & 0xFFFF, pairs[:, 1] >> 16,
                             pairs[:, 2], pairs[:, 3])
    assert np.all(te > tb)
    # longest first, by 128-token chunk count (capped at 64 chunks)
    key = np.minimum((te - tb + 127) // 128, 64)
    assert np.all(np.diff(key) <= 0), "pairs not sorted longest first"
    for i, L in enumerate(lens):
        mine = np.nonzero(seq == i)[0]
        assert len(mine) == nsplit[i], (i, len(mine), nsplit[i])
        if L == 0:
            assert nsplit[i] == 0
            continue
        assert 1 <= nsplit[i] <= ms
        assert np.all(n[mine] == nsplit[i])
        order = np.argsort(splitix[mine])
        assert np.array_equal(splitix[mine][order], np.arange(nsplit[i]))
        b, e = tb[mine][order], te[mine][order]
        assert b[0] == 0 and e[-1] == L and np.array_equal(b[1:], e[:-1]), f"seq {i} not tiled"
        if explicit_split:
            assert np.all(e - b <= explicit_split)
            assert np.all((e - b)[:-1] == explicit_split)


@pytest.mark.parametrize("name,split", [("gqa", 0), ("long", 0), ("mha", 0), ("prefix_cow", 0),
                                        ("gqa", 384), ("long", 4096)])
def test_plan_tiles_every_sequence_longest_first(name, split):
    b = W.FULL[name]("cuda")
    B, Hq, D = b.q.shape
    ws = ops.decode_workspace(B, Hq, D, b.max_context_len, b.block_size, split)
    run_step(b, split_tokens=split, workspace=ws, write=False)
    plan = read_plan(ws, B)
    check_plan(plan, b.context_lens.cpu().tolist(), b.num_kv_heads, split)


def test_plan_cuts_tails_when_sequences_are_few_and_long():
    # a few long sequences: the automatic split must leave short pieces for the
    # end of the list, not only whole split-size pieces
    b = W.FULL["long"]("cuda")
    B, Hq, D = b.q.shape
    ws = ops.decode_workspace(B, Hq, D, b.max_context_len, b.block_size)
    run_step(b, workspace=ws, write=False)
    plan = read_plan(ws, B)
    sizes = plan["pairs"][:, 3] - plan["pairs"][:, 2]
    S = plan["split_tokens"]
    assert sizes[0] == S
    assert np.sum(sizes <= S // 2) >= 64, "no short pieces at the end of the list"


@pytest.mark.parametrize("name", ["gqa", "long"])
def test_automatic_split_is_a_share_or_half_a_share(name):
    """The automatic split on the tensor-core path (one CTA per SM, two item
    streams each): one stream's share of the token-heads, rounded up to 128
    tokens, or half a share when the (sequence, KV head) units are fewer than
    the streams; never below the smallest split the workspace allows."""
    b = W.FULL[name]("cuda")
    B, Hq, D = b.q.shape
    ws = ops.decode_workspace(B, Hq, D, b.max_context_len, b.block_size)
    run_step(b, workspace=ws, write=False)
    plan = read_plan(ws, B)
    lens = b.context_lens.cpu().tolist()
    streams = 2 * torch.cuda.get_device_properties(0).multi_processor_count
    share = -(-sum(lens) * b.num_kv_heads // streams)
    base = share if B * b.num_kv_heads >= streams else (share + 1) // 2
    up128 = lambda x: -(-x // 128) * 128
    min_split = max(256, up128(-(-max(lens) // 64)))
    assert plan["split_tokens"] == max(up128(base), min_split)
    # gqa has more units than streams, the long workload fewer
    assert (B * b.num_kv_heads < streams) == (name == "long")



@pytest.mark.parametrize("case", ["many", "few_short", "few_long"])
def test_paired_heads_cut_half_pieces(case):
    """At block size 8 the tensor-core kernel reads KV heads of 4 query heads
    in pairs with at least two pairs per item stream ("many"), or with fewer
    pairs than streams when the longest context allowed leaves the halved
    pieces above the workspace's smallest split ("few_long"), not for a few
    short sequences ("few_short"). Paired, the items are (piece, pair of KV
    heads) and the automatic split is half the one-head split (a piece of the
    same work), never below the smallest split the workspace allows; the
    pieces still tile every sequence."""
    streams = 2 * torch.cuda.get_device_properties(0).multi_processor_count
    if case == "many":
        b = W.gqa("cuda", num_seqs=256, block_size=8)
    elif case == "few_short":
        b = W.gqa("cuda", num_seqs=16, max_len=600, block_size=8)
    else:
        b = W.long_context("cuda", num_q_heads=32, block_size=8)
    B, Hq, D = b.q.shape
    paired = case != "few_short"
    ws = ops.decode_workspace(B, Hq, D, b.max_context_len, b.block_size)
    run_step(b, workspace=ws, write=False)
    plan = read_plan(ws, B)
    lens = b.context_lens.cpu().tolist()
    check_plan(plan, lens, b.num_kv_heads // 2 if paired else b.num_kv_heads)
    share = -(-sum(lens) * b.num_kv_heads // streams)
    base = share if B * b.num_kv_heads >= streams else (share + 1) // 2
    up128 = lambda x: -(-x // 128) * 128
    min_split = max(256, up128(-(-b.max_context_len // 64)))
    one_head = max(up128(base), min_split)
    assert plan["split_tokens"] == (max(one_head // 2, min_split) if paired else one_head)
