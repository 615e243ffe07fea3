"""Shared prefixes read once per group (pa_decode_options.share_prefixes).

Sequences forked from one another point at the same physical blocks for
their common prefix ("Paged Attention: Virtual Memory for the KV Cache",
"Sharing comes almost for free"). With the option on, the plan groups runs
of consecutive sequences whose tables start with the same blocks and a
separate launch computes their common whole pieces once per group (tensor
cores for 16-bit KV with head_dim 128, else CUDA cores); each member's own
pieces run in the usual launch, which merges them.
The output must match the fp64 oracle within the decode tolerance, and the
per-sequence path within fp32 rounding, whatever the run lengths, prefix
lengths, group sizes and head layouts.
"""

import numpy as np
import pytest
import torch

from oracle import ORACLE
from paged_kv_cache_339_b200 import build as pa_build
from paged_kv_cache_339_b200 import ops
from paged_kv_cache_339_b200 import workloads as W
from tests.gpu_helpers import TOL, f64, max_abs_err, pool_f64, sampled_reference

pytestmark = pytest.mark.gpu

H_GROUP_ITEMS = 8   # header word: group list entries x KV heads


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pa_build.build()
    ops.library()


def shared_batch(runs, dtype=torch.float16, Hq=4, Hkv=4, D=128, BS=16, seed=21):
    """runs: list of (prefix_tokens, [own tokens of each sequence]); the
    sequences of a run share the prefix's physical blocks (prefix_tokens a
    multiple of BS), then continue in private blocks."""
    gen = torch.Generator().manual_seed(seed)
    lens, need = [], 0
    for pre, owns in runs:
        assert pre % BS == 0
        need += pre // BS
        for o in owns:
            lens.append(pre + o)
            need += (o + BS - 1) // BS
    NB = need + 4
    perm = torch.randperm(NB, generator=gen).tolist()
    tables, k = [], 0
    for pre, owns in runs:
        shared = perm[k:k + pre // BS]
        k += pre // BS
        for o in owns:
            nb = (o + BS - 1) // BS
            tables.append(shared + perm[k:k + nb])
            k += nb
    return W._assemble("shared", dtype, BS, Hq, Hkv, D, lens, tables, NB, gen, seed, "cuda")


def decode(b, share, split=0, path=ops.PA_PATH_SIMT):
    B, Hq, D = b.q.shape
    ws = ops.decode_workspace(B, Hq, D, b.max_context_len, b.block_size, split)
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    ops.pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                  b.max_context_len, b.scale, ws, split_tokens=split, path=path,
                  share_prefixes=share)
    torch.cuda.synchronize()
    assert ops.pa_decode_status(ws) == ops.PA_OK
    groups = int(ws[:64].cpu().numpy().view(np.int32)[H_GROUP_ITEMS])
    return out, groups


CASES = {
    # one run of 6 sequences behind a 1024-token prefix (two 512-token pieces)
    "one_run": dict(runs=[(1024, [5, 17, 300, 64, 1, 700])]),
    # a prefix that is not a multiple of the piece size next to a run of 2, a
    # sequence sharing nothing, and sequences whose own part is one token or
    # ends on a piece boundary
    "mixed": dict(runs=[(784, [40, 513]), (0, [333]), (1536, [16, 1, 1000, 47]),
                        (512, [512, 3])]),
    # 20 sequences behind one prefix: two groups (16 rows each, then 4)
    "two_groups": dict(runs=[(640, [i * 37 % 300 + 1 for i in range(20)])]),
    # GQA 8/2 on the CUDA-core path: 4 heads per KV head, 4 members per group
    "gqa_simt": dict(runs=[(1024, [100, 200, 300, 400, 500, 7])], Hq=8, Hkv=2,
                     dtype=torch.bfloat16),
    # fp32, head_dim 64, block size 8: groups on the CUDA cores
    "fp32_d64_bs8": dict(runs=[(768, [9, 90, 900])], dtype=torch.float32, D=64, BS=8),
    # bf16 head_dim 64: groups on the CUDA cores
    "bf16_d64": dict(runs=[(512, [1, 200, 513])], dtype=torch.bfloat16, D=64),
    # block size 32, MHA with 2 heads
    "bs32": dict(runs=[(2048, [31, 33, 64, 1])], Hq=2, Hkv=2, BS=32),
    # GQA on the tensor-core path: groups of 4 sequences x 4 heads, own
    # pieces merged by the tensor-core kernel's merge tasks
    "gqa_tc": dict(runs=[(1024, [100, 200, 300, 400, 500, 7, 64]), (256, [3, 300])],
                   Hq=16, Hkv=4, dtype=torch.bfloat16, path=ops.PA_PATH_TCGEN05),
    # G = 8 (2 sequences a group) and G = 2 (8 sequences a group)
    "g8_tc": dict(runs=[(1536, [10, 20, 30])], Hq=16, Hkv=2, dtype=torch.bfloat16,
                  path=ops.PA_PATH_TCGEN05),
    "g2": dict(runs=[(640, [50, 60, 70, 80, 90, 100, 110, 120, 130])], Hq=8, Hkv=4),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("split", [0, 256])
def test_matches_oracle_and_per_sequence_path(name, split):
    kw = dict(CASES[name])
    path = kw.pop("path", ops.PA_PATH_SIMT)
    b = shared_batch(**kw)
    bc = b.to("cpu")
    # the batch as it stands (decode only, no write)
    ref = ORACLE.decode(f64(bc.q), pool_f64(bc.k_cache), pool_f64(bc.v_cache),
                        bc.block_tables.numpy(), bc.context_lens.numpy(),
                        float(np.float32(bc.scale)))
    shared, groups = decode(b, True, split, path)
    private, none = decode(b, False, split, path)
    assert none == 0
    assert groups > 0, "no group formed"
    tol = TOL[b.dtype]
    assert max_abs_err(shared, ref) <= tol
    assert max_abs_err(private, ref) <= tol
    assert float((shared - private).abs().max()) <= 1e-4


def test_block_size_8_many_sequences_against_paired_heads():
    """Shared prefixes at block size 8 on the tensor cores (16-row group
    tiles of 8-token pages), in a batch large enough that, with the option
    off, pa_decode reads its KV heads in pairs: the two paths must agree, and
    both match the oracle on sampled rows."""
    rng = np.random.default_rng(13)
    runs = [(int(rng.choice([256, 512, 768])), [int(x) for x in rng.integers(1, 400, 5)])
            for _ in range(60)]
    b = shared_batch(runs, dtype=torch.bfloat16, Hq=16, Hkv=4, BS=8)
    streams = 2 * torch.cuda.get_device_properties(0).multi_processor_count
    assert b.q.shape[0] * 2 >= 2 * streams   # enough KV-head pairs to pair them
    shared, groups = decode(b, True, path=ops.PA_PATH_TCGEN05)
    private, none = decode(b, False, path=ops.PA_PATH_TCGEN05)
    assert groups > 0 and none == 0
    assert float((shared - private).abs().max()) <= 1e-4
    for seq in rng.choice(b.q.shape[0], 6, replace=False):
        for h in rng.choice(16, 4, replace=False):
            ref = sampled_reference(b, int(seq), int(h))
            got = shared[int(seq), int(h)].cpu().numpy().astype(np.float64)
            assert np.max(np.abs(got - ref)) <= 2e-3


def test_off_where_it_does_not_apply():
    """No groups for 16 query heads per KV head (a group would have one
    sequence), for a batch of one sequence, or for prefixes under 256 tokens."""
    b = shared_batch([(1024, [10, 20, 30, 40])], dtype=torch.bfloat16, Hq=16, Hkv=1)
    assert decode(b, True, path=ops.PA_PATH_TCGEN05)[1] == 0
    assert decode(shared_batch([(1024, [10])]), True)[1] == 0
    assert decode(shared_batch([(240, [10, 20, 30])]), True)[1] == 0


def test_full_size_prefix_cow_step():
    """The prefix + copy-on-write step at full size with groups: sampled rows
    against the oracle, every row against the per-sequence path."""
    b = W.FULL["prefix_cow"]("cuda")
    if b.cow_pairs.numel():
        ops.pa_copy_blocks(b.k_cache, b.v_cache, b.cow_pairs)
    ops.pa_write_kv(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping)
    shared, groups = decode(b, True, path=ops.PA_PATH_AUTO)
    private, _ = decode(b, False, path=ops.PA_PATH_AUTO)
    assert groups > 0
    assert float((shared - private).abs().max()) <= 1e-4
    rng = np.random.default_rng(5)
    for seq in rng.choice(b.q.shape[0], 6, replace=False):
        for h in rng.choice(b.q.shape[1], 3, replace=False):
            ref = sampled_reference(b, int(seq), int(h))
            got = shared[int(seq), int(h)].cpu().numpy().astype(np.float64)
            assert np.max(np.abs(got - ref)) <= 2e-3


def test_empty_and_invalid_sequences_inside_a_run():
    """An empty sequence and one whose length exceeds max_context_len break
    the run they sit in: the others still match the oracle, the empty row is
    zero, the invalid one is zero and flagged, and groups still form."""
    b = shared_batch([(1024, [10, 20, 30, 40, 50, 60])])
    lens = b.context_lens.clone()
    lens[2] = 0
    b.context_lens = lens
    B, Hq, D = b.q.shape
    bc = b.to("cpu")
    ref = ORACLE.decode(f64(bc.q), pool_f64(bc.k_cache), pool_f64(bc.v_cache),
                        bc.block_tables.numpy(), bc.context_lens.numpy(),
                        float(np.float32(bc.scale)))
    out, groups = decode(b, True)
    assert groups > 0
    assert max_abs_err(out, ref) <= TOL[b.dtype]
    assert torch.count_nonzero(out[2]) == 0
    # now sequence 4 claims more tokens than max_context_len allows
    max_ctx = int(lens.max().item())
    lens[4] = max_ctx + 1
    ws = ops.decode_workspace(B, Hq, D, max_ctx + 16, b.block_size)
    out2 = torch.full((B, Hq, D), float("nan"), device="cuda")
    ops.pa_decode(out2, b.q, b.k_cache, b.v_cache, b.block_tables, lens, max_ctx, b.scale, ws,
                  path=ops.PA_PATH_SIMT, share_prefixes=True)
    torch.cuda.synchronize()
    assert ops.pa_decode_status(ws) == ops.PA_ERR_INVALID_ARG
    assert torch.count_nonzero(out2[4]) == 0
    keep = [i for i in range(B) if i not in (2, 4)]
    assert max_abs_err(out2[keep], ref[keep]) <= TOL[b.dtype]


def test_largest_batch_with_groups():
    """1024 sequences (the most pa_decode groups), runs of 5 behind 256- to
    512-token prefixes: sampled rows against the oracle, all rows against the
    per-sequence path."""
    rng = np.random.default_rng(9)
    runs = [(int(rng.choice([256, 384, 512])), [int(x) for x in rng.integers(1, 200, 5)])
            for _ in range(204)] + [(256, [3, 30, 90, 199])]
    b = shared_batch(runs, dtype=torch.bfloat16, Hq=8, Hkv=8)
    assert b.q.shape[0] == 1024
    shared, groups = decode(b, True, path=ops.PA_PATH_AUTO)
    private, _ = decode(b, False, path=ops.PA_PATH_AUTO)
    assert groups > 0
    assert float((shared - private).abs().max()) <= 1e-4
    for seq in rng.choice(1024, 8, replace=False):
        h = int(rng.integers(0, 8))
        ref = sampled_reference(b, int(seq), h)
        got = shared[int(seq), h].cpu().numpy().astype(np.float64)
        assert np.max(np.abs(got - ref)) <= 2e-3


def test_no_alloc_entry_point_shares_too():
    """pa_decode_noalloc takes the option through its fixed scratch."""
    b = shared_batch([(1024, [5, 17, 300, 64, 1, 700])])
    B, Hq, D = b.q.shape
    bc = b.to("cpu")
    ref = ORACLE.decode(f64(bc.q), pool_f64(bc.k_cache), pool_f64(bc.v_cache),
                        bc.block_tables.numpy(), bc.context_lens.numpy(),
                        float(np.float32(bc.scale)))
    out = torch.full((B, Hq, D), float("nan"), device="cuda")
    ops.pa_decode_noalloc(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                          b.max_context_len, b.scale, path=ops.PA_PATH_SIMT, share_prefixes=True)
    torch.cuda.synchronize()
    assert ops.pa_decode_noalloc_status() == ops.PA_OK
    assert max_abs_err(out, ref) <= TOL[b.dtype]
