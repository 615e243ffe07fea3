"""CUDA path against the CPU oracle, through the C-ABI binding.

Bit-exact for the KV write and the block copy; max-abs error within 1e-5 (fp32
KV) or 2e-3 (fp16 / bf16 KV) of the fp64 oracle for decode. Small workloads
compare every output; full-size workloads compare sampled rows, in the launch
configuration the benchmark times.
"""

import numpy as np
import pytest
import torch

from oracle import ORACLE
from paged_kv_cache_339_b200 import build as pa_build
from paged_kv_cache_339_b200 import ops
from paged_kv_cache_339_b200 import workloads as W
from tests.gpu_helpers import (TOL, bits, f64, max_abs_err, oracle_step, pool_bits,
                               pool_f64, reference_rows, run_step, sampled_reference)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pa_build.build()
    ops.library()


def paths_for(batch):
    G = batch.num_q_heads // batch.num_kv_heads
    lib = ops.library()
    ps = [ops.PA_PATH_SIMT]
    if batch.dtype != torch.float32 and batch.head_dim == 128 and 4 <= G <= 16:
        ps.append(ops.PA_PATH_TCGEN05)
    return ps


def _path_supported(batch, path):
    """TCGEN05 is refused (UNSUPPORTED) when the library has no such kernel."""
    if path != ops.PA_PATH_TCGEN05:
        return True
    try:
        run_step(batch.to("cuda"), path=path, write=False)
        return True
    except ops.PagedAttnError as e:
        if e.status == ops.PA_ERR_UNSUPPORTED:
            return False
        raise


SMALL_NAMES = list(W.SMALL)


# ---------------------------------------------------------------------------
# KV write and block copy: bit-exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", SMALL_NAMES)
def test_write_and_copy_bit_exact(name):
    b = W.SMALL[name]("cuda")
    kb, vb = pool_bits(b.k_cache), pool_bits(b.v_cache)
    if b.cow_pairs.numel():
        ops.pa_copy_blocks(b.k_cache, b.v_cache, b.cow_pairs)
        kb, vb = ORACLE.copy_blocks(kb, vb, b.cow_pairs.cpu().numpy())
        torch.cuda.synchronize()
        assert np.array_equal(pool_bits(b.k_cache), kb) and np.array_equal(pool_bits(b.v_cache), vb)
    ops.pa_write_kv(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping)
    torch.cuda.synchronize()
    kb, vb = ORACLE.write_kv(kb, vb, bits(b.key), bits(b.value), b.slot_mapping.cpu().numpy())
    assert np.array_equal(pool_bits(b.k_cache), kb)
    assert np.array_equal(pool_bits(b.v_cache), vb)


def test_write_many_tokens_skips_padding_and_out_of_pool():
    """Prefill-sized write: 3000 tokens, padding slots (-1) and slots past the
    pool are skipped; everything else lands bit-exactly."""
    g = torch.Generator().manual_seed(7)
    NB, H, BS, D = 300, 4, 16, 128
    kc = torch.randn(NB, H, BS, D, generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn(NB, H, BS, D, generator=g).to(torch.bfloat16).cuda()
    T = 3000
    slots = torch.randperm(NB * BS, generator=g)[:T].to(torch.int64)
    slots[::7] = -1
    slots[5] = NB * BS + 3                      # outside the pool: skipped
    key = torch.randn(T, H, D, generator=g).to(torch.bfloat16)
    val = torch.randn(T, H, D, generator=g).to(torch.bfloat16)
    kb, vb = pool_bits(kc), pool_bits(vc)
    ops.pa_write_kv(kc, vc, key.cuda(), val.cuda(), slots.cuda())
    torch.cuda.synchronize()
    ok = slots.clone()
    ok[5] = -1
    kb, vb = ORACLE.write_kv(kb, vb, bits(key), bits(val), ok.numpy())
    assert np.array_equal(pool_bits(kc), kb) and np.array_equal(pool_bits(vc), vb)


# ---------------------------------------------------------------------------
# Decode against the oracle, small workloads, every output
# ---------------------------------------------------------------------------

CASES = [(n, s) for n in SMALL_NAMES for s in (0, "small")]


@pytest.mark.parametrize("name,split", CASES, ids=[f"{n}-split{s}" for n, s in CASES])
def test_step_matches_oracle(name, split):
    proto = W.SMALL[name]("cpu")
    for path in paths_for(proto):
        b = W.SMALL[name]("cuda")
        if not _path_supported(b, path):
            continue
        bc = b.to("cpu")
        st = 0 if split == 0 else (16 if name == "tiny" else 2 * b.block_size * 4)
        out = run_step(b, split_tokens=st, path=path)
        ref = oracle_step(bc)
        err = max_abs_err(out, ref)
        assert err <= TOL[b.dtype], (name, path, st, err)


# Split sequences of many pieces: counts around the merge's batches of 8
# loads, up to 200 pieces, and a batch of sequences with different counts.
PIECES = [7, 8, 9, 16, 17, 64, 65, 200, "mixed"]


@pytest.mark.parametrize("pieces", PIECES)
def test_many_pieces_merge(pieces):
    if pieces == "mixed":
        gen = np.random.default_rng(3)
        lens = [int(x) for x in gen.integers(900, 9000, 5)] + [128 * 8, 128 * 8 + 1]
    else:
        lens = [128 * pieces - 5, 128 * pieces, 128 * (pieces - 1) + 1]
    proto = _custom_batch(lens, device="cpu")
    for path in paths_for(proto):
        b = _custom_batch(lens)
        bc = b.to("cpu")
        out = run_step(b, split_tokens=128, path=path)
        err = max_abs_err(out, oracle_step(bc))
        assert err <= TOL[b.dtype], (pieces, path, err)


def _custom_batch(lens, dtype=torch.bfloat16, Hq=8, Hkv=2, D=128, BS=16, seed=11,
                  device="cuda"):
    gen = torch.Generator().manual_seed(seed)
    need = sum((L + BS - 1) // BS for L in lens)
    NB = need + 5
    tables = W._place(lens, BS, NB, gen)
    return W._assemble("custom", dtype, BS, Hq, Hkv, D, lens, tables, NB, gen, seed, device)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (16, 2)])
def test_edge_lengths(dtype, hq, hkv):
    """Empty contexts give zero rows, one token gives exactly its value, and
    ragged tails of every size around block and chunk edges match."""
    lens = [0, 1, 2, 15, 16, 17, 63, 64, 65, 127, 128, 129, 0, 300]
    b = _custom_batch(lens, dtype=dtype, Hq=hq, Hkv=hkv)
    proto = b
    for path in paths_for(proto):
        b = _custom_batch(lens, dtype=dtype, Hq=hq, Hkv=hkv)
        if not _path_supported(b, path):
            continue
        bc = b.to("cpu")
        out = run_step(b, path=path, split_tokens=32)
        ref = oracle_step(bc)
        assert max_abs_err(out, ref) <= TOL[dtype]
        o = out.cpu()
        assert torch.count_nonzero(o[0]) == 0 and torch.count_nonzero(o[12]) == 0
        G = hq // hkv
        for h in range(hq):          # L = 1: softmax weight exactly 1
            assert torch.equal(o[1, h], bc.value[1, h // G].float())


def test_nan_in_unread_slots_does_not_leak():
    """Slots past each sequence's end and blocks no table uses are NaN; the
    result must equal the oracle's and be finite."""
    lens = [5, 33, 100, 250]
    for path in (ops.PA_PATH_SIMT, ops.PA_PATH_TCGEN05):
        b = _custom_batch(lens, Hq=8, Hkv=2)
        if not _path_supported(b, path):
            continue
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
        out = run_step(b, path=path, split_tokens=64)
        assert max_abs_err(out, oracle_step(bc)) <= 2e-3


def test_permutation_invariance_bit_identical():
    """The same logical sequences at other physical places give bit-identical
    output ("blocks can sit anywhere, in any order")."""
    b = W.SMALL["gqa"]("cuda")
    outs = {}
    for path in paths_for(b):
        if not _path_supported(b, path):
            continue
        b1 = W.SMALL["gqa"]("cuda")
        o1 = run_step(b1, path=path, write=False)
        perm = torch.randperm(b1.num_blocks, generator=torch.Generator().manual_seed(3)).cuda()
        b2 = W.SMALL["gqa"]("cuda")
        kc, vc = torch.empty_like(b2.k_cache), torch.empty_like(b2.v_cache)
        kc[perm] = b2.k_cache
        vc[perm] = b2.v_cache
        b2.k_cache, b2.v_cache = kc, vc
        b2.block_tables = perm[b2.block_tables.long()].to(torch.int32)
        o2 = run_step(b2, path=path, write=False)
        assert torch.equal(o1, o2)
        outs[path] = o1


def test_shared_prefix_equals_private_copies_bit_identical():
    """After the copy-on-write step, sequences that read the shared prefix (and
    the pair-shared suffix) through their tables give exactly what they give
    when every sequence reads its own private replica of every block
    ("Sharing comes almost for free": many tables, one physical copy)."""
    for path in (ops.PA_PATH_SIMT, ops.PA_PATH_TCGEN05):
        b = W.SMALL["prefix_cow"]("cuda")
        if b.num_q_heads // b.num_kv_heads < 4 and path == ops.PA_PATH_TCGEN05:
            continue
        shared = run_step(b, path=path)
        # private copies of every shared block for every sequence
        p = W.SMALL["prefix_cow"]("cuda")
        if p.cow_pairs.numel():
            ops.pa_copy_blocks(p.k_cache, p.v_cache, p.cow_pairs)
        ops.pa_write_kv(p.k_cache, p.v_cache, p.key, p.value, p.slot_mapping)
        bt = p.block_tables.clone()
        B, nbmax = bt.shape
        NB = p.num_blocks
        kc = torch.cat([p.k_cache] + [p.k_cache] * B)
        vc = torch.cat([p.v_cache] + [p.v_cache] * B)
        for i in range(B):
            bt[i] = bt[i] + (i + 1) * NB       # sequence i reads its own replica
        p.k_cache, p.v_cache, p.block_tables = kc, vc, bt
        private = run_step(p, path=path, write=False)
        assert torch.equal(shared, private)


def test_cow_step_leaves_the_other_sibling_bit_identical():
    """Copy-on-write ("Sharing comes almost for free"): one sibling of each
    pair copies the shared partial block and writes into its copy; the
    other sibling, which does not step, decodes bit-identically before and
    after, and the copied block equals its source byte for byte."""
    b = W.SMALL["prefix_cow"]("cuda")
    coins = b.meta["coins"]
    diverge = [2 * j + c for j, c in enumerate(coins)]
    keep = [2 * j + 1 - c for j, c in enumerate(coins)]
    lens = (b.context_lens - 1).contiguous()     # the new tokens are not in the context
    B, Hq, D = b.q.shape
    max_ctx = int(lens.max().item())

    def decode():
        ws = ops.decode_workspace(B, Hq, D, max_ctx, b.block_size)
        out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
        ops.pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, lens, max_ctx, b.scale, ws)
        torch.cuda.synchronize()
        assert ops.pa_decode_status(ws) == ops.PA_OK
        return out

    before = decode()
    ops.pa_copy_blocks(b.k_cache, b.v_cache, b.cow_pairs)
    torch.cuda.synchronize()
    for src, dst in b.cow_pairs.cpu().tolist():
        assert np.array_equal(bits(b.k_cache[dst]), bits(b.k_cache[src]))
        assert np.array_equal(bits(b.v_cache[dst]), bits(b.v_cache[src]))
    slots = b.slot_mapping.clone()
    slots[keep] = -1                              # only the diverging siblings step
    ops.pa_write_kv(b.k_cache, b.v_cache, b.key, b.value, slots)
    after = decode()
    assert torch.equal(after[keep], before[keep])
    assert not torch.equal(after[diverge], before[diverge])   # their last block changed


def test_deterministic_and_split_consistent():
    b = W.SMALL["long"]("cuda")
    o1 = run_step(b, write=True)
    o2 = run_step(b, write=False)
    assert torch.equal(o1, o2)
    bc = b.to("cpu")
    ref = ORACLE.decode(f64(bc.q), pool_f64(bc.k_cache), pool_f64(bc.v_cache),
                        bc.block_tables.numpy(), bc.context_lens.numpy(),
                        float(np.float32(bc.scale)))
    for st in (32, 256, 4096):
        assert max_abs_err(run_step(b, split_tokens=st, write=False), ref) <= 2e-3


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_block_sizes(bs):
    b = W.long_context("cuda", num_seqs=2, num_q_heads=16, num_kv_heads=2, min_len=2000,
                       max_len=5000, block_size=bs)
    for path in paths_for(b):
        bb = W.long_context("cuda", num_seqs=2, num_q_heads=16, num_kv_heads=2, min_len=2000,
                            max_len=5000, block_size=bs)
        if not _path_supported(bb, path):
            continue
        bc = bb.to("cpu")
        assert max_abs_err(run_step(bb, path=path), oracle_step(bc)) <= 2e-3


def test_bad_table_entry_and_length_are_flagged_not_faulted():
    """A table entry outside the pool is read as block 0 and a length beyond
    max_context_len gives a zero row; both raise PA_ERR_INVALID_ARG in the
    status word, with every access inside the buffers."""
    b = _custom_batch([40, 40, 40], Hq=4, Hkv=4)
    b.block_tables[0, 1] = b.num_blocks + 1000
    ws = ops.decode_workspace(3, 4, 128, 64, 16)
    out = torch.empty(3, 4, 128, device="cuda")
    ops.pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, 48, b.scale, ws)
    torch.cuda.synchronize()
    assert ops.pa_decode_status(ws) == ops.PA_ERR_INVALID_ARG
    b2 = _custom_batch([40, 80, 40], Hq=4, Hkv=4)
    ops.pa_decode(out, b2.q, b2.k_cache, b2.v_cache, b2.block_tables, b2.context_lens, 64,
                  b2.scale, ws)
    torch.cuda.synchronize()
    assert ops.pa_decode_status(ws) == ops.PA_ERR_INVALID_ARG
    assert torch.count_nonzero(out[1]) == 0
    # a clean call clears the word again
    b3 = _custom_batch([40, 50, 60], Hq=4, Hkv=4)
    ops.pa_decode(out, b3.q, b3.k_cache, b3.v_cache, b3.block_tables, b3.context_lens, 64,
                  b3.scale, ws)
    torch.cuda.synchronize()
    assert ops.pa_decode_status(ws) == ops.PA_OK


# ---------------------------------------------------------------------------
# Full-size workloads: sampled rows, benchmark launch configuration
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["mha", "gqa", "prefix_cow", "long"])
def test_full_size_sampled(name):
    b = W.FULL[name]("cuda")
    out = run_step(b)            # the step the benchmark times (auto split, auto path)
    lens = b.context_lens.cpu()
    B, Hq = b.num_seqs, b.num_q_heads
    seqs = sorted({int(lens.argmax()), int(lens.argmin()), 0, B - 1, B // 2})
    heads = sorted({0, Hq - 1, Hq // 2 + 1})
    worst = 0.0
    for i in seqs:
        for h in heads:
            ref = sampled_reference(b, i, h)
            got = out[i, h].cpu().numpy().astype(np.float64)
            worst = max(worst, float(np.max(np.abs(got - ref))))
    if name == "long":
        # every query head of the longest and the shortest sequence: the rows
        # that go through the tail cut of the plan and the merge of the most
        # pieces
        for i in sorted({int(lens.argmax()), int(lens.argmin())}):
            for h, ref in reference_rows(b, i, list(range(Hq))).items():
                got = out[i, h].cpu().numpy().astype(np.float64)
                worst = max(worst, float(np.max(np.abs(got - ref))))
    assert worst <= TOL[b.dtype], (name, worst)
    # every row is finite, and rows of one KV-head group share the same keys
    assert torch.isfinite(out).all()
    # the new token really is in the cache at its slot
    BS = b.block_size
    for i in seqs:
        s = int(b.slot_mapping[i])
        kblk = pool_bits(b.k_cache[s // BS:s // BS + 1])[0]
        vblk = pool_bits(b.v_cache[s // BS:s // BS + 1])[0]
        assert np.array_equal(kblk[:, s % BS], bits(b.key[i]))
        assert np.array_equal(vblk[:, s % BS], bits(b.value[i]))


@pytest.mark.parametrize("kind", ["tc_bf16_g4", "simt_f32_g1"])
def test_maximum_sequence_count(kind):
    """56,320 sequences, the most one call takes, with short log-normal /
    uniform contexts: every row finite, sampled rows (first, last, longest,
    shortest and a spread between) within tolerance of the oracle."""
    B = 56320
    if kind == "tc_bf16_g4":
        b = W.gqa("cuda", seed=77, num_seqs=B, num_q_heads=4, num_kv_heads=1, mean_len=24,
                  min_len=1, max_len=200)
    else:
        b = W.mha("cuda", seed=78, num_seqs=B, num_heads=1, head_dim=64, min_len=1,
                  max_len=64, num_blocks=1, dtype=torch.float32)
    out = run_step(b)
    assert torch.isfinite(out).all()
    lens = b.context_lens.cpu()
    rng = np.random.default_rng(5)
    seqs = sorted({0, B - 1, int(lens.argmax()), int(lens.argmin())}
                  | {int(x) for x in rng.integers(0, B, 24)})
    worst = 0.0
    for i in seqs:
        for h in sorted({0, b.num_q_heads - 1}):
            ref = sampled_reference(b, i, h)
            got = out[i, h].cpu().numpy().astype(np.float64)
            worst = max(worst, float(np.max(np.abs(got - ref))))
    assert worst <= TOL[b.dtype], (kind, worst)

