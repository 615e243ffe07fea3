"""Pins for the CPU oracle: each check takes an oracle instance and raises
AssertionError when the instance disagrees with something the pages or the
mathematics fix independently of the oracle's own code (closed forms, a golden
fixture, invariants the pages state, brute-force special cases).

The checks are plain functions so the planted-mistake test can run them
against deliberately broken oracles.
"""

from __future__ import annotations

import json
import math
from pathlib import Path

import numpy as np

GOLDEN = Path(__file__).parent / "golden"


def _rng(seed):
    return np.random.default_rng(seed)


def _pool_from_contiguous(X, block_size, placement):
    """Lay a contiguous [L, H, D] array into a pool [NB, H, BS, D]: logical
    block b goes to physical block placement[b]. Unused pool slots get NaN so
    that reading them anywhere shows up."""
    L, H, D = X.shape
    nb = (L + block_size - 1) // block_size
    NB = max(placement) + 1 if len(placement) else 1
    pool = np.full((NB, H, block_size, D), np.nan)
    for b in range(nb):
        rows = X[b * block_size:(b + 1) * block_size]
        pool[placement[b], :, :rows.shape[0], :] = rows.transpose(1, 0, 2)
    return pool


# ---------------------------------------------------------------------------
# Attention closed forms
# ---------------------------------------------------------------------------

def check_single_token(orc):
    """One token: softmax of a single score is 1, so o = v_0 exactly."""
    r = _rng(1)
    for scale in (0.125, 3.0):
        q, K, V = r.normal(size=8), r.normal(size=(1, 8)), r.normal(size=(1, 8))
        o = orc.attend(q, K, V, scale)
        assert np.array_equal(o, V[0]), (o, V[0])


def check_zero_query_mean(orc):
    """q = 0: all scores equal, so o is the plain mean of the values."""
    r = _rng(2)
    K, V = r.normal(size=(13, 6)), r.normal(size=(13, 6))
    o = orc.attend(np.zeros(6), K, V, 0.7)
    assert np.allclose(o, V.mean(axis=0), rtol=0, atol=1e-14)


def check_equal_keys_mean(orc):
    """All keys identical: all scores equal, o = mean of the values."""
    r = _rng(3)
    k = r.normal(size=5)
    K = np.tile(k, (9, 1))
    V = r.normal(size=(9, 5))
    o = orc.attend(r.normal(size=5), K, V, 1.3)
    assert np.allclose(o, V.mean(axis=0), rtol=0, atol=1e-14)


def check_two_token_logistic(orc):
    """Two tokens: softmax reduces to the logistic function of the score
    difference, o = sigma(d) v0 + sigma(-d) v1 with d = scale q.(k0 - k1)."""
    q = np.array([0.5, -1.0, 2.0])
    k0 = np.array([1.0, 0.0, 0.5])
    k1 = np.array([-0.5, 1.0, 0.25])
    V = np.array([[2.0, -1.0, 0.0], [-3.0, 4.0, 1.0]])
    scale = 0.8
    d = scale * (0.5 * 1.5 + (-1.0) * (-1.0) + 2.0 * 0.25)   # scale * q.(k0-k1)
    w0 = 1.0 / (1.0 + math.exp(-d))
    expect = w0 * V[0] + (1.0 - w0) * V[1]
    o = orc.attend(q, np.stack([k0, k1]), V, scale)
    assert np.allclose(o, expect, rtol=0, atol=1e-14), (o, expect)


def check_golden_rational(orc):
    """Golden fixture: weights 1:2:3:4 by construction, through a shuffled
    two-block table with junk in the unused blocks."""
    g = json.loads((GOLDEN / "decode_rational_weights.json").read_text())
    BS, NB, D = g["block_size"], g["num_blocks"], g["head_dim"]
    L = g["context_len"]
    K = np.stack([np.log(np.array(g["weights"], dtype=np.float64)),
                  np.array(g["key_second_component"])], axis=1)
    V = np.array(g["values"])
    kc = np.full((NB, 1, BS, D), 1.0e6)
    vc = np.full((NB, 1, BS, D), -1.0e6)
    for j in range(L):
        b = g["block_table"][j // BS]
        kc[b, 0, j % BS] = K[j]
        vc[b, 0, j % BS] = V[j]
    q = np.array(g["q"]).reshape(1, 1, D)
    out = orc.decode(q, kc, vc, np.array([g["block_table"]]), np.array([L]),
                     g["scale"])
    expect = np.array(g["expected_numerator"]) / g["expected_denominator"]
    assert np.allclose(out[0, 0], expect, rtol=0, atol=1e-14), (out, expect)


def check_argmax_limit(orc):
    """Very large scale: the softmax becomes one-hot on the largest score, so
    o = v of the best-matching key (pins the sign of the exponent)."""
    r = _rng(4)
    K = r.normal(size=(11, 4))
    V = r.normal(size=(11, 4))
    q = r.normal(size=4)
    best = int(np.argmax(K @ q))
    o = orc.attend(q, K, V, 1.0e6)
    assert np.allclose(o, V[best], rtol=0, atol=1e-12), (o, V[best])


def check_shift_invariance(orc):
    """Adding a vector u to every key adds q.u to every score; softmax is
    invariant to a common shift, including a shift (1000) that would overflow
    exp() if the maximum were not taken out first."""
    r = _rng(5)
    K = r.normal(size=(7, 4))
    V = r.normal(size=(7, 4))
    q = np.array([1.0, 0.0, 0.0, 0.0])
    u = np.array([1000.0, 0.0, 0.0, 0.0])
    o1 = orc.attend(q, K, V, 1.0)
    o2 = orc.attend(q, K + u, V, 1.0)
    assert np.all(np.isfinite(o2))
    assert np.allclose(o1, o2, rtol=0, atol=1e-12)


def check_linear_in_values(orc):
    """For fixed q, K the output is linear in V."""
    r = _rng(6)
    q, K = r.normal(size=6), r.normal(size=(10, 6))
    V1, V2 = r.normal(size=(10, 6)), r.normal(size=(10, 6))
    o = orc.attend(q, K, 2.0 * V1 - 3.0 * V2, 0.4)
    o1, o2 = orc.attend(q, K, V1, 0.4), orc.attend(q, K, V2, 0.4)
    assert np.allclose(o, 2.0 * o1 - 3.0 * o2, rtol=0, atol=1e-13)


def check_convex_combination(orc):
    """Each output component lies within the range of that value column, and
    keys and values play different roles (a transposed operand fails)."""
    r = _rng(7)
    q, K, V = r.normal(size=3), r.normal(size=(20, 3)), r.normal(size=(20, 3))
    V[:, 0] += 100.0          # keys stay O(1); values of column 0 are ~100
    o = orc.attend(q, K, V, 0.9)
    assert np.all(o <= V.max(axis=0) + 1e-12)
    assert np.all(o >= V.min(axis=0) - 1e-12)


# ---------------------------------------------------------------------------
# Paging: gather, placement, GQA mapping, sharing, copy-on-write
# ---------------------------------------------------------------------------

def check_identity_table_is_contiguous(orc):
    """Identity table over a pool laid out from a contiguous array gathers the
    array back exactly, ragged last block included (glossary 'What is Paged
    Attention?': the sequence is read in logical order, as though stored back
    to back)."""
    r = _rng(8)
    for L, BS in ((1, 4), (13, 4), (16, 16), (33, 16), (70, 8)):
        X = r.normal(size=(L, 3, 5))
        nb = (L + BS - 1) // BS
        pool = _pool_from_contiguous(X, BS, list(range(nb)))
        got = orc.gather(pool, np.arange(nb), L)
        assert np.array_equal(got, X), (L, BS)


def check_permutation_invariance(orc):
    """Blocks can sit anywhere in any order (P1, 'The fix borrowed from
    operating systems'): relocating the blocks and rewriting the table leaves
    the decode output bit-identical."""
    r = _rng(9)
    BS, L, H, D = 4, 23, 2, 6
    nb = (L + BS - 1) // BS
    Kx, Vx = r.normal(size=(L, H, D)), r.normal(size=(L, H, D))
    q = r.normal(size=(1, H, D))
    outs = []
    for place in (list(range(nb)), list(r.permutation(nb + 5)[:nb])):
        kc = _pool_from_contiguous(Kx, BS, place)
        vc = _pool_from_contiguous(Vx, BS, place)
        outs.append(orc.decode(q, kc, vc, np.array([place]), np.array([L]), 0.5))
    assert np.array_equal(outs[0], outs[1])
    # and the paged result is plain attention on the contiguous arrays
    for h in range(H):
        direct = orc.attend(q[0, h], Kx[:, h], Vx[:, h], 0.5)
        assert np.array_equal(outs[0][0, h], direct)


def check_gqa_is_repeated_mha(orc):
    """Grouped-query attention with G query heads per KV head equals MHA whose
    KV heads are each repeated G times (consecutive query heads share a KV
    head; grouped-query attention is named in P1, 'What it does not fix')."""
    r = _rng(10)
    B, Hq, Hkv, D, BS, NB = 2, 6, 2, 4, 4, 10
    G = Hq // Hkv
    kc, vc = r.normal(size=(NB, Hkv, BS, D)), r.normal(size=(NB, Hkv, BS, D))
    q = r.normal(size=(B, Hq, D))
    bt = np.array([[3, 7, 1], [0, 9, 2]])
    lens = np.array([10, 12])
    o_gqa = orc.decode(q, kc, vc, bt, lens, 0.3)
    o_mha = orc.decode(q, np.repeat(kc, G, axis=1), np.repeat(vc, G, axis=1),
                       bt, lens, 0.3)
    assert np.array_equal(o_gqa, o_mha)


def check_context_len_bounds(orc):
    """Only the first context_len tokens count: slots past the end of the last
    block (and every block not in the table) hold NaN and must not leak in.
    An empty context gives a zero row."""
    r = _rng(11)
    BS, D = 8, 4
    kc = np.full((6, 1, BS, D), np.nan)
    vc = np.full((6, 1, BS, D), np.nan)
    L = 11                                   # block 4 full, block 2 has 3 rows
    kc[4, 0], vc[4, 0] = r.normal(size=(BS, D)), r.normal(size=(BS, D))
    kc[2, 0, :3], vc[2, 0, :3] = r.normal(size=(3, D)), r.normal(size=(3, D))
    q = r.normal(size=(2, 1, D))
    out = orc.decode(q, kc, vc, np.array([[4, 2], [4, 2]]), np.array([L, 0]), 0.5)
    assert np.all(np.isfinite(out[0]))
    assert np.array_equal(out[1], np.zeros((1, D)))
    K = np.concatenate([kc[4, 0], kc[2, 0, :3]])
    V = np.concatenate([vc[4, 0], vc[2, 0, :3]])
    assert np.allclose(out[0, 0], orc.attend(q[0, 0], K, V, 0.5), rtol=0, atol=0)


def check_prefix_sharing(orc):
    """Sequences whose tables point at one physical copy of a common prefix
    (P1, 'Sharing comes almost for free') produce exactly what they produce
    with private duplicates of that prefix."""
    r = _rng(12)
    BS, H, D = 4, 2, 3
    NB = 20
    kc, vc = r.normal(size=(NB, H, BS, D)), r.normal(size=(NB, H, BS, D))
    prefix = [5, 11, 2]
    shared_bt = np.array([prefix + [7, 0], prefix + [9, 0]])
    # private duplicates of the prefix for the second sequence
    kc2, vc2 = kc.copy(), vc.copy()
    for src, dst in zip(prefix, [14, 15, 16]):
        kc2[dst], vc2[dst] = kc[src], vc[src]
    priv_bt = np.array([prefix + [7, 0], [14, 15, 16, 9, 0]])
    lens = np.array([15, 14])
    q = r.normal(size=(2, H, D))
    a = orc.decode(q, kc, vc, shared_bt, lens, 0.6)
    b = orc.decode(q, kc2, vc2, priv_bt, lens, 0.6)
    assert np.array_equal(a, b)


def check_copy_on_write(orc):
    """Copy-on-write (P1, 'Sharing comes almost for free'): two siblings share
    a partly filled last block; sibling A diverges, gets a private copy, and
    writes its token there; B then writes in place. B's output equals what B
    gets with private blocks from the start, the copy equals its source except
    for A's new slot, and no other block changes."""
    r = _rng(13)
    BS, H, D, NB = 4, 2, 3, 12
    kc, vc = r.normal(size=(NB, H, BS, D)), r.normal(size=(NB, H, BS, D))
    shared = [3, 8]                 # 6 tokens: block 8 holds 2 rows
    pos = 6
    src, dst = 8, 10
    kA, vA = r.normal(size=(1, H, D)), r.normal(size=(1, H, D))
    kB, vB = r.normal(size=(1, H, D)), r.normal(size=(1, H, D))
    k1, v1 = orc.copy_blocks(kc, vc, np.array([[src, dst]]))
    assert np.array_equal(k1[dst], kc[src]) and np.array_equal(v1[dst], vc[src])
    bt_A, bt_B = [3, dst], [3, src]
    slotA = bt_A[pos // BS] * BS + pos % BS
    slotB = bt_B[pos // BS] * BS + pos % BS
    k2, v2 = orc.write_kv(k1, v1, np.concatenate([kA, kB]),
                          np.concatenate([vA, vB]), np.array([slotA, slotB]))
    changed = [b for b in range(NB) if not np.array_equal(k2[b], kc[b])]
    assert changed == [src, dst], changed
    q = r.normal(size=(2, H, D))
    out = orc.decode(q, k2, v2, np.array([bt_A, bt_B]), np.array([7, 7]), 0.5)
    # B alone, never shared: its own private blocks from the start
    kp, vp = kc.copy(), vc.copy()
    kp[11], vp[11] = kc[src], vc[src]
    kp[11, :, pos % BS], vp[11, :, pos % BS] = kB[0], vB[0]
    ob = orc.decode(q[1:], kp, vp, np.array([[3, 11]]), np.array([7]), 0.5)
    assert np.array_equal(out[1:], ob)
    # A sees its own token at position 6, B's token is not visible to A
    KA = orc.gather(k2, np.array(bt_A), 7)
    assert np.array_equal(KA[6], kA[0]) and not np.array_equal(KA[6], kB[0])


# ---------------------------------------------------------------------------
# Token write and block copy
# ---------------------------------------------------------------------------

def check_write_layout(orc):
    """Slot s addresses block s // BS, offset s % BS of the
    [num_blocks, num_kv_heads, block_size, head_dim] pools; slot -1 writes
    nothing; nothing else changes."""
    BS, H, D, NB = 4, 2, 3, 5
    kc = np.zeros((NB, H, BS, D), dtype=np.int32)
    vc = np.zeros((NB, H, BS, D), dtype=np.int32)
    key = np.arange(3 * H * D, dtype=np.int32).reshape(3, H, D) + 1
    val = -key
    k2, v2 = orc.write_kv(kc, vc, key, val, np.array([9, 19, -1]))
    assert np.array_equal(k2[2, :, 1, :], key[0]) and np.array_equal(v2[2, :, 1, :], val[0])
    assert np.array_equal(k2[4, :, 3, :], key[1]) and np.array_equal(v2[4, :, 3, :], val[1])
    mask = np.ones(k2.shape, dtype=bool)
    mask[2, :, 1, :] = False
    mask[4, :, 3, :] = False
    assert not k2[mask].any() and not v2[mask].any()
    assert not kc.any()                       # inputs untouched


def check_write_then_gather(orc):
    """A token written at the slot of logical position p of a sequence is what
    the gather returns at position p (incremental allocation, P1, 'The fix
    borrowed from operating systems')."""
    r = _rng(14)
    BS, H, D, NB = 8, 2, 4, 16
    kc, vc = r.normal(size=(NB, H, BS, D)), r.normal(size=(NB, H, BS, D))
    table = np.array([6, 1, 12])
    for p in (0, 7, 8, 20, 23):
        slot = table[p // BS] * BS + p % BS
        k_new, v_new = r.normal(size=(1, H, D)), r.normal(size=(1, H, D))
        k2, v2 = orc.write_kv(kc, vc, k_new, v_new, np.array([slot]))
        assert np.array_equal(orc.gather(k2, table, p + 1)[p], k_new[0])
        assert np.array_equal(orc.gather(v2, table, p + 1)[p], v_new[0])
        assert np.array_equal(orc.gather(k2, table, p), orc.gather(kc, table, p))


def check_copy_blocks(orc):
    """Each dst block of both pools becomes a copy of its src block; src and
    every other block are unchanged."""
    r = _rng(15)
    NB, H, BS, D = 9, 2, 4, 3
    kc = r.integers(0, 1 << 16, size=(NB, H, BS, D), dtype=np.uint16)
    vc = r.integers(0, 1 << 16, size=(NB, H, BS, D), dtype=np.uint16)
    pairs = np.array([[1, 7], [4, 2], [1, 5]])
    k2, v2 = orc.copy_blocks(kc, vc, pairs)
    for s, d in pairs:
        assert np.array_equal(k2[d], kc[s]) and np.array_equal(v2[d], vc[s])
    for b in set(range(NB)) - {7, 2, 5}:
        assert np.array_equal(k2[b], kc[b]) and np.array_equal(v2[b], vc[b])


def check_swap_blocks(orc):
    """Swap out copies device blocks to host blocks, swap in copies them back;
    the other side and every untouched block are unchanged, pairs outside
    either pool are skipped, and a sequence evicted and brought back into
    other blocks (its table rewritten) reads the same context ("What it does
    not fix": preemption by swapping)."""
    r = _rng(18)
    NB, NH, H, BS, D = 6, 4, 2, 4, 3
    dk = r.integers(0, 1 << 16, size=(NB, H, BS, D), dtype=np.uint16)
    dv = r.integers(0, 1 << 16, size=(NB, H, BS, D), dtype=np.uint16)
    hk = r.integers(0, 1 << 16, size=(NH, H, BS, D), dtype=np.uint16)
    hv = r.integers(0, 1 << 16, size=(NH, H, BS, D), dtype=np.uint16)
    out_pairs = np.array([[1, 3], [4, 0], [9, 1], [2, 7], [-1, 2]])
    dk1, dv1, hk1, hv1 = orc.swap_blocks(dk, dv, hk, hv, out_pairs, 0)
    assert np.array_equal(dk1, dk) and np.array_equal(dv1, dv)
    assert np.array_equal(hk1[3], dk[1]) and np.array_equal(hv1[3], dv[1])
    assert np.array_equal(hk1[0], dk[4]) and np.array_equal(hv1[0], dv[4])
    for b in (1, 2):   # skipped pairs left the host blocks alone
        assert np.array_equal(hk1[b], hk[b]) and np.array_equal(hv1[b], hv[b])
    in_pairs = np.array([[3, 5], [0, 2], [5, 0], [1, 6]])
    dk2, dv2, hk2, hv2 = orc.swap_blocks(dk1, dv1, hk1, hv1, in_pairs, 1)
    assert np.array_equal(hk2, hk1) and np.array_equal(hv2, hv1)
    assert np.array_equal(dk2[5], dk[1]) and np.array_equal(dv2[5], dv[1])
    assert np.array_equal(dk2[2], dk[4]) and np.array_equal(dv2[2], dv[4])
    for b in (0, 1, 3, 4):
        assert np.array_equal(dk2[b], dk[b]) and np.array_equal(dv2[b], dv[b])
    # evict a 6-token sequence held in blocks [1, 4], bring it back into [5, 2]
    L = 6
    before = orc.gather(dk, np.array([1, 4]), L)
    after = orc.gather(dk2, np.array([5, 2]), L)
    assert np.array_equal(before, after)


# ---------------------------------------------------------------------------
# Split-context regrouping
# ---------------------------------------------------------------------------

def check_merge_partition(orc):
    """Merging softmax pieces over any partition of the tokens gives the
    unsplit result (exact algebra; small fp64 rounding only)."""
    r = _rng(16)
    L, D = 37, 5
    q, K, V = r.normal(size=D), r.normal(size=(L, D)) * 3, r.normal(size=(L, D))
    full = orc.attend(q, K, V, 0.7)
    for cuts in ([0, 37], [0, 1, 37], [0, 16, 32, 37], [0, 5, 6, 20, 36, 37]):
        parts = [orc.partial(q, K, V, 0.7, a, b) for a, b in zip(cuts, cuts[1:])]
        assert np.allclose(orc.merge(parts), full, rtol=0, atol=1e-13), cuts


def check_tile_layout(orc):
    """The stored order of a (block, head) tile: every element of the logical
    view sits at the offset the storage formula gives, the conversion is a
    bijection, and head_dim 64 is plain row-major."""
    r = _rng(17)
    for BS, D in ((8, 128), (16, 128), (32, 128), (16, 64), (32, 64)):
        NB, H = 3, 2
        phys = r.integers(0, 1 << 30, size=(NB, H, BS, D))
        log = orc.logical_pool(phys)
        flat = phys.reshape(NB, H, BS * D)
        for (b, h, t, d) in ((0, 0, 0, 0), (2, 1, BS - 1, D - 1), (1, 0, BS // 2, 63),
                             (1, 1, min(BS - 1, 17), D // 2), (0, 1, 7, 64 % D)):
            assert log[b, h, t, d] == flat[b, h, orc.tile_offset(t, d, BS, D)]
        assert np.array_equal(orc.physical_pool(log), phys)
        assert len(np.unique(log)) == len(np.unique(phys))
    row_major = r.integers(0, 100, size=(2, 2, 16, 64))
    assert np.array_equal(orc.logical_pool(row_major), row_major)
    # BS 16, D 128: column 64 of token 0 is the first element of the second half
    assert orc.tile_offset(0, 64, 16, 128) == 16 * 64
    assert orc.tile_offset(16, 0, 32, 128) == 2 * 16 * 64


ALL_CHECKS = [
    check_single_token, check_zero_query_mean, check_equal_keys_mean,
    check_two_token_logistic, check_golden_rational, check_argmax_limit,
    check_shift_invariance, check_linear_in_values, check_convex_combination,
    check_identity_table_is_contiguous, check_permutation_invariance,
    check_gqa_is_repeated_mha, check_context_len_bounds, check_prefix_sharing,
    check_copy_on_write, check_write_layout, check_write_then_gather,
    check_copy_blocks, check_swap_blocks, check_merge_partition, check_tile_layout,
]
