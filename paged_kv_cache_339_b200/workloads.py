"""Seeded synthetic decode batches.

This module only draws random numbers and lays out block tables; it holds none
of the arithmetic of the hot path (no attention, no scatter, no copy). Both the
CUDA path and the CPU oracle consume what it returns.

Every batch is one decode step over a paged KV cache: a pool of fixed-size
physical blocks (``[num_blocks, num_kv_heads, block_size, head_dim]`` for K and
for V), one block table per sequence listing its blocks in logical order, one
new token per sequence to be written into its slot, and the query of that new
token. ``context_lens`` counts the new token, so position ``L - 1`` of every
sequence is written by the step and positions ``0 .. L - 2`` already hold K/V
(here: the random pool contents).

Recipe (fixed draw order, one ``torch.Generator`` per stream):
  * seed = 1000 + workload index (1..5); lengths, pool placement, coin flips,
    q, new K and new V are drawn on the CPU generator in that order;
  * the pool contents are drawn from a second generator (seed + 1) on the
    target device, as fp32 N(0, 1) rounded to the workload dtype;
  * physical blocks are handed out in the order of a seeded permutation of the
    whole pool, so sequences sit at scattered, shuffled places.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass
class DecodeBatch:
    name: str
    dtype: torch.dtype
    block_size: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    scale: float
    k_cache: torch.Tensor        # [NB, Hkv, BS, D]
    v_cache: torch.Tensor        # [NB, Hkv, BS, D]
    block_tables: torch.Tensor   # int32 [B, max_blocks_per_seq], padded with 0
    context_lens: torch.Tensor   # int32 [B], new token included
    q: torch.Tensor              # [B, Hq, D]
    key: torch.Tensor            # [B, Hkv, D]   K of the new token
    value: torch.Tensor          # [B, Hkv, D]   V of the new token
    slot_mapping: torch.Tensor   # int64 [B]     slot of the new token
    cow_pairs: torch.Tensor      # int64 [P, 2]  (src, dst) block copies before the write
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.q.shape[0])

    @property
    def num_blocks(self) -> int:
        return int(self.k_cache.shape[0])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max().item()) if self.num_seqs else 0

    @property
    def elem_bytes(self) -> int:
        return torch.empty((), dtype=self.dtype).element_size()

    def kv_bytes_logical(self) -> int:
        """Algorithmic K+V bytes one decode reads: every logical token of
        every sequence, every KV head, once."""
        tokens = int(self.context_lens.to(torch.int64).sum().item())
        return 2 * tokens * self.num_kv_heads * self.head_dim * self.elem_bytes

    def kv_bytes_unique(self) -> int:
        """K+V bytes of the distinct physical slots the batch reads (shared
        prefix blocks counted once)."""
        bs = self.block_size
        used = set()
        bt = self.block_tables.cpu().tolist()
        for i, L in enumerate(self.context_lens.cpu().tolist()):
            nb = (L + bs - 1) // bs
            for j in range(nb):
                rows = min(bs, L - j * bs)
                used.add((bt[i][j], rows))
        per_block = {}
        for b, rows in used:
            per_block[b] = max(per_block.get(b, 0), rows)
        tokens = sum(per_block.values())
        return 2 * tokens * self.num_kv_heads * self.head_dim * self.elem_bytes

    def to(self, device) -> "DecodeBatch":
        kw = {}
        for f in ("k_cache", "v_cache", "block_tables", "context_lens", "q",
                  "key", "value", "slot_mapping", "cow_pairs"):
            kw[f] = getattr(self, f).to(device)
        return DecodeBatch(self.name, self.dtype, self.block_size,
                           self.num_q_heads, self.num_kv_heads, self.head_dim,
                           self.scale, meta=dict(self.meta), **kw)


def _randn(shape, dtype, gen, device, chunk_elems=1 << 26):
    """fp32 N(0,1) rounded to dtype, drawn in chunks to bound temporaries."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device,
                                dtype=torch.float32).to(dtype)
    return out


def _pool(num_blocks, Hkv, BS, D, dtype, seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed + 1)
    k = _randn((num_blocks, Hkv, BS, D), dtype, g, device)
    v = _randn((num_blocks, Hkv, BS, D), dtype, g, device)
    return k, v


def _assemble(name, dtype, BS, Hq, Hkv, D, lens, tables, num_blocks, gen, seed,
              device, cow_pairs=None, slots=None, meta=None):
    """Common tail: draw q / new K / new V on the CPU generator, build padded
    tables and slot mapping, draw the pool on the device."""
    B = len(lens)
    max_nb = max([len(t) for t in tables] + [1])
    bt = torch.zeros((B, max_nb), dtype=torch.int32)
    for i, t in enumerate(tables):
        if t:
            bt[i, :len(t)] = torch.tensor(t, dtype=torch.int32)
    q = torch.randn((B, Hq, D), generator=gen, dtype=torch.float32).to(dtype)
    key = torch.randn((B, Hkv, D), generator=gen, dtype=torch.float32).to(dtype)
    value = torch.randn((B, Hkv, D), generator=gen, dtype=torch.float32).to(dtype)
    if slots is None:
        slots = []
        for i, L in enumerate(lens):
            if L == 0:
                slots.append(-1)
            else:
                pos = L - 1
                slots.append(tables[i][pos // BS] * BS + pos % BS)
    k_cache, v_cache = _pool(num_blocks, Hkv, BS, D, dtype, seed, device)
    pairs = torch.tensor(cow_pairs if cow_pairs else [], dtype=torch.int64).reshape(-1, 2)
    return DecodeBatch(
        name=name, dtype=dtype, block_size=BS, num_q_heads=Hq,
        num_kv_heads=Hkv, head_dim=D, scale=1.0 / math.sqrt(D),
        k_cache=k_cache, v_cache=v_cache, block_tables=bt.to(device),
        context_lens=torch.tensor(lens, dtype=torch.int32).to(device),
        q=q.to(device), key=key.to(device), value=value.to(device),
        slot_mapping=torch.tensor(slots, dtype=torch.int64).to(device),
        cow_pairs=pairs.to(device), meta=meta or {})


def _place(lens, BS, num_blocks, gen, contiguous=False):
    """Hand out physical blocks from a seeded permutation of the pool, in
    sequence order; returns one table per sequence. contiguous=True hands
    them out in pool order instead (each sequence's blocks adjacent, for the
    paged-vs-contiguous comparison); the permutation is drawn either way so
    every later draw is the same."""
    perm = torch.randperm(num_blocks, generator=gen).tolist()
    if contiguous:
        perm = list(range(num_blocks))
    tables, k = [], 0
    for L in lens:
        nb = (L + BS - 1) // BS
        tables.append(perm[k:k + nb])
        k += nb
    assert k <= num_blocks, "pool too small"
    return tables


# ---------------------------------------------------------------------------
# The five workloads
# ---------------------------------------------------------------------------

def tiny(device="cpu", seed=1001):
    """4 sequences of 1, 7, 16 and 33 tokens, block 16, one head, D=64, fp32,
    in a pool of 16 blocks placed by a seeded permutation."""
    gen = torch.Generator().manual_seed(seed)
    lens = [1, 7, 16, 33]
    BS, NB = 16, 16
    tables = _place(lens, BS, NB, gen)
    return _assemble("tiny_b4_h1_d64_f32", torch.float32, BS, 1, 1, 64, lens,
                     tables, NB, gen, seed, device)


def mha(device="cpu", seed=1002, num_seqs=64, num_heads=32, head_dim=128,
        min_len=128, max_len=2048, block_size=16, num_blocks=16384,
        dtype=torch.bfloat16, contiguous=False):
    """MHA decode step: context lengths uniform in [min_len, max_len], blocks
    drawn from a shuffled pool."""
    gen = torch.Generator().manual_seed(seed)
    lens = torch.randint(min_len, max_len + 1, (num_seqs,), generator=gen).tolist()
    need = sum((L + block_size - 1) // block_size for L in lens)
    num_blocks = max(num_blocks, need)
    tables = _place(lens, block_size, num_blocks, gen, contiguous)
    name = f"mha_b{num_seqs}_h{num_heads}_d{head_dim}_bs{block_size}_ctx{min_len}-{max_len}"
    name += "_contiguous" if contiguous else ""
    return _assemble(name, dtype, block_size, num_heads, num_heads, head_dim,
                     lens, tables, num_blocks, gen, seed, device)


def lognormal_lens(num_seqs, mean, sigma, lo, hi, gen):
    """Lengths round(LogNormal(mu, sigma)) with mu = ln(mean) - sigma^2 / 2
    (so the unclipped mean is `mean`), clipped to [lo, hi]."""
    mu = math.log(mean) - sigma * sigma / 2.0
    z = torch.randn(num_seqs, generator=gen, dtype=torch.float64)
    x = torch.exp(mu + sigma * z).round().clamp(lo, hi)
    return [int(v) for v in x.tolist()]


def gqa(device="cpu", seed=1003, num_seqs=256, num_q_heads=32, num_kv_heads=8,
        head_dim=128, mean_len=512, sigma=1.0, min_len=16, max_len=4096,
        block_size=16, dtype=torch.bfloat16, free_frac=0.10, contiguous=False):
    """GQA high-concurrency decode: log-normal lengths, pool sized to fit all
    sequences plus `free_frac` free blocks, shuffled."""
    gen = torch.Generator().manual_seed(seed)
    lens = lognormal_lens(num_seqs, mean_len, sigma, min_len, max_len, gen)
    need = sum((L + block_size - 1) // block_size for L in lens)
    num_blocks = int(math.ceil(need * (1.0 + free_frac)))
    tables = _place(lens, block_size, num_blocks, gen, contiguous)
    name = (f"gqa_b{num_seqs}_hq{num_q_heads}_hkv{num_kv_heads}_d{head_dim}"
            f"_bs{block_size}_lognormal{mean_len}") + ("_contiguous" if contiguous else "")
    return _assemble(name, dtype, block_size, num_q_heads, num_kv_heads,
                     head_dim, lens, tables, num_blocks, gen, seed, device)


def prefix_cow(device="cpu", seed=1004, num_pairs=32, prefix_len=2048,
               max_suffix=512, num_heads=40, head_dim=128, block_size=16,
               dtype=torch.float16, free_frac=0.10):
    """Prefix sharing + copy-on-write.

    2 * num_pairs sequences share one prefix of prefix_len tokens. The two
    siblings of a pair (parallel samples of one prompt) also share a suffix of
    s_j tokens, s_j uniform in [1, max_suffix] and not a multiple of the block
    size, so their last block is partly filled and shared. In this step each
    sibling writes one token at position prefix_len + s_j. The sibling picked
    by a seeded coin writes first: it gets a private copy of the shared block
    (a (src, dst) pair for the block copy) and writes into the copy; the other
    sibling then owns the original block alone and writes into it in place."""
    gen = torch.Generator().manual_seed(seed)
    BS = block_size
    assert prefix_len % BS == 0
    suffix = []
    for _ in range(num_pairs):
        while True:
            s = int(torch.randint(1, max_suffix + 1, (1,), generator=gen).item())
            if s % BS != 0:
                break
        suffix.append(s)
    n_prefix = prefix_len // BS
    n_suffix = [(s + BS - 1) // BS for s in suffix]
    need = n_prefix + sum(n_suffix) + num_pairs
    num_blocks = int(math.ceil(need * (1.0 + free_frac)))
    perm = torch.randperm(num_blocks, generator=gen).tolist()
    k = 0
    prefix_blocks = perm[k:k + n_prefix]; k += n_prefix
    pair_blocks = []
    for nb in n_suffix:
        pair_blocks.append(perm[k:k + nb]); k += nb
    coins = torch.randint(0, 2, (num_pairs,), generator=gen).tolist()
    lens, tables, slots, pairs = [], [], [], []
    for j in range(num_pairs):
        pos = prefix_len + suffix[j]            # position of the new token
        shared = prefix_blocks + pair_blocks[j]
        src = shared[-1]
        dst = perm[k]; k += 1
        for sib in range(2):
            if sib == coins[j]:                 # diverges first: copy-on-write
                tab = shared[:-1] + [dst]
                pairs.append([src, dst])
            else:                               # sole owner after the copy
                tab = list(shared)
            tables.append(tab)
            lens.append(pos + 1)
            slots.append(tab[pos // BS] * BS + pos % BS)
    name = (f"prefix_cow_b{2 * num_pairs}_h{num_heads}_d{head_dim}_bs{BS}"
            f"_prefix{prefix_len}")
    meta = {"prefix_blocks": prefix_blocks, "coins": coins, "suffix": suffix}
    return _assemble(name, dtype, BS, num_heads, num_heads, head_dim, lens,
                     tables, num_blocks, gen, seed, device, cow_pairs=pairs,
                     slots=slots, meta=meta)


def long_context(device="cpu", seed=1005, num_seqs=8, num_q_heads=64,
                 num_kv_heads=8, head_dim=128, min_len=32768, max_len=131072,
                 block_size=32, dtype=torch.bfloat16, free_frac=0.10):
    """Long-context decode: few sequences of 32K-128K tokens, GQA 64/8."""
    gen = torch.Generator().manual_seed(seed)
    lens = torch.randint(min_len, max_len + 1, (num_seqs,), generator=gen).tolist()
    need = sum((L + block_size - 1) // block_size for L in lens)
    num_blocks = int(math.ceil(need * (1.0 + free_frac)))
    tables = _place(lens, block_size, num_blocks, gen)
    name = (f"long_b{num_seqs}_hq{num_q_heads}_hkv{num_kv_heads}_d{head_dim}"
            f"_bs{block_size}_ctx{min_len}-{max_len}")
    return _assemble(name, dtype, block_size, num_q_heads, num_kv_heads,
                     head_dim, lens, tables, num_blocks, gen, seed, device)


def random_batch(device="cpu", seed=0, tensor_core_shape=False):
    """A small decode step with randomly drawn shapes, for broad parity
    coverage: dtype, head_dim 64/128, block size 8/16/32, 1-3 KV heads,
    1-16 query heads per KV head, 1-6 sequences whose lengths mix the edge
    cases (0, 1, a block boundary +- 1) with random lengths up to 700.
    tensor_core_shape=True draws only shapes the tensor-core kernel takes
    (16-bit, head_dim 128, 4-16 query heads per KV head, >= 16 query rows)."""
    gen = torch.Generator().manual_seed((6000 if tensor_core_shape else 5000) + seed)
    pick = lambda xs: xs[int(torch.randint(len(xs), (1,), generator=gen).item())]
    if tensor_core_shape:
        dtype = pick([torch.float16, torch.bfloat16])
        D = 128
    else:
        dtype = pick([torch.float32, torch.float16, torch.bfloat16])
        D = pick([64, 128])
    BS = pick([8, 16, 32])
    Hkv = pick([1, 2, 3])
    G = pick([4, 5, 6, 8, 12, 16] if tensor_core_shape else [1, 2, 3, 4, 5, 6, 8, 12, 16])
    B = int(torch.randint(1, 7, (1,), generator=gen).item())
    if tensor_core_shape:
        B = max(B, -(-16 // (G * Hkv)))
    lens = []
    for _ in range(B):
        kind = int(torch.randint(4, (1,), generator=gen).item())
        if kind == 0:
            lens.append(pick([0, 1, BS - 1, BS, BS + 1, 2 * BS + 1]))
        else:
            lens.append(int(torch.randint(1, 701, (1,), generator=gen).item()))
    need = sum((L + BS - 1) // BS for L in lens)
    NB = need + 3
    tables = _place(lens, BS, NB, gen)
    name = (f"random{'tc' if tensor_core_shape else ''}{seed}_b{B}_hq{G * Hkv}_hkv{Hkv}"
            f"_d{D}_bs{BS}_{str(dtype)[6:]}")
    return _assemble(name, dtype, BS, G * Hkv, Hkv, D, lens, tables, NB, gen,
                     (6000 if tensor_core_shape else 5000) + seed, device)


# Full-size workloads, in the order of the task's configuration list.
FULL = {
    "tiny": tiny,
    "mha": mha,
    "gqa": gqa,
    "prefix_cow": prefix_cow,
    "long": long_context,
}

# Reduced sizes the oracle finishes in seconds; each still spans several
# 128-token tiles, several splits and a ragged last block.
SMALL = {
    "tiny": lambda device="cpu": tiny(device),
    "mha": lambda device="cpu": mha(device, num_seqs=6, num_heads=4,
                                    min_len=1, max_len=700, num_blocks=400),
    "gqa": lambda device="cpu": gqa(device, num_seqs=12, num_q_heads=16,
                                    num_kv_heads=4, mean_len=300, min_len=1,
                                    max_len=1500),
    "gqa8": lambda device="cpu": gqa(device, seed=1013, num_seqs=6,
                                     num_q_heads=16, num_kv_heads=2,
                                     mean_len=600, min_len=1, max_len=2500),
    "prefix_cow": lambda device="cpu": prefix_cow(device, num_pairs=3,
                                                  prefix_len=256,
                                                  max_suffix=200, num_heads=4),
    "long": lambda device="cpu": long_context(device, num_seqs=2,
                                              num_q_heads=16, num_kv_heads=2,
                                              min_len=3000, max_len=6000),
}
