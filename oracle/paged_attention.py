"""Plain fp64 CPU oracle for paged KV-cache decode.

TEST INFRASTRUCTURE. Only the test suite, the smoke check of the package entry
point and the CPU-baseline / reference leg of the benchmark may import this
module. The CUDA library never does, and the two share no code: the only thing
both sides consume is the seeded input generator, which holds none of the
arithmetic below.

What is computed, and which passage each step follows
------------------------------------------------------
Pages: "Paged Attention: Virtual Memory for the KV Cache" (P1),
"Paged Attention as a Memory Manager" (P2), and the glossary entry
"Paged attention" (P3).

* Pool of fixed-size blocks. The cache is cut into blocks of ``block_size``
  tokens, each holding the keys and values of those tokens (P1, "The fix
  borrowed from operating systems"; P2, "Virtual Memory as the Blueprint").
  Layout reading: two pools ``k_cache`` / ``v_cache`` of shape
  ``[num_blocks, num_kv_heads, block_size, head_dim]``.
* In-block storage order. Each (block, KV head) tile of block_size x head_dim
  elements is stored contiguously, its rows cut into 64-element halves and
  grouped 16 tokens at a time: element (t, d) sits at
  ((t // SH) * NH + d // 64) * SH * 64 + (t % SH) * 64 + d % 64 with
  SH = min(block_size, 16) and NH = head_dim // 64 (plain row-major when
  head_dim is 64). ``logical_pool`` / ``physical_pool`` convert between this
  order and the logical ``[num_blocks, num_kv_heads, block_size, head_dim]``
  view every other function here works on. The pages leave the inside of a
  block open; this order lets one copy of a tile feed the tensor cores.
* Block table. Each sequence keeps an ordered list of the physical blocks that
  hold it; logical token ``j`` lives in block ``table[j // block_size]`` at
  offset ``j % block_size`` (P1, "The fix borrowed from operating systems").
* The kernel walks the logical sequence in order, as though its tokens sat
  back to back (P3, "What is
  Paged Attention?"). So the oracle gathers each sequence into one contiguous
  array and then runs ordinary attention on it.
* Attention formula. The pages name the operation but never write it (P2's
  section "How the Kernel Executes Paged Attention" stops after one paragraph).
  Reading taken: scaled dot-product decode attention,
  ``o = softmax(scale * q . K^T) . V`` over the first ``context_len`` tokens,
  query head ``h`` using KV head ``h // (num_q_heads // num_kv_heads)``
  (grouped-query attention is named in P1, "What it does not fix").
* Writing a token into its slot: a request takes a new block only once its
  current one is full (P1, "The fix borrowed from operating systems"); slot ``s`` addresses block ``s // block_size``, offset
  ``s % block_size``. A negative slot means "no write" (padding).
* Copy-on-write: a sequence that diverges inside a shared block first gets its
  own copy of that block (P1, "Sharing comes almost for free"; P2, "Virtual
  Memory as the Blueprint").
* Swapping blocks out to host memory and back: when memory runs out the
  server evicts a sequence and later recomputes or swaps its blocks back (P1,
  "What it does not fix"). A swap is a block copy between the device pools
  and a host pool, in either direction.
* Split-context partial softmax and merge: not on the pages. It is the exact
  algebraic regrouping of the softmax sum over a partition of the tokens; the
  oracle keeps it only to pin that regrouping (see ``partial`` / ``merge``).

Every function is pinned by tests that do not re-type it (closed forms, a
golden fixture, invariants the pages state, and planted-mistake checks); none
is "parity unpinned".
"""

from __future__ import annotations

import numpy as np


class PagedAttentionOracle:
    """fp64 reference. Methods are overridable so the pin suite can plant
    mistakes in a subclass and check that some pin catches each one."""

    # ------------------------------------------------------------------
    # In-block storage order (a reading: the pages leave it open)
    # ------------------------------------------------------------------
    def tile_offset(self, t: int, d: int, block_size: int, head_dim: int) -> int:
        """Element offset of (token t, column d) inside one (block, head) tile."""
        sh = min(block_size, 16)
        nh = head_dim // 64
        return ((t // sh) * nh + d // 64) * sh * 64 + (t % sh) * 64 + d % 64

    def logical_pool(self, pool: np.ndarray) -> np.ndarray:
        """Stored pool [NB, Hkv, BS, D] (tiles in storage order) -> logical
        [NB, Hkv, BS, D] with element [b, h, t, d] = K/V of token t, column d."""
        NB, H, BS, D = pool.shape
        sh, nh = min(BS, 16), D // 64
        return (pool.reshape(NB, H, BS // sh, nh, sh, 64)
                .transpose(0, 1, 2, 4, 3, 5).reshape(NB, H, BS, D))

    def physical_pool(self, pool: np.ndarray) -> np.ndarray:
        """Inverse of logical_pool."""
        NB, H, BS, D = pool.shape
        sh, nh = min(BS, 16), D // 64
        return (pool.reshape(NB, H, BS // sh, sh, nh, 64)
                .transpose(0, 1, 2, 4, 3, 5).reshape(NB, H, BS, D))

    # ------------------------------------------------------------------
    # Block addressing (P1, "The fix borrowed from operating systems")
    # ------------------------------------------------------------------
    def locate(self, slot: int, block_size: int) -> tuple[int, int]:
        """Physical (block, offset) of a slot index."""
        return slot // block_size, slot % block_size

    def gather(self, cache: np.ndarray, table_row: np.ndarray,
               context_len: int) -> np.ndarray:
        """Contiguous ``[context_len, num_kv_heads, head_dim]`` view of one
        sequence: logical token j comes from block table_row[j // block_size],
        offset j % block_size (P3, "What is Paged Attention?": the sequence is
        read in logical order, as though stored back to back)."""
        block_size = cache.shape[2]
        j = np.arange(context_len)
        blocks = np.asarray(table_row)[j // block_size]
        offsets = j % block_size
        return cache[blocks, :, offsets, :]

    # ------------------------------------------------------------------
    # Attention on a contiguous sequence (reading: plain scaled dot-product)
    # ------------------------------------------------------------------
    def attend(self, q: np.ndarray, K: np.ndarray, V: np.ndarray,
               scale: float) -> np.ndarray:
        """softmax(scale * K q) . V for one query vector, in fp64.
        q: [D]; K, V: [L, D]; L >= 1."""
        q = np.asarray(q, dtype=np.float64)
        K = np.asarray(K, dtype=np.float64)
        V = np.asarray(V, dtype=np.float64)
        s = (K @ q) * np.float64(scale)
        p = np.exp(s - s.max())
        return (p @ V) / p.sum()

    def kv_head_of(self, h: int, num_q_heads: int, num_kv_heads: int) -> int:
        """Grouped-query mapping: consecutive query heads share one KV head."""
        return h // (num_q_heads // num_kv_heads)

    def decode_one(self, q_row: np.ndarray, k_cache: np.ndarray,
                   v_cache: np.ndarray, table_row: np.ndarray,
                   context_len: int, h: int, num_q_heads: int,
                   scale: float) -> np.ndarray:
        """Output row [D] of query head h of one sequence. Zero when the
        context is empty (reading: nothing to attend to)."""
        D = k_cache.shape[3]
        if context_len == 0:
            return np.zeros(D, dtype=np.float64)
        kv = self.kv_head_of(h, num_q_heads, k_cache.shape[1])
        K = self.gather(k_cache, table_row, context_len)[:, kv, :]
        V = self.gather(v_cache, table_row, context_len)[:, kv, :]
        return self.attend(q_row, K, V, scale)

    def decode(self, q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
               block_tables: np.ndarray, context_lens: np.ndarray,
               scale: float) -> np.ndarray:
        """Paged decode for a batch: q [B, Hq, D] -> out [B, Hq, D] fp64."""
        B, Hq, D = q.shape
        out = np.zeros((B, Hq, D), dtype=np.float64)
        for i in range(B):
            L = int(context_lens[i])
            for h in range(Hq):
                out[i, h] = self.decode_one(q[i, h], k_cache, v_cache,
                                            block_tables[i], L, h, Hq, scale)
        return out

    # ------------------------------------------------------------------
    # Split-context regrouping (not on the pages; exact algebra)
    # ------------------------------------------------------------------
    def partial(self, q: np.ndarray, K: np.ndarray, V: np.ndarray,
                scale: float, start: int, end: int):
        """Softmax pieces over tokens [start, end): (m, l, acc) with
        m = max s, l = sum exp(s - m), acc = sum exp(s - m) v."""
        s = (np.asarray(K[start:end], np.float64) @ np.asarray(q, np.float64)) * np.float64(scale)
        m = s.max()
        p = np.exp(s - m)
        return m, p.sum(), p @ np.asarray(V[start:end], np.float64)

    def merge(self, parts) -> np.ndarray:
        """Combine pieces from a partition of the tokens:
        M = max m_p, L = sum l_p e^(m_p - M), o = sum acc_p e^(m_p - M) / L."""
        M = max(m for m, _, _ in parts)
        L = sum(l * np.exp(m - M) for m, l, _ in parts)
        acc = sum(a * np.exp(m - M) for m, _, a in parts)
        return acc / L

    # ------------------------------------------------------------------
    # Cache mutation: token write and copy-on-write block copy
    # ------------------------------------------------------------------
    def write_kv(self, k_cache: np.ndarray, v_cache: np.ndarray,
                 key: np.ndarray, value: np.ndarray,
                 slot_mapping: np.ndarray):
        """Store token t's K/V ([T, Hkv, D]) into slot slot_mapping[t] of both
        pools; slots < 0 are skipped. Returns new arrays (inputs untouched).
        Works on any dtype, including raw integer views, so comparisons with
        the device result are bit-exact."""
        k_out, v_out = k_cache.copy(), v_cache.copy()
        block_size = k_cache.shape[2]
        for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
            if slot < 0:
                continue
            b, off = self.locate(int(slot), block_size)
            k_out[b, :, off, :] = key[t]
            v_out[b, :, off, :] = value[t]
        return k_out, v_out

    def copy_blocks(self, k_cache: np.ndarray, v_cache: np.ndarray,
                    pairs: np.ndarray):
        """Copy-on-write copies: for each (src, dst), block dst of both pools
        becomes a byte copy of block src. Returns new arrays."""
        k_out, v_out = k_cache.copy(), v_cache.copy()
        for src, dst in np.asarray(pairs).reshape(-1, 2).tolist():
            k_out[dst] = k_cache[src]
            v_out[dst] = v_cache[src]
        return k_out, v_out


    def swap_blocks(self, dev_k: np.ndarray, dev_v: np.ndarray, host_k: np.ndarray,
                    host_v: np.ndarray, pairs: np.ndarray, direction: int):
        """Swap (P1, "What it does not fix"): direction 0 (out) copies device
        block src to host block dst, direction 1 (in) host block src to device
        block dst, both pools; pairs with an index outside its pool are
        skipped. Returns new (dev_k, dev_v, host_k, host_v)."""
        dk, dv, hk, hv = dev_k.copy(), dev_v.copy(), host_k.copy(), host_v.copy()
        if direction == 0:
            src_k, src_v, dst_k, dst_v = dev_k, dev_v, hk, hv
        else:
            src_k, src_v, dst_k, dst_v = host_k, host_v, dk, dv
        for src, dst in np.asarray(pairs).reshape(-1, 2).tolist():
            if not (0 <= src < len(src_k) and 0 <= dst < len(dst_k)):
                continue
            dst_k[dst] = src_k[src]
            dst_v[dst] = src_v[src]
        return dk, dv, hk, hv


ORACLE = PagedAttentionOracle()

# Module-level names for the common calls.
logical_pool = ORACLE.logical_pool
physical_pool = ORACLE.physical_pool
tile_offset = ORACLE.tile_offset
gather = ORACLE.gather
attend = ORACLE.attend
decode = ORACLE.decode
decode_one = ORACLE.decode_one
write_kv = ORACLE.write_kv
copy_blocks = ORACLE.copy_blocks
swap_blocks = ORACLE.swap_blocks
partial = ORACLE.partial
merge = ORACLE.merge
