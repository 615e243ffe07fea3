"""The CPU oracle against its pins, and the pins against planted mistakes.

Each pin (tests/oracle_pins.py) checks the oracle against something fixed
independently of its code. The second half plants one plausible mistake at a
time in a subclass of the oracle (on the CPU) and requires that at least one
pin fails, so a wrong oracle cannot pass the pin suite unnoticed.
"""

import numpy as np
import pytest

from oracle import PagedAttentionOracle
from tests import oracle_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(PagedAttentionOracle())


# ---------------------------------------------------------------------------
# Planted mistakes
# ---------------------------------------------------------------------------

class NoScale(PagedAttentionOracle):
    def attend(self, q, K, V, scale):
        return super().attend(q, K, V, 1.0)


class NegatedScores(PagedAttentionOracle):
    def attend(self, q, K, V, scale):
        return super().attend(-np.asarray(q, np.float64), K, V, scale)


class KeysValuesSwapped(PagedAttentionOracle):
    def attend(self, q, K, V, scale):
        return super().attend(q, V, K, scale)


class GqaModulo(PagedAttentionOracle):
    def kv_head_of(self, h, num_q_heads, num_kv_heads):
        return h % num_kv_heads


class GatherIndexSwap(PagedAttentionOracle):
    def gather(self, cache, table_row, context_len):
        bs = cache.shape[2]
        j = np.arange(context_len)
        return cache[np.asarray(table_row)[np.minimum(j % bs, len(table_row) - 1)], :, (j // bs) % bs, :]


class GatherWrongOffset(PagedAttentionOracle):
    def gather(self, cache, table_row, context_len):
        bs = cache.shape[2]
        j = np.arange(context_len)
        return cache[np.asarray(table_row)[j // bs], :, (j + 1) % bs, :]


class ContextOffByOne(PagedAttentionOracle):
    def decode_one(self, q_row, k_cache, v_cache, table_row, context_len, h,
                   num_q_heads, scale):
        return super().decode_one(q_row, k_cache, v_cache, table_row,
                                  max(context_len - 1, 1) if context_len else 0,
                                  h, num_q_heads, scale)


class NoMaxSubtraction(PagedAttentionOracle):
    def attend(self, q, K, V, scale):
        s = (np.asarray(K, np.float64) @ np.asarray(q, np.float64)) * scale
        p = np.exp(s)
        return (p @ np.asarray(V, np.float64)) / p.sum()


class NoNormalisation(PagedAttentionOracle):
    def attend(self, q, K, V, scale):
        s = (np.asarray(K, np.float64) @ np.asarray(q, np.float64)) * scale
        p = np.exp(s - s.max())
        return p @ np.asarray(V, np.float64)


class WriteSlotSwap(PagedAttentionOracle):
    def locate(self, slot, block_size):
        return slot % block_size, slot // block_size


class WriteKeyIntoBoth(PagedAttentionOracle):
    def write_kv(self, k_cache, v_cache, key, value, slot_mapping):
        return super().write_kv(k_cache, v_cache, key, key, slot_mapping)


class WriteNegativeSlotWraps(PagedAttentionOracle):
    def write_kv(self, k_cache, v_cache, key, value, slot_mapping):
        k_out, v_out = k_cache.copy(), v_cache.copy()
        bs = k_cache.shape[2]
        for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
            b, off = self.locate(int(slot), bs)       # no skip for slot < 0
            k_out[b, :, off, :] = key[t]
            v_out[b, :, off, :] = value[t]
        return k_out, v_out


class CopyReversed(PagedAttentionOracle):
    def copy_blocks(self, k_cache, v_cache, pairs):
        return super().copy_blocks(k_cache, v_cache, np.asarray(pairs)[:, ::-1])


class MergeWithoutRescale(PagedAttentionOracle):
    def merge(self, parts):
        return sum(a for _, _, a in parts) / sum(l for _, l, _ in parts)


class EmptyContextNotZero(PagedAttentionOracle):
    def decode_one(self, q_row, k_cache, v_cache, table_row, context_len, h,
                   num_q_heads, scale):
        return super().decode_one(q_row, k_cache, v_cache, table_row,
                                  max(context_len, 1), h, num_q_heads, scale)


class TileHalvesSwapped(PagedAttentionOracle):
    def logical_pool(self, pool):
        NB, H, BS, D = pool.shape
        sh, nh = min(BS, 16), D // 64
        return (pool.reshape(NB, H, BS // sh, sh, nh, 64)
                .transpose(0, 1, 2, 3, 4, 5).reshape(NB, H, BS, D))


class TileGroupOf8(PagedAttentionOracle):
    def tile_offset(self, t, d, block_size, head_dim):
        sh, nh = min(block_size, 8), head_dim // 64
        return ((t // sh) * nh + d // 64) * sh * 64 + (t % sh) * 64 + d % 64


class SwapDirectionIgnored(PagedAttentionOracle):
    def swap_blocks(self, dev_k, dev_v, host_k, host_v, pairs, direction):
        return super().swap_blocks(dev_k, dev_v, host_k, host_v, pairs, 0)


class SwapPairsReversed(PagedAttentionOracle):
    def swap_blocks(self, dev_k, dev_v, host_k, host_v, pairs, direction):
        return super().swap_blocks(dev_k, dev_v, host_k, host_v,
                                   np.asarray(pairs)[:, ::-1], direction)


class SwapKeysOnly(PagedAttentionOracle):
    def swap_blocks(self, dev_k, dev_v, host_k, host_v, pairs, direction):
        dk, _, hk, _ = super().swap_blocks(dev_k, dev_v, host_k, host_v, pairs, direction)
        return dk, dev_v.copy(), hk, host_v.copy()


MUTANTS = [SwapDirectionIgnored, SwapPairsReversed, SwapKeysOnly, TileHalvesSwapped, TileGroupOf8, NoScale, NegatedScores, KeysValuesSwapped, GqaModulo,
           GatherIndexSwap, GatherWrongOffset, ContextOffByOne,
           NoMaxSubtraction, NoNormalisation, WriteSlotSwap, WriteKeyIntoBoth,
           WriteNegativeSlotWraps, CopyReversed, MergeWithoutRescale,
           EmptyContextNotZero]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda c: c.__name__)
def test_planted_mistake_is_caught(mutant):
    orc = mutant()
    failed = []
    with np.errstate(all="ignore"):
        for check in pins.ALL_CHECKS:
            try:
                check(orc)
            except Exception:  # noqa: BLE001 - any failure counts as caught
                failed.append(check.__name__)
    assert failed, f"no pin catches {mutant.__name__}"
