"""Host-side pieces of bench.py, on the CPU: the packed input buffer of the
end-to-end pipeline and the parity bookkeeping of the CPU-baseline sample."""

import numpy as np
import pytest
import torch

import bench
from oracle import ORACLE
from paged_kv_cache_339_b200 import workloads as W


@pytest.mark.parametrize("name", ["tiny", "gqa8", "prefix_cow", "long"])
def test_packed_step_inputs_round_trip(name):
    b = W.SMALL[name]("cpu")
    buf, offs = bench.pack_step_inputs(b)
    assert buf.dtype == torch.uint8 and buf.numel() % 256 == 0
    assert all(o % 256 == 0 for o in offs.values())
    views = bench.step_input_views(buf, b, offs)
    for k in bench.STEP_INPUTS:
        t = getattr(b, k)
        v = views[k]
        assert v.dtype == t.dtype and v.shape == t.shape, k
        assert torch.equal(v, t), k                        # every byte recovered
    # inputs do not overlap: each lies inside its own 256-byte-rounded span
    spans = sorted((offs[k], offs[k] + getattr(b, k).numel() * getattr(b, k).element_size())
                   for k in bench.STEP_INPUTS)
    assert all(e <= s2 for (_, e), (s2, _) in zip(spans, spans[1:]))


def test_parity_bookkeeping_catches_a_planted_error():
    b = W.tiny("cpu")
    f = lambda t: t.float().numpy().astype(np.float64)
    ref = ORACLE.decode(f(b.q), ORACLE.logical_pool(f(b.k_cache)),
                        ORACLE.logical_pool(f(b.v_cache)), b.block_tables.numpy(),
                        b.context_lens.numpy(), float(np.float32(b.scale)))
    out = torch.from_numpy(ref.astype(np.float32))
    nbytes, _, rows, nseq, _, err = bench.oracle_sample(b, 5.0, out)
    assert nseq == b.num_seqs and rows == b.num_seqs * b.num_q_heads
    assert nbytes == b.kv_bytes_logical()                  # a whole batch: every KV byte once
    assert err < 1e-6                                      # fp32 rounding of the oracle only
    planted = out.clone()
    planted[2, 0, 5] += 0.01
    _, _, _, _, _, err2 = bench.oracle_sample(b, 5.0, planted)
    assert err2 == pytest.approx(0.01, rel=1e-3)


def test_oracle_sample_credits_kv_bytes_per_query_head_row():
    """With query groups, each (sequence, query head) row carries 1 / G of its
    KV head's bytes, so rows of a whole batch add up to its KV bytes."""
    b = W.SMALL["gqa8"]("cpu")
    G = b.num_q_heads // b.num_kv_heads
    nbytes, _, rows, _, _, _ = bench.oracle_sample(b, 60.0)
    assert rows == b.num_seqs * b.num_q_heads and G > 1
    assert nbytes == pytest.approx(b.kv_bytes_logical(), rel=1e-12)
    # a tiny budget stops after the first row: 2 * L_0 * D * e / G bytes
    nb1, _, r1, s1, _, _ = bench.oracle_sample(b, 0.0)
    L0 = int(b.context_lens[0])
    assert (r1, s1) == (1, 1)
    assert nb1 == pytest.approx(2 * L0 * b.head_dim * b.elem_bytes / G)
