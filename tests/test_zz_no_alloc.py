"""pa_decode_noalloc against pa_decode and the fp64 oracle, through the C-ABI.

pa_decode_noalloc serves callers that cannot allocate device memory (a process
that gave nearly all of HBM to its KV-cache pool, or a latency-critical path
that cannot take cudaMalloc's synchronisation): it runs the same decode with
the library's fixed 32 MiB device scratch instead of a caller workspace, and
pa_decode_noalloc_status reads the status word the kernels leave in that
scratch. This file sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process, where
its first call performs the one-time set-up.
"""

import pytest
import torch

from paged_kv_cache_339_b200 import build as pa_build
from paged_kv_cache_339_b200 import ops
from paged_kv_cache_339_b200 import workloads as W
from tests.gpu_helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pa_build.build()
    ops.library()


def _both(b, split=0):
    """Write the step's new tokens, then decode with pa_decode and with
    pa_decode_noalloc; returns (noalloc output, pa_decode output, status of
    the noalloc call)."""
    if b.cow_pairs.numel():
        ops.pa_copy_blocks(b.k_cache, b.v_cache, b.cow_pairs)
    ops.pa_write_kv(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping)
    B, Hq, D = b.q.shape
    max_ctx = b.max_context_len
    ws = ops.decode_workspace(B, Hq, D, max_ctx, b.block_size, split)
    ref = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
    ops.pa_decode(ref, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, max_ctx,
                  b.scale, ws, split_tokens=split)
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    ops.pa_decode_noalloc(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                          max_ctx, b.scale, split_tokens=split)
    status = ops.pa_decode_noalloc_status()
    torch.cuda.synchronize()
    return out, ref, status


def test_noalloc_matches_pa_decode_and_oracle_on_two_calls_in_a_row():
    # call 1: GQA (tensor-core path), several splits per sequence
    b1 = W.SMALL["gqa8"]("cuda")
    bc1 = b1.to("cpu")
    out1, ref1, st1 = _both(b1, split=128)
    assert st1 == ops.PA_OK
    assert torch.isfinite(out1).all()
    assert (out1 - ref1).abs().max().item() <= TOL[b1.dtype]
    assert max_abs_err(out1, oracle_step(bc1)) <= TOL[b1.dtype]
    # call 2: a different shape (MHA, CUDA-core path) over the scratch the first
    # call left behind
    b2 = W.SMALL["mha"]("cuda")
    bc2 = b2.to("cpu")
    out2, ref2, st2 = _both(b2)
    assert st2 == ops.PA_OK
    assert torch.isfinite(out2).all()
    assert (out2 - ref2).abs().max().item() <= TOL[b2.dtype]
    assert max_abs_err(out2, oracle_step(bc2)) <= TOL[b2.dtype]


def test_noalloc_status_reports_a_bad_table_entry_and_clears():
    """A table entry outside the pool is read as block 0 and raises
    PA_ERR_INVALID_ARG in the scratch's status word; the next clean call
    clears it."""
    b = W.SMALL["mha"]("cuda")
    B, Hq, D = b.q.shape
    b.block_tables[0, 0] = b.num_blocks + 1000
    out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
    ops.pa_decode_noalloc(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                          b.max_context_len, b.scale)
    assert ops.pa_decode_noalloc_status() == ops.PA_ERR_INVALID_ARG
    b = W.SMALL["mha"]("cuda")
    ops.pa_decode_noalloc(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                          b.max_context_len, b.scale)
    assert ops.pa_decode_noalloc_status() == ops.PA_OK


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 4096 sequences x 64 heads x 128-dim partials need far more than 32 MiB
    q = torch.zeros((4096, 64, 128), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    kc = torch.zeros((16, 64, 16, 128), dtype=torch.float32, device="cuda")
    bt = torch.zeros((4096, 4096), dtype=torch.int32, device="cuda")
    lens = torch.ones(4096, dtype=torch.int32, device="cuda")
    with pytest.raises(ops.PagedAttnError) as e:
        ops.pa_decode_noalloc(out, q, kc, kc, bt, lens, 65536, 0.1)
    assert e.value.status == ops.PA_ERR_WORKSPACE_TOO_SMALL
    # other argument errors are reported as such, not as a scratch that is too
    # small: 64 query heads over 48 KV heads is not a whole group
    kc48 = torch.zeros((16, 48, 16, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(ops.PagedAttnError) as e:
        ops.pa_decode_noalloc(out, q, kc48, kc48, bt, lens, 65536, 0.1)
    assert e.value.status == ops.PA_ERR_INVALID_ARG
