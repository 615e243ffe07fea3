"""Shared pieces of the GPU parity tests: moving inputs to NumPy for the
oracle, running one decode step through the C-ABI binding, comparing."""

from __future__ import annotations

import numpy as np
import torch

from oracle import ORACLE
from paged_kv_cache_339_b200 import ops

TOL = {torch.float32: 1e-5, torch.float16: 2e-3, torch.bfloat16: 2e-3}
RAW = {torch.float32: torch.int32, torch.float16: torch.int16, torch.bfloat16: torch.int16}


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact upcast of a (possibly 16-bit) tensor to fp64 NumPy."""
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit pattern, for bit-exact comparisons."""
    return t.detach().contiguous().view(RAW[t.dtype]).cpu().numpy()


def pool_f64(t: torch.Tensor) -> np.ndarray:
    """A stored KV pool, as the oracle's logical [NB, Hkv, BS, D] fp64 view."""
    return ORACLE.logical_pool(f64(t))


def pool_bits(t: torch.Tensor) -> np.ndarray:
    """A stored KV pool's bit patterns in the logical [NB, Hkv, BS, D] view."""
    return ORACLE.logical_pool(bits(t))


def run_step(batch, split_tokens=0, path=ops.PA_PATH_AUTO, workspace=None, write=True):
    """copy-on-write copies, new-token write, decode - the whole hot path."""
    if write:
        if batch.cow_pairs.numel():
            ops.pa_copy_blocks(batch.k_cache, batch.v_cache, batch.cow_pairs)
        ops.pa_write_kv(batch.k_cache, batch.v_cache, batch.key, batch.value,
                        batch.slot_mapping)
    B, Hq, D = batch.q.shape
    max_ctx = max(batch.max_context_len, 1)
    if workspace is None:
        workspace = ops.decode_workspace(B, Hq, D, max_ctx, batch.block_size, split_tokens)
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device=batch.q.device)
    ops.pa_decode(out, batch.q, batch.k_cache, batch.v_cache, batch.block_tables,
                  batch.context_lens, max_ctx, batch.scale, workspace,
                  split_tokens=split_tokens, path=path)
    torch.cuda.synchronize()
    assert ops.pa_decode_status(workspace) == ops.PA_OK
    return out


def oracle_step(batch_cpu):
    """The same step on the CPU oracle, from host copies of the inputs."""
    kc, vc = pool_f64(batch_cpu.k_cache), pool_f64(batch_cpu.v_cache)
    if batch_cpu.cow_pairs.numel():
        kc, vc = ORACLE.copy_blocks(kc, vc, batch_cpu.cow_pairs.numpy())
    kc, vc = ORACLE.write_kv(kc, vc, f64(batch_cpu.key), f64(batch_cpu.value),
                             batch_cpu.slot_mapping.numpy())
    return ORACLE.decode(f64(batch_cpu.q), kc, vc, batch_cpu.block_tables.numpy(),
                         batch_cpu.context_lens.numpy(), float(np.float32(batch_cpu.scale)))


def max_abs_err(out: torch.Tensor, ref: np.ndarray) -> float:
    o = out.detach().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o)), "non-finite output"
    return float(np.max(np.abs(o - ref))) if o.size else 0.0


def sampled_reference(batch, seq, h):
    """Oracle output row for (seq, query head h) of a device-resident batch,
    computed from just that sequence's blocks of its KV head (copied back)."""
    L = int(batch.context_lens[seq].item())
    BS = batch.block_size
    nb = (L + BS - 1) // BS
    G = batch.num_q_heads // batch.num_kv_heads
    kv = h // G
    rows = batch.block_tables[seq, :nb].long()
    ksub = pool_f64(batch.k_cache[rows][:, kv:kv + 1])      # [nb, 1, BS, D]
    vsub = pool_f64(batch.v_cache[rows][:, kv:kv + 1])
    return ORACLE.decode_one(f64(batch.q[seq, h]), ksub, vsub, np.arange(nb), L, 0, 1,
                             float(np.float32(batch.scale)))


def reference_rows(batch, seq, heads):
    """Oracle output rows {h: row} for the given query heads of one sequence,
    copying each KV head's blocks back once for all its query heads."""
    L = int(batch.context_lens[seq].item())
    BS = batch.block_size
    nb = (L + BS - 1) // BS
    G = batch.num_q_heads // batch.num_kv_heads
    rows = batch.block_tables[seq, :nb].long()
    scale = float(np.float32(batch.scale))
    res = {}
    for kv in sorted({h // G for h in heads}):
        ksub = pool_f64(batch.k_cache[rows][:, kv:kv + 1])
        vsub = pool_f64(batch.v_cache[rows][:, kv:kv + 1])
        for h in heads:
            if h // G == kv:
                res[h] = ORACLE.decode_one(f64(batch.q[seq, h]), ksub, vsub, np.arange(nb),
                                           L, 0, 1, scale)
    return res
