"""pa_swap_blocks on the GPU: blocks moved between the device pools and a
pinned host pool ("Paged Attention: Virtual Memory for the KV Cache", "What it
does not fix": preemption by swapping). Bit-exact against the oracle's block
copy, and a sequence evicted and brought back into other blocks decodes to
exactly the same output."""

import numpy as np
import pytest
import torch

from oracle import ORACLE
from paged_kv_cache_339_b200 import build as pa_build
from paged_kv_cache_339_b200 import ops
from paged_kv_cache_339_b200 import workloads as W
from tests.gpu_helpers import bits, run_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pa_build.build()
    ops.library()


def _host_pool(like, nblocks, gen):
    t = torch.empty((nblocks,) + tuple(like.shape[1:]), dtype=like.dtype, pin_memory=True)
    raw = torch.randint(-(1 << 15), 1 << 15, t.shape, generator=gen, dtype=torch.int32)
    if like.dtype == torch.float32:
        t.view(torch.int32).copy_(raw)
    else:
        t.view(torch.int16).copy_(raw.to(torch.int16))
    return t


@pytest.mark.parametrize("name", ["tiny", "gqa8", "prefix_cow"])
def test_swap_out_and_in_bit_exact(name):
    b = W.SMALL[name]("cuda")
    gen = torch.Generator().manual_seed(77)
    NB = b.k_cache.shape[0]
    NH = 5
    hk, hv = _host_pool(b.k_cache, NH, gen), _host_pool(b.v_cache, NH, gen)
    # out: device src -> host dst, with pairs outside either pool skipped
    out_pairs = np.array([[1, 3], [NB - 1, 0], [NB + 2, 1], [2, NH + 4], [-1, 2]], np.int64)
    dk0, dv0 = bits(b.k_cache), bits(b.v_cache)
    hk0, hv0 = bits(hk), bits(hv)
    ops.pa_swap_blocks(b.k_cache, b.v_cache, hk, hv, torch.from_numpy(out_pairs).cuda(),
                       ops.PA_SWAP_OUT)
    torch.cuda.synchronize()
    ek = ORACLE.swap_blocks(dk0, dv0, hk0, hv0, out_pairs, 0)
    assert np.array_equal(bits(b.k_cache), ek[0]) and np.array_equal(bits(b.v_cache), ek[1])
    assert np.array_equal(bits(hk), ek[2]) and np.array_equal(bits(hv), ek[3])
    # in: host src -> device dst
    in_pairs = np.array([[3, 0], [0, NB - 2], [4, NB + 1], [NH, 1]], np.int64)
    ops.pa_swap_blocks(b.k_cache, b.v_cache, hk, hv, torch.from_numpy(in_pairs).cuda(),
                       ops.PA_SWAP_IN)
    torch.cuda.synchronize()
    ei = ORACLE.swap_blocks(*ek, in_pairs, 1)
    assert np.array_equal(bits(b.k_cache), ei[0]) and np.array_equal(bits(b.v_cache), ei[1])
    assert np.array_equal(bits(hk), ei[2]) and np.array_equal(bits(hv), ei[3])


def test_evicted_sequence_decodes_identically_after_swap_in():
    b = W.SMALL["gqa8"]("cuda")
    before = run_step(b)                      # write + decode
    seq = int(torch.argmax(b.context_lens).item())
    L = int(b.context_lens[seq].item())
    nblk = (L + b.block_size - 1) // b.block_size
    old = b.block_tables[seq, :nblk].clone()
    # evict to host
    hk = torch.empty((nblk,) + tuple(b.k_cache.shape[1:]), dtype=b.k_cache.dtype, pin_memory=True)
    hv = torch.empty_like(hk, pin_memory=True)
    out_pairs = torch.stack([old.long(), torch.arange(nblk, device="cuda")], 1).contiguous()
    ops.pa_swap_blocks(b.k_cache, b.v_cache, hk, hv, out_pairs, ops.PA_SWAP_OUT)
    # the freed blocks are reused by someone else (garbage), the sequence comes
    # back into blocks at the end of the pool (grown for it)
    b.k_cache[old.long()] = float("nan")
    b.v_cache[old.long()] = float("nan")
    NB = b.k_cache.shape[0]
    grow = lambda t: torch.cat([t, torch.full((nblk,) + tuple(t.shape[1:]), float("nan"),
                                              dtype=t.dtype, device="cuda")])
    b.k_cache, b.v_cache = grow(b.k_cache), grow(b.v_cache)
    new = torch.arange(NB, NB + nblk, dtype=torch.int32, device="cuda")
    in_pairs = torch.stack([torch.arange(nblk, device="cuda"), new.long()], 1).contiguous()
    ops.pa_swap_blocks(b.k_cache, b.v_cache, hk, hv, in_pairs, ops.PA_SWAP_IN)
    b.block_tables[seq, :nblk] = new
    after = run_step(b, write=False)
    assert torch.equal(after[seq], before[seq]), "restored sequence decodes differently"


def test_swap_rejects_pageable_host_memory():
    b = W.SMALL["tiny"]("cuda")
    hk = torch.empty((2,) + tuple(b.k_cache.shape[1:]), dtype=b.k_cache.dtype)   # not pinned
    pairs = torch.tensor([[0, 0]], dtype=torch.int64, device="cuda")
    lib = ops.library()
    desc = ops.kv_cache_desc(b.k_cache, b.v_cache)
    import ctypes
    st = lib.pa_swap_blocks(ctypes.byref(desc), hk.data_ptr(), hk.data_ptr(), 2,
                            pairs.data_ptr(), 1, ops.PA_SWAP_OUT, None)
    assert st == ops.PA_ERR_INVALID_ARG
