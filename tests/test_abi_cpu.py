"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching CUDA."""

import ctypes
import re
from pathlib import Path

import pytest

from paged_kv_cache_339_b200 import build as pa_build

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "pa.h"


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    from paged_kv_cache_339_b200 import ops
    return ops.library()


def declared_functions():
    text = re.sub(r"/\*.*?\*/", "", HEADER.read_text(), flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("pa_write_kv", "pa_copy_blocks", "pa_decode"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    from paged_kv_cache_339_b200 import ops
    for code in range(7):
        assert lib.pa_status_string(code)
    assert b"sm_100a" in lib.pa_version()
    assert ops.pa_version().startswith("pagedattn")


def _cache(ops, **kw):
    d = dict(k_cache=0x10000, v_cache=0x20000, num_blocks=16, num_kv_heads=2,
             block_size=16, head_dim=128, dtype=ops.PA_BF16)
    d.update(kw)
    return ops.PaKvCache(**d)


def _decode(lib, ops, cache, **kw):
    a = dict(out=0x30000, q=0x40000, bt=0x50000, bt_stride=4, lens=0x60000, B=2, Hq=4,
             max_ctx=64, scale=0.1, split=0, path=0, share=0, ws=0x70000, ws_bytes=1 << 30)
    a.update(kw)
    opts = ops.PaDecodeOptions(a["split"], a["path"], a["share"])
    return lib.pa_decode(ctypes.byref(cache), a["out"], a["q"], a["bt"], a["bt_stride"],
                         a["lens"], a["B"], a["Hq"], a["max_ctx"], a["scale"],
                         ctypes.byref(opts), a["ws"], a["ws_bytes"], None)


def test_host_side_rejections(lib):
    """Every case below is refused by the host checks before any CUDA call;
    the pointers are never dereferenced."""
    from paged_kv_cache_339_b200 import ops
    c = _cache(ops)
    assert lib.pa_decode(None, 0, 0, 0, 1, 0, 1, 1, 1, 1.0, None, 0, 0, None) == ops.PA_ERR_INVALID_ARG
    assert _decode(lib, ops, _cache(ops, head_dim=96)) == ops.PA_ERR_UNSUPPORTED
    assert _decode(lib, ops, _cache(ops, block_size=12)) == ops.PA_ERR_UNSUPPORTED
    assert _decode(lib, ops, _cache(ops, dtype=7)) == ops.PA_ERR_UNSUPPORTED
    assert _decode(lib, ops, _cache(ops, k_cache=0x10008)) == ops.PA_ERR_MISALIGNED
    assert _decode(lib, ops, c, Hq=3) == ops.PA_ERR_INVALID_ARG            # 3 % 2 != 0
    assert _decode(lib, ops, c, Hq=64) == ops.PA_ERR_UNSUPPORTED           # group 32
    assert _decode(lib, ops, c, split=24) == ops.PA_ERR_INVALID_ARG        # not k * 16
    assert _decode(lib, ops, c, split=16, max_ctx=16 * 257, bt_stride=300) == ops.PA_ERR_INVALID_ARG
    assert _decode(lib, ops, c, max_ctx=65) == ops.PA_ERR_INVALID_ARG      # > 4 * 16
    assert _decode(lib, ops, c, scale=float("nan")) == ops.PA_ERR_INVALID_ARG
    assert _decode(lib, ops, c, path=5) == ops.PA_ERR_INVALID_ARG
    assert _decode(lib, ops, c, share=2) == ops.PA_ERR_INVALID_ARG
    assert _decode(lib, ops, c, out=0x30004) == ops.PA_ERR_MISALIGNED
    assert _decode(lib, ops, c, ws_bytes=100) == ops.PA_ERR_WORKSPACE_TOO_SMALL
    assert _decode(lib, ops, c, B=0) == ops.PA_OK                          # nothing to do
    # the plan keeps one length per sequence in shared memory: 56,320 at most
    assert _decode(lib, ops, c, B=56321) == ops.PA_ERR_UNSUPPORTED
    # 40,000 sequences x 53,688 query heads (26,844 KV heads, group 2) is past 2^31 query rows
    big = _cache(ops, num_kv_heads=26844)
    assert _decode(lib, ops, big, B=40000, Hq=53688, max_ctx=16, ws_bytes=1 << 62) == ops.PA_ERR_UNSUPPORTED
    assert lib.pa_write_kv(ctypes.byref(c), 0x1000, 0x2000, 0x3000, 0, None) == ops.PA_OK
    assert lib.pa_write_kv(ctypes.byref(c), 0x1000, 0x2000, 0x3000, -1, None) == ops.PA_ERR_INVALID_ARG
    assert lib.pa_write_kv(ctypes.byref(c), 0x1004, 0x2000, 0x3000, 3, None) == ops.PA_ERR_MISALIGNED
    assert lib.pa_write_kv(ctypes.byref(c), None, 0x2000, 0x3000, 3, None) == ops.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(ctypes.byref(c), 0x3000, 0, None) == ops.PA_OK
    assert lib.pa_copy_blocks(ctypes.byref(c), None, 2, None) == ops.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(ctypes.byref(c), 0x3004, 2, None) == ops.PA_ERR_MISALIGNED
    # swap: checked before the host pool's memory type is asked for
    sw = lib.pa_swap_blocks
    assert sw(ctypes.byref(c), 0x8000, 0x9000, 4, 0x3000, 0, 0, None) == ops.PA_OK
    assert sw(ctypes.byref(c), 0x8000, 0x9000, 4, 0x3000, 2, 2, None) == ops.PA_ERR_INVALID_ARG
    assert sw(ctypes.byref(c), 0x8000, 0x9000, -1, 0x3000, 2, 0, None) == ops.PA_ERR_INVALID_ARG
    assert sw(ctypes.byref(c), None, 0x9000, 4, 0x3000, 2, 1, None) == ops.PA_ERR_INVALID_ARG
    assert sw(ctypes.byref(c), 0x8000, 0x9000, 4, None, 2, 1, None) == ops.PA_ERR_INVALID_ARG
    assert sw(ctypes.byref(c), 0x8008, 0x9000, 4, 0x3000, 2, 1, None) == ops.PA_ERR_MISALIGNED
    assert sw(ctypes.byref(c), 0x8000, 0x9000, 4, 0x3004, 2, 1, None) == ops.PA_ERR_MISALIGNED


def test_workspace_size_layout(lib):
    """Header 256 B, then pairs, splits per sequence, the list of split
    sequences, merge counters, the group list, partial (m, l) and partial o,
    each rounded up to 256 B; split capacity from the split rule."""
    from paged_kv_cache_339_b200 import ops

    def expect(B, H, D, max_ctx, split):
        s = split if split > 0 else max(256, -(-(-(-max_ctx // 64)) // 128) * 128)
        ms = max(1, -(-max_ctx // s))
        r = lambda x: -(-x // 256) * 256
        return (256 + r(B * ms * 16) + r(B * 4) + r(B * 4) + r(B * H * 4) + r(B * ms * 16)
                + r(B * H * ms * 8) + r(B * H * ms * D * 4))

    for args in ((64, 32, 128, 2048, 0), (256, 32, 128, 4096, 0), (8, 64, 128, 131072, 0),
                 (4, 1, 64, 33, 16), (3, 8, 128, 1000, 32)):
        got = ops.pa_decode_workspace_size(args[0], args[1], args[2], args[3], 16, args[4])
        assert got == expect(*args), args


def test_noalloc_checks_arguments_before_its_scratch_size(lib):
    """pa_decode_noalloc runs pa_decode's argument checks first and compares
    the fixed scratch size last; neither touches CUDA."""
    from paged_kv_cache_339_b200 import ops
    c = _cache(ops)

    def noalloc(cache, B=2, Hq=4, max_ctx=64, bt_stride=4, split=0):
        opts = ops.PaDecodeOptions(split, 0)
        return lib.pa_decode_noalloc(ctypes.byref(cache), 0x30000, 0x40000, 0x50000, bt_stride,
                                     0x60000, B, Hq, max_ctx, 0.1, ctypes.byref(opts), None)

    assert noalloc(c, Hq=3) == ops.PA_ERR_INVALID_ARG                  # 3 % 2 != 0
    assert noalloc(_cache(ops, head_dim=96)) == ops.PA_ERR_UNSUPPORTED
    assert noalloc(c, split=24) == ops.PA_ERR_INVALID_ARG              # not k * 16
    assert noalloc(c, B=0) == ops.PA_OK
    # 4096 sequences x 64 heads (group 32 is refused first) ...
    assert noalloc(_cache(ops, num_kv_heads=2), B=4096, Hq=64, max_ctx=65536,
                   bt_stride=4096) == ops.PA_ERR_UNSUPPORTED
    # ... while a valid shape that needs more than the 32 MiB scratch is refused as such
    big = _cache(ops, num_kv_heads=8)
    assert noalloc(big, B=4096, Hq=64, max_ctx=65536, bt_stride=4096) == \
        ops.PA_ERR_WORKSPACE_TOO_SMALL


def test_device_timeout_status_is_reported(lib):
    """A kernel that gave up waiting is reported by name, through the status
    string and the binding's exception."""
    from paged_kv_cache_339_b200 import ops
    assert b"PA_ERR_DEVICE_TIMEOUT" in lib.pa_status_string(ops.PA_ERR_DEVICE_TIMEOUT)
    e = ops.PagedAttnError("pa_decode", ops.PA_ERR_DEVICE_TIMEOUT)
    assert e.status == ops.PA_ERR_DEVICE_TIMEOUT and "gave up waiting" in str(e)
