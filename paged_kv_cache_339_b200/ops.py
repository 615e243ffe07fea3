"""Python binding of libpagedattn.so: the C-ABI calls of include/pa.h with the
same names, taking torch tensors. Argument marshalling only: every step runs in
the library's CUDA kernels; there is no CPU or PyTorch fallback, and a missing
library is an error.
"""

from __future__ import annotations

import ctypes
from pathlib import Path
from typing import Optional

import torch

_LIB_PATH = Path(__file__).resolve().parent / "libpagedattn.so"

PA_F32, PA_F16, PA_BF16 = 0, 1, 2
PA_PATH_AUTO, PA_PATH_SIMT, PA_PATH_TCGEN05 = 0, 1, 2
PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_MISALIGNED = 0, 1, 2, 3
PA_ERR_WORKSPACE_TOO_SMALL, PA_ERR_CUDA, PA_ERR_DEVICE_TIMEOUT = 4, 5, 6

_DTYPE_CODE = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}


class PaKvCache(ctypes.Structure):
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("num_blocks", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int)]


class PaDecodeOptions(ctypes.Structure):
    _fields_ = [("split_tokens", ctypes.c_int32), ("path", ctypes.c_int32),
                ("share_prefixes", ctypes.c_int32)]


class PagedAttnError(RuntimeError):
    def __init__(self, call: str, status: int):
        lib = _load()
        msg = lib.pa_status_string(status).decode()
        if status == PA_ERR_CUDA:
            msg += " (" + lib.pa_last_cuda_error().decode() + ")"
        super().__init__(f"{call}: {msg}")
        self.status = status


_lib = None

EXPORTS = ("pa_write_kv", "pa_copy_blocks", "pa_swap_blocks", "pa_decode_workspace_size",
           "pa_decode",
           "pa_decode_noalloc", "pa_decode_noalloc_status", "pa_decode_status",
           "pa_status_string", "pa_last_cuda_error", "pa_version")


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not _LIB_PATH.exists():
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with "
            "`python -m paged_kv_cache_339_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(str(_LIB_PATH))
    vp, i32, i64p = ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p
    lib.pa_write_kv.argtypes = [ctypes.POINTER(PaKvCache), vp, vp, i64p, i32, vp]
    lib.pa_write_kv.restype = ctypes.c_int
    lib.pa_copy_blocks.argtypes = [ctypes.POINTER(PaKvCache), i64p, i32, vp]
    lib.pa_copy_blocks.restype = ctypes.c_int
    lib.pa_swap_blocks.argtypes = [ctypes.POINTER(PaKvCache), vp, vp, i32, i64p, i32, i32, vp]
    lib.pa_swap_blocks.restype = ctypes.c_int
    lib.pa_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.pa_decode_workspace_size.restype = ctypes.c_size_t
    lib.pa_decode.argtypes = [ctypes.POINTER(PaKvCache), vp, vp, vp, i32, vp, i32, i32, i32,
                              ctypes.c_float, ctypes.POINTER(PaDecodeOptions), vp,
                              ctypes.c_size_t, vp]
    lib.pa_decode.restype = ctypes.c_int
    lib.pa_decode_noalloc.argtypes = [ctypes.POINTER(PaKvCache), vp, vp, vp, i32, vp, i32, i32,
                                      i32, ctypes.c_float, ctypes.POINTER(PaDecodeOptions), vp]
    lib.pa_decode_noalloc.restype = ctypes.c_int
    lib.pa_decode_status.argtypes = [vp, vp]
    lib.pa_decode_status.restype = ctypes.c_int
    lib.pa_decode_noalloc_status.argtypes = [vp]
    lib.pa_decode_noalloc_status.restype = ctypes.c_int
    lib.pa_status_string.argtypes = [ctypes.c_int]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_last_cuda_error.argtypes = []
    lib.pa_last_cuda_error.restype = ctypes.c_char_p
    lib.pa_version.argtypes = []
    lib.pa_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def library():
    """The loaded ctypes library (raises ImportError if it was not built)."""
    return _load()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev_tensor(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def kv_cache_desc(k_cache: torch.Tensor, v_cache: torch.Tensor) -> PaKvCache:
    """Describe pools of shape [num_blocks, num_kv_heads, block_size, head_dim]."""
    if k_cache.shape != v_cache.shape or k_cache.dtype != v_cache.dtype or k_cache.dim() != 4:
        raise ValueError("k_cache and v_cache must have the same 4-D shape and dtype")
    if k_cache.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported cache dtype {k_cache.dtype}")
    nb, hkv, bs, d = k_cache.shape
    return PaKvCache(_dev_tensor(k_cache, "k_cache"), _dev_tensor(v_cache, "v_cache"),
                     nb, hkv, bs, d, _DTYPE_CODE[k_cache.dtype])


def _check(call: str, status: int):
    if status != PA_OK:
        raise PagedAttnError(call, status)


def pa_write_kv(k_cache, v_cache, key, value, slot_mapping, stream=None) -> None:
    """Store key/value [T, Hkv, D] into slots slot_mapping (int64 [T]); slot < 0
    skips the token."""
    desc = kv_cache_desc(k_cache, v_cache)
    T = key.shape[0]
    if key.shape != (T,) + tuple(k_cache.shape[1:2]) + tuple(k_cache.shape[3:]):
        raise ValueError("key must be [num_tokens, num_kv_heads, head_dim]")
    if value.shape != key.shape or slot_mapping.shape != (T,):
        raise ValueError("value / slot_mapping shape mismatch")
    st = _load().pa_write_kv(ctypes.byref(desc), _dev_tensor(key, "key", k_cache.dtype),
                             _dev_tensor(value, "value", k_cache.dtype),
                             _dev_tensor(slot_mapping, "slot_mapping", torch.int64), T,
                             _stream(stream))
    _check("pa_write_kv", st)


def pa_copy_blocks(k_cache, v_cache, block_pairs, stream=None) -> None:
    """Copy block src -> dst of both pools for every (src, dst) row of the
    int64 [P, 2] tensor block_pairs."""
    desc = kv_cache_desc(k_cache, v_cache)
    P = block_pairs.shape[0] if block_pairs.numel() else 0
    if P and tuple(block_pairs.shape) != (P, 2):
        raise ValueError("block_pairs must be [num_pairs, 2]")
    ptr = _dev_tensor(block_pairs, "block_pairs", torch.int64) if P else None
    st = _load().pa_copy_blocks(ctypes.byref(desc), ptr, P, _stream(stream))
    _check("pa_copy_blocks", st)


PA_SWAP_OUT, PA_SWAP_IN = 0, 1


def pa_swap_blocks(k_cache, v_cache, host_k, host_v, block_pairs, direction, stream=None) -> None:
    """Move blocks between the device pools and a pinned host pool (host_k,
    host_v: pinned CPU tensors shaped like the pools, any number of blocks).
    PA_SWAP_OUT: host[dst] = device[src]; PA_SWAP_IN: device[dst] = host[src],
    for every (src, dst) row of the int64 [P, 2] device tensor block_pairs."""
    desc = kv_cache_desc(k_cache, v_cache)
    for name, t in (("host_k", host_k), ("host_v", host_v)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_pinned():
            raise TypeError(f"{name} must be a pinned CPU tensor")
        if not t.is_contiguous() or t.dtype != k_cache.dtype or t.shape[1:] != k_cache.shape[1:]:
            raise ValueError(f"{name} must be contiguous [blocks, {', '.join(map(str, k_cache.shape[1:]))}] "
                             f"{k_cache.dtype}")
    if host_k.shape != host_v.shape:
        raise ValueError("host_k and host_v must have the same shape")
    P = block_pairs.shape[0] if block_pairs.numel() else 0
    if P and tuple(block_pairs.shape) != (P, 2):
        raise ValueError("block_pairs must be [num_pairs, 2]")
    ptr = _dev_tensor(block_pairs, "block_pairs", torch.int64) if P else None
    st = _load().pa_swap_blocks(ctypes.byref(desc), host_k.data_ptr(), host_v.data_ptr(),
                                host_k.shape[0], ptr, P, int(direction), _stream(stream))
    _check("pa_swap_blocks", st)


def pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, block_size,
                             split_tokens=0) -> int:
    return int(_load().pa_decode_workspace_size(num_seqs, num_q_heads, head_dim,
                                                max_context_len, block_size, split_tokens))


def decode_workspace(num_seqs, num_q_heads, head_dim, max_context_len, block_size,
                     split_tokens=0, device="cuda") -> torch.Tensor:
    """Allocate (through torch) a workspace of the size pa_decode needs."""
    n = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, block_size,
                                 split_tokens)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
              workspace, split_tokens=0, path=PA_PATH_AUTO, stream=None,
              share_prefixes=False) -> torch.Tensor:
    """out[i, h] = softmax(scale * q[i, h] . K_i^T) . V_i over context_lens[i]
    tokens reached through block_tables[i]; out is fp32 [B, Hq, D]."""
    desc = kv_cache_desc(k_cache, v_cache)
    B, Hq, D = q.shape
    if out.shape != (B, Hq, D) or out.dtype != torch.float32:
        raise ValueError("out must be fp32 [num_seqs, num_q_heads, head_dim]")
    if D != k_cache.shape[3] or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("shape mismatch between q, caches and block_tables")
    if context_lens.shape != (B,):
        raise ValueError("context_lens must be [num_seqs]")
    opts = PaDecodeOptions(int(split_tokens), int(path), int(bool(share_prefixes)))
    st = _load().pa_decode(
        ctypes.byref(desc), _dev_tensor(out, "out", torch.float32),
        _dev_tensor(q, "q", k_cache.dtype), _dev_tensor(block_tables, "block_tables", torch.int32),
        int(block_tables.shape[1]), _dev_tensor(context_lens, "context_lens", torch.int32), B, Hq,
        int(max_context_len), float(scale), ctypes.byref(opts),
        _dev_tensor(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("pa_decode", st)
    return out


def pa_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len,
                      scale, split_tokens=0, path=PA_PATH_AUTO, stream=None,
                      share_prefixes=False) -> torch.Tensor:
    """pa_decode with the library's fixed 32 MiB device scratch instead of a
    workspace, for callers that cannot allocate device memory (see
    include/pa.h). Calls must not overlap on the GPU."""
    desc = kv_cache_desc(k_cache, v_cache)
    B, Hq, D = q.shape
    if out.shape != (B, Hq, D) or out.dtype != torch.float32:
        raise ValueError("out must be fp32 [num_seqs, num_q_heads, head_dim]")
    if D != k_cache.shape[3] or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("shape mismatch between q, caches and block_tables")
    if context_lens.shape != (B,):
        raise ValueError("context_lens must be [num_seqs]")
    opts = PaDecodeOptions(int(split_tokens), int(path), int(bool(share_prefixes)))
    st = _load().pa_decode_noalloc(
        ctypes.byref(desc), _dev_tensor(out, "out", torch.float32),
        _dev_tensor(q, "q", k_cache.dtype), _dev_tensor(block_tables, "block_tables", torch.int32),
        int(block_tables.shape[1]), _dev_tensor(context_lens, "context_lens", torch.int32), B, Hq,
        int(max_context_len), float(scale), ctypes.byref(opts), _stream(stream))
    _check("pa_decode_noalloc", st)
    return out


def pa_decode_status(workspace, stream=None) -> int:
    """Device status word of the last pa_decode on this workspace (synchronises)."""
    return int(_load().pa_decode_status(_dev_tensor(workspace, "workspace"), _stream(stream)))


def pa_decode_noalloc_status(stream=None) -> int:
    """Device status word of the last pa_decode_noalloc on the current device
    (synchronises)."""
    return int(_load().pa_decode_noalloc_status(_stream(stream)))


def pa_version() -> str:
    return _load().pa_version().decode()
