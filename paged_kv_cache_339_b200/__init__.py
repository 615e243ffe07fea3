"""B200-native paged KV-cache decode: C-ABI library (libpagedattn.so) with
hand-written sm_100a kernels for the KV write, the copy-on-write block copy and
paged decode attention, plus host-side block bookkeeping."""

from .block_manager import BlockManager, OutOfBlocks  # noqa: F401

__all__ = ["BlockManager", "OutOfBlocks"]
