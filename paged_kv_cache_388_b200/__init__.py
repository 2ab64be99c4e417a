"""B200-native paged KV-cache attention (PagedAttention decode).

The compute path is the C-ABI library ``libpa.so`` (hand-written sm_100a CUDA
kernels) reached through the thin ctypes binding in ``_lib``; the host block
allocator builds its inputs.
"""
from .allocator import BlockAllocator, PoolExhausted  # noqa: F401
