"""Thin ctypes binding of libpa.so (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
computation of its own: it reads shapes off the tensors, checks that they are
contiguous CUDA tensors of the right dtype, and passes raw device pointers and
the current CUDA stream to the library.  There is no fallback: if the CUDA
library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_388_b200.build` "
        "(nvcc, sm_100a).  There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

P = ctypes.c_void_p
I = ctypes.c_int
F = ctypes.c_float
SZ = ctypes.c_size_t

_lib.pa_reshape_and_cache.restype = I
_lib.pa_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P]
_lib.pa_copy_blocks.restype = I
_lib.pa_copy_blocks.argtypes = [P, P, P, I, I, I, I, I, I, P]
_lib.pa_reshape_and_cache_fp8.restype = I
_lib.pa_reshape_and_cache_fp8.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, F, P]
_lib.pa_decode_fp8.restype = I
_lib.pa_decode_fp8.argtypes = [P, P, P, P, P, I, P, I, I, I, I, I, I, F, F, F, I, I, P, SZ, P]
_lib.pa_decode_fp8_rows.restype = I
_lib.pa_decode_fp8_rows.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, I, I, I, F, F, F, I, I, I,
                                    P, SZ, P]
_lib.pa_decode_fp8_rows_workspace_size.restype = SZ
_lib.pa_decode_fp8_rows_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
_lib.pa_swap_blocks.restype = I
_lib.pa_swap_blocks.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P]
_lib.pa_decode_workspace_size.restype = SZ
_lib.pa_decode_workspace_size.argtypes = [I, I, I, I, I, I, I]
_lib.pa_decode.restype = I
_lib.pa_decode.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, I, I, I, F, I, I, I, P, SZ, P]
_lib.pa_decode_noalloc.restype = I
_lib.pa_decode_noalloc.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, I, I, I, F, I, I, I, P]
_lib.pa_decode_shared_prefix.restype = I
_lib.pa_decode_shared_prefix.argtypes = [P, P, P, P, P, I, P, I, P, P, I, I, I, I, I, I, I, F, I, I,
                                         P, SZ, P]
_lib.pa_decode_shared_prefix_workspace_size.restype = SZ
_lib.pa_decode_shared_prefix_workspace_size.argtypes = [I, I, I, I, I, I]
_lib.pa_decode_shared_prefix_fp8.restype = I
_lib.pa_decode_shared_prefix_fp8.argtypes = [P, P, P, P, P, I, P, I, P, P, I, I, I, I, I, I, I, F,
                                             F, F, I, I, I, P, SZ, P]
_lib.pa_decode_shared_prefix_fp8_workspace_size.restype = SZ
_lib.pa_decode_shared_prefix_fp8_workspace_size.argtypes = [I, I, I, I, I, I, I, I, I]
_lib.pa_noalloc_scratch_bytes.restype = SZ
_lib.pa_noalloc_scratch_bytes.argtypes = []
_lib.pa_get_device_error.restype = I
_lib.pa_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), P]
_lib.pa_status_string.restype = ctypes.c_char_p
_lib.pa_status_string.argtypes = [I]
_lib.pa_abi_version.restype = I
_lib.pa_abi_version.argtypes = []

PA_F32, PA_F16, PA_BF16, PA_FP8_E4M3 = 0, 1, 2, 3
_DT = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16,
       torch.uint8: PA_FP8_E4M3, torch.float8_e4m3fn: PA_FP8_E4M3}

PA_DEVERR_BLOCK_ID = 0x1
PA_DEVERR_SLOT = 0x2
PA_DEVERR_CONTEXT_LEN = 0x4
PA_DEVERR_QUERY_LEN = 0x8
PA_DEVERR_TIMEOUT = 0x10
PA_DEVERR_PREFIX = 0x20
PA_DEVERR_STAGING = 0x40


class PAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_lib.pa_status_string(status).decode()} ({status})")


def library():
    """The loaded ctypes library (for tests that call entry points directly)."""
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name, dtype=None):
    """A contiguous CUDA tensor on the current device (the library launches on
    the current device and would otherwise dereference another GPU's memory)."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name} is on {t.device} but the current device is cuda:{cur}; "
                         "call under torch.cuda.device(...) of the tensors' device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _shape(cond, what):
    if not cond:
        raise ValueError(what)


def _cache_shapes(k_cache, v_cache):
    """(num_blocks, num_kv_heads, block_size, head_dim) of a pair of caches."""
    _shape(k_cache.dim() == 4, "k_cache must be [num_blocks, num_kv_heads, block_size, head_dim]")
    _shape(tuple(v_cache.shape) == tuple(k_cache.shape), "k_cache and v_cache shapes disagree")
    return tuple(k_cache.shape)


def _new_token_shapes(key, value, k_cache, v_cache, slot_mapping):
    nb, hk, bs, d = _cache_shapes(k_cache, v_cache)
    _shape(key.dim() == 3 and tuple(key.shape[1:]) == (hk, d),
           f"key must be [num_tokens, {hk}, {d}] to match the caches, got {tuple(key.shape)}")
    _shape(tuple(value.shape) == tuple(key.shape), "key and value shapes disagree")
    _shape(slot_mapping.dim() == 1 and slot_mapping.shape[0] == key.shape[0],
           "slot_mapping must hold one slot per key/value token")
    return nb, hk, bs, d


def _decode_shapes(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc=None):
    """Shapes of a decode call; every tensor must agree with the others."""
    nb, hk, bs, d = _cache_shapes(k_cache, v_cache)
    _shape(q.dim() == 3 and q.shape[2] == d, f"q must be [tokens, heads, {d}] to match the caches")
    _shape(tuple(out.shape) == tuple(q.shape), "out and q shapes disagree")
    tq, h, _ = q.shape
    _shape(h % hk == 0, "num_heads must be a multiple of num_kv_heads")
    _shape(block_tables.dim() == 2, "block_tables must be [num_seqs, max_blocks_per_seq]")
    s, mbps = block_tables.shape
    _shape(context_lens.dim() == 1 and context_lens.shape[0] == s,
           "block_tables and context_lens disagree on the number of sequences")
    if query_start_loc is None:
        _shape(tq == s, "without query_start_loc q must hold one row per sequence")
    else:
        _shape(query_start_loc.dim() == 1 and query_start_loc.shape[0] == s + 1,
               "query_start_loc must have num_seqs + 1 entries")
    return tq, h, d, nb, hk, bs, s, mbps


def _check(rc, what):
    if rc != 0:
        raise PAError(rc, what)


def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None):
    """key/value [T, Hk, D]; caches [NB, Hk, bs, D]; slot_mapping int64 [T]."""
    nb, hk, bs, d = _new_token_shapes(key, value, k_cache, v_cache, slot_mapping)
    _dev(key, "key")
    _dev(value, "value", key.dtype)
    _dev(k_cache, "k_cache", key.dtype)
    _dev(v_cache, "v_cache", key.dtype)
    _dev(slot_mapping, "slot_mapping", torch.int64)
    rc = _lib.pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                   _ptr(slot_mapping), key.shape[0], hk, d, bs, nb,
                                   _DT[key.dtype], _stream(stream))
    _check(rc, "pa_reshape_and_cache")


def pa_copy_blocks(k_cache, v_cache, block_mapping, stream=None):
    """block_mapping int64 [P, 2] of (src, dst) physical block ids."""
    nb, hk, bs, d = _cache_shapes(k_cache, v_cache)
    _shape(block_mapping.dim() == 2 and block_mapping.shape[1] == 2,
           "block_mapping must be [num_pairs, 2]")
    _dev(k_cache, "k_cache")
    _dev(v_cache, "v_cache", k_cache.dtype)
    _dev(block_mapping, "block_mapping", torch.int64)
    rc = _lib.pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_mapping),
                             block_mapping.shape[0], hk, d, bs, nb, _DT[k_cache.dtype],
                             _stream(stream))
    _check(rc, "pa_copy_blocks")


def pa_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                             stream=None):
    """key/value [T, Hk, D] (fp32/fp16/bf16); caches uint8 [NB, Hk, bs, D] of
    E4M3 codes; slot_mapping int64 [T]."""
    nb, hk, bs, d = _new_token_shapes(key, value, k_cache, v_cache, slot_mapping)
    _dev(key, "key")
    _dev(value, "value", key.dtype)
    _dev(k_cache, "k_cache", torch.uint8)
    _dev(v_cache, "v_cache", torch.uint8)
    _dev(slot_mapping, "slot_mapping", torch.int64)
    rc = _lib.pa_reshape_and_cache_fp8(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(slot_mapping), key.shape[0], hk, d, bs, nb,
                                       _DT[key.dtype], float(k_scale), float(v_scale),
                                       _stream(stream))
    _check(rc, "pa_reshape_and_cache_fp8")


def pa_decode_fp8_rows_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                      max_context_len, max_blocks_per_seq, staged_blocks) -> int:
    return int(_lib.pa_decode_fp8_rows_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim,
                                                      block_size, max_context_len,
                                                      max_blocks_per_seq, staged_blocks))


def pa_decode_fp8(out, q, k_cache, v_cache, block_tables, context_lens, scale, k_scale, v_scale,
                  max_context_len=0, workspace=None, query_start_loc=None, max_query_len=1,
                  staged_blocks=0, stream=None):
    """out/q [S, H, D] fp16/bf16; caches uint8 E4M3 codes [NB, Hk, bs, D];
    workspace: uint8 CUDA tensor of >= pa_decode_workspace_size(...) bytes.
    With query_start_loc (chunked-prefill rows as in pa_decode) the call is
    pa_decode_fp8_rows: staged_blocks bounds the blocks of the sequences with
    more than one row (batch.staged_blocks_needed), and the workspace must hold
    pa_decode_fp8_rows_workspace_size(...) bytes."""
    tq, h, d, nb, hk, bs, s, mbps = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                                   context_lens, query_start_loc)
    if query_start_loc is not None:
        _dev(query_start_loc, "query_start_loc", torch.int32)
    _dev(q, "q")
    _dev(out, "out", q.dtype)
    _dev(k_cache, "k_cache", torch.uint8)
    _dev(v_cache, "v_cache", torch.uint8)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    if workspace is not None:
        _dev(workspace, "workspace")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if query_start_loc is not None:
        pa_decode_fp8_rows(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                           scale, k_scale, v_scale, max_query_len, staged_blocks,
                           max_context_len=max_context_len, workspace=workspace, stream=stream)
        return
    rc = _lib.pa_decode_fp8(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                            mbps, _ptr(context_lens), s, h, hk, d, bs, nb, float(scale),
                            float(k_scale), float(v_scale), int(max_context_len), _DT[q.dtype],
                            _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "pa_decode_fp8")


def pa_decode_fp8_rows(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                       scale, k_scale, v_scale, max_query_len, staged_blocks, max_context_len=0,
                       workspace=None, stream=None):
    """pa_decode_fp8 over a batch with chunked-prefill rows: q/out [Tq, H, D],
    query_start_loc int32 [S + 1]; staged_blocks bounds the blocks of the
    sequences with more than one row; workspace uint8 of
    >= pa_decode_fp8_rows_workspace_size(...) bytes."""
    tq, h, d, nb, hk, bs, s, mbps = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                                   context_lens, query_start_loc)
    _dev(q, "q")
    _dev(out, "out", q.dtype)
    _dev(k_cache, "k_cache", torch.uint8)
    _dev(v_cache, "v_cache", torch.uint8)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    _dev(query_start_loc, "query_start_loc", torch.int32)
    if workspace is not None:
        _dev(workspace, "workspace")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib.pa_decode_fp8_rows(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(block_tables), mbps, _ptr(context_lens),
                                 _ptr(query_start_loc), s, tq, int(max_query_len), h, hk, d, bs,
                                 nb, float(scale), float(k_scale), float(v_scale),
                                 int(max_context_len), int(staged_blocks), _DT[q.dtype],
                                 _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "pa_decode_fp8_rows")


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, block_mapping, stream=None):
    """Copy blocks (src, dst) of block_mapping int64 [P, 2] from the
    (src_k, src_v) pool into the (dst_k, dst_v) pool.  Pools and mapping may
    be CUDA tensors or pinned CPU tensors (not pageable ones)."""
    for name, t in (("dst_k", dst_k), ("dst_v", dst_v), ("src_k", src_k), ("src_v", src_v),
                    ("block_mapping", block_mapping)):
        if t.is_cuda:
            _dev(t, name)
        elif not t.is_pinned():
            raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if block_mapping.dtype != torch.int64:
        raise ValueError("block_mapping must be int64")
    if not (dst_k.dtype == dst_v.dtype == src_k.dtype == src_v.dtype):
        raise ValueError("pools must share one dtype")
    nd, hk, bs, d = dst_k.shape
    ns = src_k.shape[0]
    if tuple(src_k.shape[1:]) != (hk, bs, d) or src_v.shape != src_k.shape or dst_v.shape != dst_k.shape:
        raise ValueError("pool shapes disagree")
    rc = _lib.pa_swap_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(src_k), _ptr(src_v),
                             _ptr(block_mapping), block_mapping.shape[0], hk, d, bs, ns, nd,
                             _DT[dst_k.dtype], _stream(stream))
    _check(rc, "pa_swap_blocks")


def pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                             max_context_len, kv_split_tokens=0) -> int:
    return int(_lib.pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim,
                                             block_size, max_context_len, kv_split_tokens))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale,
              query_start_loc=None, max_query_len=1, max_context_len=0, kv_split_tokens=0,
              workspace=None, stream=None):
    """out/q [Tq, H, D]; caches [NB, Hk, bs, D]; block_tables int32 [S, mbps];
    context_lens int32 [S]; query_start_loc int32 [S+1] or None; workspace: a
    uint8 CUDA tensor of >= pa_decode_workspace_size(...) bytes (or None when
    that size is 0)."""
    tq, h, d, nb, hk, bs, s, mbps = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                                   context_lens, query_start_loc)
    _dev(q, "q")
    _dev(out, "out", q.dtype)
    _dev(k_cache, "k_cache", q.dtype)
    _dev(v_cache, "v_cache", q.dtype)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    if query_start_loc is not None:
        _dev(query_start_loc, "query_start_loc", torch.int32)
    if workspace is not None:
        _dev(workspace, "workspace")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib.pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                        mbps, _ptr(context_lens), _ptr(query_start_loc), s, tq,
                        int(max_query_len), h, hk, d, bs, nb, float(scale), int(max_context_len),
                        int(kv_split_tokens), _DT[q.dtype], _ptr(workspace), ws_bytes,
                        _stream(stream))
    _check(rc, "pa_decode")


def pa_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                      query_start_loc=None, max_query_len=1, max_context_len=0, kv_split_tokens=0,
                      stream=None):
    """pa_decode with the library's static scratch instead of a workspace, for
    callers that cannot allocate device memory.  Calls must not overlap on
    the GPU (they share the scratch); make the first call on a device before
    any stream capture."""
    tq, h, d, nb, hk, bs, s, mbps = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                                   context_lens, query_start_loc)
    _dev(q, "q")
    _dev(out, "out", q.dtype)
    _dev(k_cache, "k_cache", q.dtype)
    _dev(v_cache, "v_cache", q.dtype)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    if query_start_loc is not None:
        _dev(query_start_loc, "query_start_loc", torch.int32)
    rc = _lib.pa_decode_noalloc(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                _ptr(block_tables), mbps, _ptr(context_lens), _ptr(query_start_loc),
                                s, tq, int(max_query_len), h, hk, d, bs, nb, float(scale),
                                int(max_context_len), int(kv_split_tokens), _DT[q.dtype],
                                _stream(stream))
    _check(rc, "pa_decode_noalloc")


def pa_decode_shared_prefix_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                           max_context_len) -> int:
    return int(_lib.pa_decode_shared_prefix_workspace_size(num_seqs, num_heads, num_kv_heads,
                                                           head_dim, block_size, max_context_len))


def pa_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, context_lens, group_start,
                            group_shared_blocks, scale, max_group_size=0, max_context_len=0,
                            workspace=None, stream=None):
    """Decode with shared-prefix groups.  out/q [S, H, D]; group_start int32
    [G+1] and group_shared_blocks int32 [G] on the device; workspace: uint8
    CUDA tensor of >= pa_decode_shared_prefix_workspace_size(...) bytes."""
    s, h, d, nb, hk, bs, _, mbps = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                                  context_lens)
    _shape(group_start.dim() == 1 and group_shared_blocks.dim() == 1 and
           group_start.shape[0] == group_shared_blocks.shape[0] + 1,
           "group_start must have one more entry than group_shared_blocks")
    _dev(q, "q")
    _dev(out, "out", q.dtype)
    _dev(k_cache, "k_cache", q.dtype)
    _dev(v_cache, "v_cache", q.dtype)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    _dev(group_start, "group_start", torch.int32)
    _dev(group_shared_blocks, "group_shared_blocks", torch.int32)
    if workspace is not None:
        _dev(workspace, "workspace")
    g = group_shared_blocks.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib.pa_decode_shared_prefix(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(block_tables), mbps, _ptr(context_lens), s,
                                      _ptr(group_start), _ptr(group_shared_blocks), g,
                                      int(max_group_size), h, hk, d, bs, nb, float(scale),
                                      int(max_context_len), _DT[q.dtype], _ptr(workspace),
                                      ws_bytes, _stream(stream))
    _check(rc, "pa_decode_shared_prefix")


def pa_decode_shared_prefix_fp8_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim,
                                               block_size, max_context_len, max_blocks_per_seq,
                                               num_groups, staged_blocks) -> int:
    return int(_lib.pa_decode_shared_prefix_fp8_workspace_size(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
        max_blocks_per_seq, num_groups, staged_blocks))


def pa_decode_shared_prefix_fp8(out, q, k_cache, v_cache, block_tables, context_lens, group_start,
                                group_shared_blocks, scale, k_scale, v_scale, staged_blocks,
                                max_group_size=0, max_context_len=0, workspace=None, stream=None):
    """pa_decode_shared_prefix over FP8 (E4M3) caches (uint8 codes); out/q
    fp16/bf16 [S, H, D]; staged_blocks bounds the groups' shared blocks
    (their sum); workspace uint8 of
    >= pa_decode_shared_prefix_fp8_workspace_size(...) bytes."""
    s, h, d, nb, hk, bs, _, mbps = _decode_shapes(out, q, k_cache, v_cache, block_tables,
                                                  context_lens)
    _shape(group_start.dim() == 1 and group_shared_blocks.dim() == 1 and
           group_start.shape[0] == group_shared_blocks.shape[0] + 1,
           "group_start must have one more entry than group_shared_blocks")
    _dev(q, "q")
    _dev(out, "out", q.dtype)
    _dev(k_cache, "k_cache", torch.uint8)
    _dev(v_cache, "v_cache", torch.uint8)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    _dev(group_start, "group_start", torch.int32)
    _dev(group_shared_blocks, "group_shared_blocks", torch.int32)
    if workspace is not None:
        _dev(workspace, "workspace")
    g = group_shared_blocks.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib.pa_decode_shared_prefix_fp8(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(block_tables), mbps, _ptr(context_lens), s,
                                          _ptr(group_start), _ptr(group_shared_blocks), g,
                                          int(max_group_size), h, hk, d, bs, nb, float(scale),
                                          float(k_scale), float(v_scale), int(max_context_len),
                                          int(staged_blocks), _DT[q.dtype], _ptr(workspace),
                                          ws_bytes, _stream(stream))
    _check(rc, "pa_decode_shared_prefix_fp8")


def pa_noalloc_scratch_bytes() -> int:
    return int(_lib.pa_noalloc_scratch_bytes())


def pa_get_device_error(stream=None) -> int:
    """Synchronise the stream, return and clear the device error word."""
    code = ctypes.c_uint(0)
    rc = _lib.pa_get_device_error(ctypes.byref(code), _stream(stream))
    _check(rc, "pa_get_device_error")
    return int(code.value)


def pa_abi_version() -> int:
    return int(_lib.pa_abi_version())
