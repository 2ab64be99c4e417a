"""CPU oracle for paged KV-cache attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product package never imports it and it never imports the product package;
the two share nothing but the seeded input generators in ``workloads/``.

Contents
--------
``pa_oracle.c``   plain C, fp64, OpenMP over (query row, head): paged
                  attention, reshape_and_cache, copy_blocks, swap_blocks, and the
                  FP8 (E4M3) codec with quantising reshape and FP8-cache decode.
``brute.py``      NumPy attention over *contiguous* per-sequence K/V, for tiny
                  inputs (pins the paged gather).
``alloc_model.py`` the block-allocation rules written as plain definitions.

Every function is pinned by ``tests/test_oracle*.py`` against things other
than itself: the pages' worked examples (``tests/golden/``), closed forms,
invariants and brute force.  Nothing here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_SO = os.path.join(_HERE, "_pa_oracle.so")
_lock = threading.Lock()
_lib = None

DTYPES = {"f32": 0, "f16": 1, "bf16": 2, "fp8": 3}  # "fp8": E4M3 codes, for the byte movers
_STATUS = {
    0: "ok",
    1: "bad argument",
    2: "block id out of range",
    3: "bad context/query length",
    4: "slot out of range",
    5: "out of memory",
}


def build(src: str = _SRC, out: str = _SO, force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-Wall",
           "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _bind(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.oracle_decode.restype = I
    lib.oracle_decode.argtypes = [P, P, P, P, I, P, I, P, P, I, I, I, I, I, I,
                                  ctypes.c_double, P, I]
    lib.oracle_reshape_and_cache.restype = I
    lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I, I]
    lib.oracle_copy_blocks.restype = I
    lib.oracle_copy_blocks.argtypes = [P, P, P, I, I, I, I, I, I]
    lib.oracle_swap_blocks.restype = I
    lib.oracle_swap_blocks.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_reshape_and_cache_fp8.restype = I
    lib.oracle_reshape_and_cache_fp8.argtypes = [P, P, P, P, I, P, I, I, I, I, I,
                                                 ctypes.c_float, ctypes.c_float]
    lib.oracle_decode_fp8.restype = I
    lib.oracle_decode_fp8.argtypes = [P, P, I, P, P, ctypes.c_double, ctypes.c_double, P, I, P,
                                      P, I, I, I, I, I, I, ctypes.c_double, P, I]
    lib.oracle_max_threads.restype = I
    lib.oracle_max_threads.argtypes = []
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt=None):
    if a is None:
        return None
    a = np.asarray(a)
    if dt is not None and a.dtype != dt:
        a = a.astype(dt)
    return np.ascontiguousarray(a)


def _raw(a):
    """Value arrays: float32 / float16 as-is; bf16 as uint16 bit patterns."""
    a = np.ascontiguousarray(a)
    assert a.dtype in (np.float32, np.float16, np.uint16), a.dtype
    return a


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what}: {_STATUS.get(rc, rc)}")


def decode(q, k_cache, v_cache, block_tables, context_lens, scale, dtype,
           query_start_loc=None, rows=None, threads=0, lib=None):
    """Paged attention in fp64.

    q: [Tq, H, D]; caches: [NB, Hk, bs, D] (dtype 'f32'|'f16'|'bf16'; bf16 is
    passed as uint16 bit patterns); block_tables int32 [S, max_blocks];
    context_lens int32 [S]; query_start_loc int32 [S+1] or None.  ``rows``:
    optional iterable of query-row indices to compute (others stay NaN).
    Returns float64 [Tq, H, D].
    """
    lib = lib or load()
    q = _raw(q)
    k_cache = _raw(k_cache)
    v_cache = _raw(v_cache)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    qsl = _c(query_start_loc, np.int32)
    tq, h, d = q.shape
    nb, hk, bs, d2 = k_cache.shape
    assert d2 == d and v_cache.shape == k_cache.shape
    s = cl.shape[0]
    out = np.full((tq, h, d), np.nan, dtype=np.float64)
    sel = None
    if rows is not None:
        sel = np.zeros(tq, dtype=np.uint8)
        sel[np.asarray(list(rows), dtype=np.int64)] = 1
    rc = lib.oracle_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                           DTYPES[dtype], _ptr(bt), bt.shape[1] if bt.ndim == 2 else 0,
                           _ptr(cl), _ptr(qsl), s, h, hk, d, bs, nb, float(scale),
                           _ptr(sel), int(threads))
    _check(rc, "decode")
    return out


def decode_fp8(q, q_dtype, k_codes, v_codes, k_scale, v_scale, block_tables, context_lens,
               scale, query_start_loc=None, rows=None, threads=0, lib=None):
    """Paged attention in fp64 over E4M3 caches (uint8 codes [NB, Hk, bs, D])
    whose elements are code value * k_scale / v_scale; q in q_dtype."""
    lib = lib or load()
    q = _raw(q)
    kc = _c(k_codes, np.uint8)
    vc = _c(v_codes, np.uint8)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    qsl = _c(query_start_loc, np.int32)
    tq, h, d = q.shape
    nb, hk, bs, d2 = kc.shape
    assert d2 == d and vc.shape == kc.shape
    out = np.full((tq, h, d), np.nan, dtype=np.float64)
    sel = None
    if rows is not None:
        sel = np.zeros(tq, dtype=np.uint8)
        sel[np.asarray(list(rows), dtype=np.int64)] = 1
    rc = lib.oracle_decode_fp8(_ptr(out), _ptr(q), DTYPES[q_dtype], _ptr(kc), _ptr(vc),
                               float(k_scale), float(v_scale), _ptr(bt),
                               bt.shape[1] if bt.ndim == 2 else 0, _ptr(cl), _ptr(qsl),
                               cl.shape[0], h, hk, d, bs, nb, float(scale), _ptr(sel), int(threads))
    _check(rc, "decode_fp8")
    return out


def reshape_and_cache_fp8(k_codes, v_codes, key, value, in_dtype, slot_mapping, k_scale, v_scale,
                          lib=None):
    """Quantise key/value [T, Hk, D] (in_dtype) to E4M3 codes of x / scale and
    scatter them into the uint8 caches in place."""
    lib = lib or load()
    assert k_codes.dtype == np.uint8 and v_codes.dtype == np.uint8
    assert k_codes.flags.c_contiguous and v_codes.flags.c_contiguous
    key = _raw(key)
    value = _raw(value)
    sm = _c(slot_mapping, np.int64)
    nb, hk, bs, d = k_codes.shape
    rc = lib.oracle_reshape_and_cache_fp8(_ptr(k_codes), _ptr(v_codes), _ptr(key), _ptr(value),
                                          DTYPES[in_dtype], _ptr(sm), sm.shape[0], hk, d, bs, nb,
                                          float(k_scale), float(v_scale))
    _check(rc, "reshape_and_cache_fp8")


def e4m3_decode(code, lib=None) -> float:
    return float((lib or load()).oracle_e4m3_decode(int(code)))


def e4m3_encode(x, lib=None) -> int:
    return int((lib or load()).oracle_e4m3_encode(float(x)))


def reshape_and_cache(k_cache, v_cache, key, value, slot_mapping, dtype, lib=None):
    """Scatter key/value [T, Hk, D] into the caches in place (byte copies)."""
    lib = lib or load()
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    key = _raw(key)
    value = _raw(value)
    sm = _c(slot_mapping, np.int64)
    nb, hk, bs, d = k_cache.shape
    rc = lib.oracle_reshape_and_cache(_ptr(k_cache), _ptr(v_cache), _ptr(key), _ptr(value),
                                      _ptr(sm), sm.shape[0], hk, d, bs, nb, DTYPES[dtype])
    _check(rc, "reshape_and_cache")


def copy_blocks(k_cache, v_cache, block_mapping, dtype, lib=None):
    """Copy whole blocks (src, dst) in place; all reads precede all writes."""
    lib = lib or load()
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    bm = _c(np.asarray(block_mapping).reshape(-1, 2), np.int64)
    nb, hk, bs, d = k_cache.shape
    rc = lib.oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(bm), bm.shape[0],
                                hk, d, bs, nb, DTYPES[dtype])
    _check(rc, "copy_blocks")


def swap_blocks(dst_k, dst_v, src_k, src_v, block_mapping, dtype, lib=None):
    """Copy whole blocks (src, dst) from the (src_k, src_v) pool into the
    (dst_k, dst_v) pool, in place."""
    lib = lib or load()
    for t in (dst_k, dst_v, src_k, src_v):
        assert t.flags.c_contiguous
    bm = _c(np.asarray(block_mapping).reshape(-1, 2), np.int64)
    nd, hk, bs, d = dst_k.shape
    ns = src_k.shape[0]
    assert src_k.shape[1:] == dst_k.shape[1:] and src_v.shape == src_k.shape and dst_v.shape == dst_k.shape
    rc = lib.oracle_swap_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(src_k), _ptr(src_v), _ptr(bm),
                                bm.shape[0], hk, d, bs, ns, nd, DTYPES[dtype])
    _check(rc, "swap_blocks")


def max_threads(lib=None) -> int:
    return (lib or load()).oracle_max_threads()
