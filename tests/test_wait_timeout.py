"""A wait inside a kernel that runs out ends in PA_DEVERR_TIMEOUT, not a hang.

libpa_waittest.so is libpa built with a 50 ms wait limit and a decode kernel
whose CTA 0 announces one K/V copy on its stage barrier and never issues it,
so nothing ever completes that barrier.  The consumer warps' wait for the
stage expires; the CTA unwinds (every later wait returns at once, the
producer lets the copies it did start land before the CTA exits) and the
host reads the timeout bit.  Outputs the unwound CTA owned are zeros, every
other (token, head) equals the normal library's output, and the device keeps
working: the normal library runs correctly right after.
"""
import ctypes

import pytest
import torch

import workloads
from gpu_harness import device_inputs
from paged_kv_cache_388_b200.batch import build_batch

pytestmark = pytest.mark.gpu

PA_DEVERR_TIMEOUT = 0x10


def _bind(path):
    lib = ctypes.CDLL(path)
    P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.pa_decode.restype = I
    lib.pa_decode.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, I, I, I, F, I, I, I, P, SZ, P]
    lib.pa_get_device_error.restype = I
    lib.pa_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), P]
    return lib


def test_expired_wait_unwinds_with_timeout_bit():
    from paged_kv_cache_388_b200 import _lib, build
    wt = _bind(build.WAITTEST_LIB)
    wl = workloads.make("3s")  # 40 sequences, 32 q / 8 kv heads, bf16: the balanced partition
    vals = workloads.values(wl)
    batch = build_batch(wl)
    d = device_inputs(wl, vals, batch)
    _lib.pa_reshape_and_cache(d["key"], d["value"], d["k_cache"], d["v_cache"], d["slot_mapping"])
    ws = torch.empty(max(16, _lib.pa_decode_workspace_size(
        batch.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
        batch.max_context_len, 0)), dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(d["q"])
    _lib.pa_decode(ref, d["q"], d["k_cache"], d["v_cache"], d["block_tables"], d["context_lens"],
                   wl.scale, max_context_len=batch.max_context_len, workspace=ws)
    torch.cuda.synchronize()
    assert _lib.pa_get_device_error() == 0

    out = torch.full_like(d["q"], 7.0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = wt.pa_decode(out.data_ptr(), d["q"].data_ptr(), d["k_cache"].data_ptr(),
                      d["v_cache"].data_ptr(), d["block_tables"].data_ptr(),
                      d["block_tables"].shape[1], d["context_lens"].data_ptr(), None,
                      batch.num_seqs, batch.num_seqs, 1, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                      wl.block_size, wl.num_blocks, wl.scale, batch.max_context_len, 0, 2,
                      ws.data_ptr(), ws.numel(), stream)
    assert rc == 0
    code = ctypes.c_uint(0)
    assert wt.pa_get_device_error(ctypes.byref(code), stream) == 0
    assert code.value & PA_DEVERR_TIMEOUT, hex(code.value)

    o, r = out.float(), ref.float()
    assert not torch.isnan(o).any()
    same = (o == r).all(dim=2)   # per (token, head)
    zero = (o == 0).all(dim=2)
    assert bool((same | zero).all()), "an output is neither the reference nor zero"
    assert bool(zero.any()), "the unwound CTA's outputs should be zeros"
    assert bool(same.any())

    # the device is still usable: the normal library gives the reference again
    again = torch.empty_like(d["q"])
    _lib.pa_decode(again, d["q"], d["k_cache"], d["v_cache"], d["block_tables"], d["context_lens"],
                   wl.scale, max_context_len=batch.max_context_len, workspace=ws)
    torch.cuda.synchronize()
    assert _lib.pa_get_device_error() == 0
    assert torch.equal(again, ref)
