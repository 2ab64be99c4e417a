"""Host-side argument checks of the Python binding (no GPU needed).

Every entry point reads its sizes from one tensor and indexes the others with
them on the device, so the binding must refuse tensors whose shapes disagree
before anything reaches a kernel, and tensors that live on another GPU than
the current one (the kernels run on the current device).
"""
import pytest
import torch

from paged_kv_cache_388_b200 import _lib


def _decode_args(S=2, H=8, Hk=2, D=128, bs=16, nb=8, mbps=4, tq=None, dtype=torch.bfloat16):
    q = torch.zeros(S if tq is None else tq, H, D, dtype=dtype)
    return dict(out=torch.zeros_like(q), q=q, k_cache=torch.zeros(nb, Hk, bs, D, dtype=dtype),
                v_cache=torch.zeros(nb, Hk, bs, D, dtype=dtype),
                block_tables=torch.zeros(S, mbps, dtype=torch.int32),
                context_lens=torch.zeros(S, dtype=torch.int32), scale=0.1)


def _call(fn, a, **kw):
    return fn(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"], a["context_lens"],
              a["scale"], **kw)


@pytest.mark.parametrize("fn", [_lib.pa_decode, _lib.pa_decode_noalloc])
def test_decode_shape_disagreements(fn):
    a = _decode_args()
    a["context_lens"] = torch.zeros(3, dtype=torch.int32)
    with pytest.raises(ValueError, match="number of sequences"):
        _call(fn, a)
    a = _decode_args()
    a["v_cache"] = torch.zeros(8, 2, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="k_cache and v_cache"):
        _call(fn, a)
    a = _decode_args(tq=5)
    with pytest.raises(ValueError, match="one row per sequence"):
        _call(fn, a)
    a = _decode_args(tq=5)
    with pytest.raises(ValueError, match="num_seqs \\+ 1"):
        _call(fn, a, query_start_loc=torch.tensor([0, 5], dtype=torch.int32), max_query_len=4)
    a = _decode_args()
    a["out"] = torch.zeros(2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="out and q"):
        _call(fn, a)
    a = _decode_args(H=6, Hk=4)
    with pytest.raises(ValueError, match="multiple of num_kv_heads"):
        _call(fn, a)


def test_decode_passes_shapes_then_wants_cuda():
    # consistent shapes get as far as the device check
    a = _decode_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        _call(_lib.pa_decode, a)


def test_fp8_and_shared_prefix_shape_disagreements():
    a = _decode_args()
    kc = torch.zeros(8, 2, 16, 128, dtype=torch.uint8)
    with pytest.raises(ValueError, match="number of sequences"):
        _lib.pa_decode_fp8(a["out"], a["q"], kc, kc, a["block_tables"],
                           torch.zeros(1, dtype=torch.int32), 0.1, 1.0, 1.0)
    with pytest.raises(ValueError, match="group_start"):
        _lib.pa_decode_shared_prefix(a["out"], a["q"], a["k_cache"], a["v_cache"],
                                     a["block_tables"], a["context_lens"],
                                     torch.zeros(3, dtype=torch.int32),
                                     torch.zeros(1, dtype=torch.int32), 0.1)


@pytest.mark.parametrize("fn", [_lib.pa_reshape_and_cache, _lib.pa_reshape_and_cache_fp8])
def test_reshape_shape_disagreements(fn):
    cache_dt = torch.uint8 if fn is _lib.pa_reshape_and_cache_fp8 else torch.bfloat16
    kc = torch.zeros(8, 2, 16, 128, dtype=cache_dt)
    extra = (1.0, 1.0) if fn is _lib.pa_reshape_and_cache_fp8 else ()
    key = torch.zeros(3, 2, 128, dtype=torch.bfloat16)
    slots = torch.zeros(3, dtype=torch.int64)
    with pytest.raises(ValueError, match="key and value"):
        fn(key, torch.zeros(4, 2, 128, dtype=torch.bfloat16), kc, kc, slots, *extra)
    with pytest.raises(ValueError, match="one slot per"):
        fn(key, key, kc, kc, torch.zeros(2, dtype=torch.int64), *extra)
    with pytest.raises(ValueError, match="to match the caches"):
        fn(torch.zeros(3, 4, 128, dtype=torch.bfloat16), torch.zeros(3, 4, 128, dtype=torch.bfloat16),
           kc, kc, slots, *extra)
    with pytest.raises(ValueError, match="k_cache and v_cache"):
        fn(key, key, kc, torch.zeros(9, 2, 16, 128, dtype=cache_dt), slots, *extra)


def test_copy_blocks_mapping_shape():
    kc = torch.zeros(8, 2, 16, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="num_pairs, 2"):
        _lib.pa_copy_blocks(kc, kc, torch.zeros(3, dtype=torch.int64))


class _FakeCudaTensor:
    """Stands in for a CUDA tensor on device 1 (no GPU here)."""
    is_cuda = True
    dtype = torch.bfloat16

    class device:  # noqa: N801
        index = 1

    def is_contiguous(self):
        return True


def test_tensor_on_another_device_is_refused(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="current device is cuda:0"):
        _lib._dev(_FakeCudaTensor(), "q")
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    assert isinstance(_lib._dev(_FakeCudaTensor(), "q"), _FakeCudaTensor)


def _fp8_args(S=2, tq=None):
    a = _decode_args(S=S, tq=tq)
    a["k_cache"] = torch.zeros(8, 2, 16, 128, dtype=torch.uint8)
    a["v_cache"] = torch.zeros(8, 2, 16, 128, dtype=torch.uint8)
    return a


def test_fp8_rows_and_shared_prefix_fp8_shape_disagreements():
    a = _fp8_args(tq=5)
    with pytest.raises(ValueError, match="num_seqs \\+ 1"):
        _lib.pa_decode_fp8_rows(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                                a["context_lens"], torch.tensor([0, 5], dtype=torch.int32), 0.1,
                                1.0, 1.0, 4, 1)
    a = _fp8_args()
    a["context_lens"] = torch.zeros(3, dtype=torch.int32)
    with pytest.raises(ValueError, match="number of sequences"):
        _lib.pa_decode_shared_prefix_fp8(a["out"], a["q"], a["k_cache"], a["v_cache"],
                                         a["block_tables"], a["context_lens"],
                                         torch.tensor([0, 2], dtype=torch.int32),
                                         torch.tensor([1], dtype=torch.int32), 0.1, 1.0, 1.0, 1)
    a = _fp8_args()
    with pytest.raises(ValueError, match="one more entry"):
        _lib.pa_decode_shared_prefix_fp8(a["out"], a["q"], a["k_cache"], a["v_cache"],
                                         a["block_tables"], a["context_lens"],
                                         torch.tensor([0, 2], dtype=torch.int32),
                                         torch.tensor([1, 1], dtype=torch.int32), 0.1, 1.0, 1.0, 2)


def test_staged_blocks_needed():
    """The staging bound counts the blocks of the sequences with more than one
    query row (ceil(L / block_size)), nothing for decode rows or empty ones."""
    from paged_kv_cache_388_b200.batch import staged_blocks_needed
    qsl = [0, 1, 97, 98, 98, 610]          # rows 1, 96, 1, 0, 512
    lens = [5000, 796, 17, 0, 16896]
    assert staged_blocks_needed(qsl, lens, 16) == 50 + 1056
    assert staged_blocks_needed(qsl, lens, 32) == 25 + 528
    assert staged_blocks_needed([0, 1, 2], [10, 20], 16) == 0
