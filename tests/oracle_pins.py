"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each pin takes the oracle shared library handle, so the same pins run on the
real oracle (tests/test_oracle.py) and on deliberately broken copies of it
(tests/test_oracle_mutants.py, which shows every planted mistake fails one).

The pins: the pages' worked examples (tests/golden/), NumPy brute force on
contiguous, never-paged K/V, closed forms of softmax attention, and the
invariants of paging (placement, sharing, causal truncation, GQA grouping).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle
from oracle import alloc_model
from oracle.brute import attention_contiguous

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        return json.load(f)


# ----------------------------------------------------------------------------
# helpers: build paged inputs from contiguous per-sequence K/V (test side)
# ----------------------------------------------------------------------------
def _bits(x, dtype):
    """float64 array -> storage array of the cache dtype."""
    if dtype == "f32":
        return x.astype(np.float32)
    if dtype == "f16":
        return x.astype(np.float16)
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _as_f64(a, dtype):
    if dtype == "bf16":
        import torch
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    return a.astype(np.float64)


def page_sequences(ks, vs, bs, nb, rng, perm=None):
    """Place contiguous K/V ([L_i, Hk, D] each) into a pool [nb, Hk, bs, D]:
    logical block j of sequence i goes to the next block of a random
    permutation of the pool.  Returns (k_pool, v_pool, tables)."""
    hk, d = ks[0].shape[1], ks[0].shape[2]
    k_pool = rng.standard_normal((nb, hk, bs, d))  # junk in unused slots
    v_pool = rng.standard_normal((nb, hk, bs, d))
    order = list(rng.permutation(nb)) if perm is None else list(perm)
    tables = []
    for k, v in zip(ks, vs):
        L = k.shape[0]
        nblk = -(-L // bs)
        t = [int(order.pop(0)) for _ in range(nblk)]
        for j, pb in enumerate(t):
            lo, hi = j * bs, min(L, (j + 1) * bs)
            # pool[pb, head, offset, :] holds token j*bs + offset
            k_pool[pb, :, : hi - lo, :] = np.transpose(k[lo:hi], (1, 0, 2))
            v_pool[pb, :, : hi - lo, :] = np.transpose(v[lo:hi], (1, 0, 2))
        tables.append(t)
    width = max(len(t) for t in tables)
    bt = np.zeros((len(tables), width), dtype=np.int32)
    for i, t in enumerate(tables):
        bt[i, : len(t)] = t
    return k_pool, v_pool, bt


def random_case(rng, lens, qlens, H, Hk, D, bs, dtype, nb_extra=3):
    """Contiguous K/V and queries, rounded to the dtype, plus their paged form."""
    ks = [_as_f64(_bits(rng.standard_normal((L, Hk, D)), dtype), dtype) for L in lens]
    vs = [_as_f64(_bits(rng.standard_normal((L, Hk, D)), dtype), dtype) for L in lens]
    nb = sum(-(-L // bs) for L in lens) + nb_extra
    k_pool, v_pool, bt = page_sequences(ks, vs, bs, nb, rng)
    tq = sum(qlens)
    q = _as_f64(_bits(rng.standard_normal((tq, H, D)), dtype), dtype)
    qsl = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    return dict(ks=ks, vs=vs, q=q, k_pool=_bits(k_pool, dtype), v_pool=_bits(v_pool, dtype),
                bt=bt, cl=np.asarray(lens, np.int32), qsl=qsl, H=H, Hk=Hk, D=D, bs=bs,
                dtype=dtype)


def run_oracle(lib, c, scale, use_qsl=True, rows=None):
    return oracle.decode(_bits(c["q"], c["dtype"]), c["k_pool"], c["v_pool"], c["bt"], c["cl"],
                         scale, c["dtype"], query_start_loc=c["qsl"] if use_qsl else None,
                         rows=rows, lib=lib)


def run_brute(c, scale):
    outs = []
    for i, (k, v) in enumerate(zip(c["ks"], c["vs"])):
        q = c["q"][c["qsl"][i]: c["qsl"][i + 1]]
        outs.append(attention_contiguous(q, k, v, scale, c["H"] // c["Hk"]))
    return np.concatenate(outs, axis=0)


# ----------------------------------------------------------------------------
# pins
# ----------------------------------------------------------------------------
def pin_brute_force(lib):
    """Paged oracle == NumPy attention on contiguous K/V, many shapes."""
    rng = np.random.default_rng(7)
    shapes = [  # (lens, qlens, H, Hk, D, bs, dtype)
        ([17, 33, 64, 100], [1, 1, 1, 1], 4, 4, 64, 16, "f32"),
        ([1, 16, 31, 50], [1, 1, 1, 1], 8, 2, 64, 16, "f16"),
        ([40, 70], [1, 1], 16, 2, 128, 32, "bf16"),
        ([37, 65, 20], [5, 1, 20], 8, 2, 64, 16, "bf16"),
        ([48], [16], 4, 1, 64, 32, "f32"),
    ]
    for lens, qlens, H, Hk, D, bs, dt in shapes:
        c = random_case(rng, lens, qlens, H, Hk, D, bs, dt)
        scale = 1.0 / math.sqrt(D)
        got = run_oracle(lib, c, scale)
        want = run_brute(c, scale)
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12), (lens, H, Hk, D, bs, dt)


def pin_decode_without_qsl(lib):
    """query_start_loc=None means one query token per sequence."""
    rng = np.random.default_rng(8)
    c = random_case(rng, [5, 19, 33], [1, 1, 1], 4, 2, 64, 16, "f32")
    a = run_oracle(lib, c, 0.125, use_qsl=True)
    b = run_oracle(lib, c, 0.125, use_qsl=False)
    assert np.array_equal(a, b)


def pin_identical_keys_mean(lib):
    """All keys equal -> every weight equal -> output = mean of visible V."""
    rng = np.random.default_rng(9)
    L, H, Hk, D, bs = 37, 4, 2, 64, 16
    krow = rng.standard_normal((Hk, D))
    ks = [np.broadcast_to(krow, (L, Hk, D)).copy()]
    vs = [_as_f64(_bits(rng.standard_normal((L, Hk, D)), "f32"), "f32")]
    kp, vp, bt = page_sequences(ks, vs, bs, 6, rng)
    q = rng.standard_normal((1, H, D))
    out = oracle.decode(_bits(q, "f32"), _bits(kp, "f32"), _bits(vp, "f32"), bt,
                        np.asarray([L], np.int32), 0.7, "f32", lib=lib)
    for h in range(H):
        want = vs[0][:, h // (H // Hk), :].mean(axis=0)
        assert np.allclose(out[0, h], want, rtol=1e-12, atol=1e-13)


def pin_single_key(lib):
    """One visible key -> output equals that V row exactly."""
    rng = np.random.default_rng(10)
    for dt in ("f32", "f16", "bf16"):
        c = random_case(rng, [1, 1], [1, 1], 4, 2, 64, 16, dt)
        out = run_oracle(lib, c, 0.125)
        for i in range(2):
            for h in range(4):
                assert np.array_equal(out[i, h], c["vs"][i][0, h // 2, :])


def pin_dominant_logit(lib):
    """q parallel to K[j] and large -> softmax is one-hot on j -> output V[j]."""
    rng = np.random.default_rng(11)
    L, D, bs = 40, 64, 16
    k = rng.standard_normal((L, 1, D))
    k /= np.linalg.norm(k, axis=2, keepdims=True)
    v = rng.standard_normal((L, 1, D))
    kp, vp, bt = page_sequences([k], [v], bs, 5, rng)
    for j in (0, 17, 39):
        q = (60.0 * k[j, 0, :]).reshape(1, 1, D) * 8.0  # scale 1/8 undone
        out = oracle.decode(_bits(q, "f32"), _bits(kp, "f32"), _bits(vp, "f32"), bt,
                            np.asarray([L], np.int32), 0.125, "f32", lib=lib)
        vj = _as_f64(_bits(v[j, 0, :], "f32"), "f32")
        assert np.allclose(out[0, 0], vj, atol=1e-6), j
    # logits large enough to overflow exp() unless the maximum is subtracted
    q = (2000.0 * k[5, 0, :]).reshape(1, 1, D)
    out = oracle.decode(_bits(q, "f32"), _bits(kp, "f32"), _bits(vp, "f32"), bt,
                        np.asarray([L], np.int32), 1.0, "f32", lib=lib)
    assert np.all(np.isfinite(out))


def pin_v_linearity(lib):
    """Doubling V doubles the output exactly (power-of-two scaling is exact)."""
    rng = np.random.default_rng(12)
    c = random_case(rng, [29, 50], [1, 3], 8, 4, 64, 16, "f32")
    a = run_oracle(lib, c, 0.125)
    c2 = dict(c)
    c2["v_pool"] = (c["v_pool"] * 2).astype(np.float32)
    b = run_oracle(lib, c2, 0.125)
    assert np.array_equal(b, 2 * a)


def pin_scale_zero_mean(lib):
    """scale = 0 -> uniform weights -> mean of visible V (per causal row)."""
    rng = np.random.default_rng(13)
    c = random_case(rng, [23], [4], 4, 2, 64, 16, "f32")
    out = run_oracle(lib, c, 0.0)
    for t in range(4):
        n = 23 - 4 + t + 1
        for h in range(4):
            want = c["vs"][0][:n, h // 2, :].mean(axis=0)
            assert np.allclose(out[t, h], want, rtol=1e-12, atol=1e-13)


def pin_hand_example(lib):
    """A two-key example worked by hand: D=2, scale 1, q=(1,0),
    K=((0,0),(ln 3, 0)) -> weights (1/4, 3/4); V=((4,0),(8,2)) -> (7, 1.5)."""
    kp = np.zeros((1, 1, 16, 2))
    vp = np.zeros((1, 1, 16, 2))
    kp[0, 0, 1] = (math.log(3.0), 0.0)
    vp[0, 0, 0] = (4.0, 0.0)
    vp[0, 0, 1] = (8.0, 2.0)
    q = np.array([[[1.0, 0.0]]])
    out = oracle.decode(_bits(q, "f32"), _bits(kp, "f32"), _bits(vp, "f32"),
                        np.zeros((1, 1), np.int32), np.asarray([2], np.int32), 1.0, "f32", lib=lib)
    # ln 3 is rounded to fp32; the weight of key 1 is exp(fl(ln3))/(1+exp(fl(ln3)))
    assert np.allclose(out[0, 0], [7.0, 1.5], atol=1e-6)


def pin_gqa_equals_replicated_mha(lib):
    """GQA over Hk heads == MHA after replicating every KV head g times."""
    rng = np.random.default_rng(14)
    H, Hk, D, bs = 8, 2, 64, 16
    g = H // Hk
    c = random_case(rng, [21, 45], [1, 2], H, Hk, D, bs, "f32")
    a = run_oracle(lib, c, 0.125)
    rep = lambda p: np.repeat(p, g, axis=1)  # noqa: E731  kv head j -> heads j*g..j*g+g-1
    b = oracle.decode(_bits(c["q"], "f32"), rep(c["k_pool"]), rep(c["v_pool"]), c["bt"], c["cl"],
                      0.125, "f32", query_start_loc=c["qsl"], lib=lib)
    assert np.array_equal(a, b)


def pin_placement_invariance(lib):
    """Relabelling physical blocks (moving the data, rewriting the tables)
    leaves every output bit-identical."""
    rng = np.random.default_rng(15)
    c = random_case(rng, [30, 64, 7], [1, 4, 1], 8, 2, 64, 16, "bf16")
    a = run_oracle(lib, c, 0.125)
    nb = c["k_pool"].shape[0]
    pi = rng.permutation(nb)             # old block b -> new block pi[b]
    kp = np.empty_like(c["k_pool"])
    vp = np.empty_like(c["v_pool"])
    kp[pi] = c["k_pool"]
    vp[pi] = c["v_pool"]
    c2 = dict(c, k_pool=kp, v_pool=vp, bt=pi[c["bt"]].astype(np.int32))
    # unused table entries are never read; keep them in range
    b = run_oracle(lib, c2, 0.125)
    assert np.array_equal(a, b)


def pin_shared_equals_duplicated(lib):
    """Sequences pointing at the same physical blocks give the same outputs as
    sequences holding private copies of those blocks."""
    rng = np.random.default_rng(16)
    H, Hk, D, bs, P = 8, 2, 64, 16, 48
    prompt_k = rng.standard_normal((P, Hk, D))
    prompt_v = rng.standard_normal((P, Hk, D))
    tails = [5, 17, 1]
    ks = [np.concatenate([prompt_k, rng.standard_normal((t, Hk, D))]) for t in tails]
    vs = [np.concatenate([prompt_v, rng.standard_normal((t, Hk, D))]) for t in tails]
    kp, vp, bt = page_sequences(ks, vs, bs, 20, rng)           # private copies
    shared_bt = bt.copy()
    shared_bt[:, : P // bs] = bt[0, : P // bs]                  # all point at seq 0's prompt
    q = _bits(rng.standard_normal((3, H, D)), "f32")
    lens = np.asarray([P + t for t in tails], np.int32)
    a = oracle.decode(q, _bits(kp, "f32"), _bits(vp, "f32"), bt, lens, 0.125, "f32", lib=lib)
    b = oracle.decode(q, _bits(kp, "f32"), _bits(vp, "f32"), shared_bt, lens, 0.125, "f32", lib=lib)
    assert np.array_equal(a, b)


def pin_causal_truncation(lib):
    """Row t of a Q-token chunk == a decode of the same sequence truncated to
    L - Q + t + 1 tokens."""
    rng = np.random.default_rng(17)
    L, Q = 70, 12
    c = random_case(rng, [L], [Q], 8, 2, 64, 16, "f32")
    full = run_oracle(lib, c, 0.125)
    for t in (0, 5, 11):
        n = L - Q + t + 1
        one = oracle.decode(_bits(c["q"][t: t + 1], "f32"), c["k_pool"], c["v_pool"], c["bt"],
                            np.asarray([n], np.int32), 0.125, "f32", lib=lib)
        assert np.array_equal(full[t], one[0]), t


def pin_empty_context(lib):
    """Context length 0 gives a zero output (defined edge case)."""
    rng = np.random.default_rng(18)
    c = random_case(rng, [9], [1], 4, 4, 64, 16, "f32")
    out = oracle.decode(_bits(c["q"], "f32"), c["k_pool"], c["v_pool"], c["bt"],
                        np.asarray([0], np.int32), 0.125, "f32", lib=lib)
    assert np.array_equal(out, np.zeros_like(out))


def pin_dtype_decoding(lib):
    """Exact fp16 / bf16 -> double decoding, checked on every 16-bit pattern
    against the library conversions (L = 1 returns V unchanged)."""
    import torch
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    for dt in ("f16", "bf16"):
        D = 64
        n = pats.size // D
        vp = pats.reshape(n, 1, 1, D)
        vp = np.concatenate([vp, np.zeros((n, 1, 15, D), np.uint16)], axis=2)
        kp = np.zeros_like(vp)
        if dt == "f16":
            want = pats.view(np.float16).astype(np.float64)
            v_arr, k_arr, q = vp.view(np.float16), kp.view(np.float16), np.zeros((n, 1, D), np.float16)
        else:
            want = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
            v_arr, k_arr, q = vp, kp, np.zeros((n, 1, D), np.uint16)
        bt = np.arange(n, dtype=np.int32).reshape(n, 1)
        out = oracle.decode(q, k_arr, v_arr, bt, np.ones(n, np.int32), 1.0, dt, lib=lib)
        got = out.reshape(-1)
        fin = np.isfinite(want)
        assert np.array_equal(got[fin], want[fin]), dt
        assert np.array_equal(np.isnan(got), np.isnan(want)), dt


def pin_worked_block_table(lib):
    """The pages' table [5, 2, 8, 1]: tokens 0-63 of one sequence sit where
    the page says; checked through the oracle's gather (single-key reads)."""
    g = golden("block_table_worked_example.json")
    bs = g["block_size"]
    table = g["block_table"]
    for lo, hi, pb in g["logical_ranges"]:
        for p in (lo, hi):
            assert table[p // bs] == pb
    for tok, slot in g["slots_derived_by_hand"].items():
        assert alloc_model.slot_of(table, int(tok), bs) == slot
    # Through the oracle: mark every (block, offset) of the pool with its own
    # slot number in V; a query whose only visible key is logical token p
    # (causal row of a 64-token chunk, first row sees token 0 ...) returns the
    # slot number that the gather visited.
    nb, D = 9, 64
    vp = np.zeros((nb, 1, bs, D), np.float32)
    for b in range(nb):
        for o in range(bs):
            vp[b, 0, o, :] = b * bs + o
    kp = np.zeros_like(vp)
    q = np.zeros((64, 1, D), np.float32)
    bt = np.asarray([table], np.int32)
    # scale 0 -> row t returns the mean of the slot numbers of tokens 0..t
    out = oracle.decode(q, kp, vp, bt, np.asarray([64], np.int32), 0.0, "f32",
                        query_start_loc=np.asarray([0, 64], np.int32), lib=lib)
    means = out[:, 0, 0]
    slots = [means[0]] + [(t + 1) * means[t] - t * means[t - 1] for t in range(1, 64)]
    for tok, slot in g["slots_derived_by_hand"].items():
        assert abs(slots[int(tok)] - slot) < 1e-9, tok


def pin_block_counts(lib):
    g = golden("block_count_worked_example.json")
    bs, n = g["block_size"], g["tokens"]
    assert alloc_model.blocks_needed(n, bs) == g["blocks"]
    assert n - (g["blocks"] - 1) * bs == g["tokens_in_last_block"]
    m = alloc_model.PoolModel(range(20), bs)
    m.new_sequence("a", n)
    assert len(m.tables["a"]) == g["blocks"]
    g = golden("on_demand_growth.json")
    m = alloc_model.PoolModel(g["free_order_head"] + list(range(10, 20)), g["block_size"])
    m.new_sequence("a", 0)
    for n in range(1, 65):
        m.append("a")
        if str(n) in g["table_after_tokens"]:
            assert m.tables["a"] == g["table_after_tokens"][str(n)], n


def pin_reshape_then_gather(lib):
    """Writing every token of a sequence with reshape_and_cache (slots from the
    worked table rule) and reading them back through the oracle's gather
    reproduces NumPy attention over the contiguous K/V."""
    rng = np.random.default_rng(19)
    H, Hk, D, bs, L = 8, 2, 64, 16, 45
    k = rng.standard_normal((L, Hk, D)).astype(np.float32)
    v = rng.standard_normal((L, Hk, D)).astype(np.float32)
    nb = 8
    kp = rng.standard_normal((nb, Hk, bs, D)).astype(np.float32)
    vp = rng.standard_normal((nb, Hk, bs, D)).astype(np.float32)
    before_k, before_v = kp.copy(), vp.copy()
    table = [6, 1, 3]
    slots = np.asarray([alloc_model.slot_of(table, p, bs) for p in range(L)], np.int64)
    slots_pad = np.concatenate([slots[:20], [-1], slots[20:]])       # a padding token
    kk = np.concatenate([k[:20], np.full((1, Hk, D), 99, np.float32), k[20:]])
    vv = np.concatenate([v[:20], np.full((1, Hk, D), 99, np.float32), v[20:]])
    oracle.reshape_and_cache(kp, vp, kk, vv, slots_pad, "f32", lib=lib)
    # untouched blocks and the tail of the last block keep their bytes
    for b in range(nb):
        if b not in table:
            assert np.array_equal(kp[b], before_k[b]) and np.array_equal(vp[b], before_v[b])
    assert np.array_equal(kp[3, :, L - 32:], before_k[3, :, L - 32:])
    q = rng.standard_normal((3, H, D)).astype(np.float32)
    bt = np.asarray([table], np.int32)
    out = oracle.decode(q, kp, vp, bt, np.asarray([L], np.int32), 0.125, "f32",
                        query_start_loc=np.asarray([0, 3], np.int32), lib=lib)
    want = attention_contiguous(q.astype(np.float64), k, v, 0.125, H // Hk)
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12)


def pin_copy_blocks(lib):
    """Copy-on-write copies: dst gets src's bytes, every other block keeps its
    own; with a chain (a->b, b->c) c receives b's bytes from before the call."""
    rng = np.random.default_rng(20)
    nb, Hk, bs, D = 10, 2, 16, 64
    for dt in ("f32", "bf16"):
        kp = _bits(rng.standard_normal((nb, Hk, bs, D)), dt)
        vp = _bits(rng.standard_normal((nb, Hk, bs, D)), dt)
        k0, v0 = kp.copy(), vp.copy()
        pairs = [(1, 7), (4, 2), (7, 9)]          # 7 is read (for 9) and written (from 1)
        oracle.copy_blocks(kp, vp, pairs, dt, lib=lib)
        assert np.array_equal(kp[7], k0[1]) and np.array_equal(vp[7], v0[1])
        assert np.array_equal(kp[2], k0[4]) and np.array_equal(vp[2], v0[4])
        assert np.array_equal(kp[9], k0[7]) and np.array_equal(vp[9], v0[7])
        for b in set(range(nb)) - {7, 2, 9}:
            assert np.array_equal(kp[b], k0[b]) and np.array_equal(vp[b], v0[b])


def pin_swap_blocks(lib):
    """Moving blocks between two pools (device tier <-> host tier): every
    destination block named by a pair holds its source block's bytes, K from K
    and V from V, every other destination block is untouched, the source pool
    is not modified, and swapping out then back in restores the original
    bytes at the original block ids."""
    rng = np.random.default_rng(21)
    Hk, bs, D = 2, 16, 64
    for dt in ("f32", "bf16"):
        dev_k = _bits(rng.standard_normal((12, Hk, bs, D)), dt)
        dev_v = _bits(rng.standard_normal((12, Hk, bs, D)), dt)
        host_k = _bits(rng.standard_normal((5, Hk, bs, D)), dt)
        host_v = _bits(rng.standard_normal((5, Hk, bs, D)), dt)
        d0k, d0v, h0k, h0v = dev_k.copy(), dev_v.copy(), host_k.copy(), host_v.copy()
        out_pairs = [(3, 0), (11, 4), (7, 2)]    # device block -> host block
        oracle.swap_blocks(host_k, host_v, dev_k, dev_v, out_pairs, dt, lib=lib)
        assert np.array_equal(dev_k, d0k) and np.array_equal(dev_v, d0v)
        for s, d in out_pairs:
            assert np.array_equal(host_k[d], d0k[s]) and np.array_equal(host_v[d], d0v[s])
        for d in (1, 3):
            assert np.array_equal(host_k[d], h0k[d]) and np.array_equal(host_v[d], h0v[d])
        # the device blocks are reused by others, then the sequence comes back
        dev_k[[3, 11, 7]] = 0
        dev_v[[3, 11, 7]] = 0
        oracle.swap_blocks(dev_k, dev_v, host_k, host_v, [(d, s) for s, d in out_pairs], dt, lib=lib)
        assert np.array_equal(dev_k, d0k) and np.array_equal(dev_v, d0v)
        # against the definition by array indexing, on a random mapping
        src = rng.permutation(12)[:6]
        dst = rng.permutation(5)[:4]
        pairs = list(zip(src[:4].tolist(), dst.tolist()))
        want_k, want_v = host_k.copy(), host_v.copy()
        want_k[dst] = dev_k[src[:4]]
        want_v[dst] = dev_v[src[:4]]
        oracle.swap_blocks(host_k, host_v, dev_k, dev_v, pairs, dt, lib=lib)
        assert np.array_equal(host_k, want_k) and np.array_equal(host_v, want_v)


def _torch_e4m3(x32):
    """float32 array -> E4M3 codes by torch's own float8_e4m3fn conversion
    (round to nearest even; inputs kept within +-448, where it saturates
    nothing)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_e4m3_codec(lib):
    """The E4M3 codec against torch's float8_e4m3fn: every one of the 256
    codes decodes to torch's value, and quantisation of random magnitudes
    across the whole range, of exact ties (ties go to the even code) and of
    subnormals gives torch's code; beyond 448 the oracle saturates."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = np.array([oracle.e4m3_decode(c, lib=lib) for c in codes])
    assert np.array_equal(np.isnan(got), np.isnan(want))
    assert np.array_equal(got[~np.isnan(got)], want[~np.isnan(want)])
    rng = np.random.default_rng(22)
    x = rng.standard_normal(4000) * rng.choice([1e-3, 3e-2, 1.0, 30.0, 200.0], 4000)
    finite = want[np.isfinite(want)]
    mids = (np.unique(finite)[1:] + np.unique(finite)[:-1]) / 2  # every tie between neighbours
    x = np.concatenate([x, mids, -mids[:50], [0.0, -0.0, 2.0 ** -9, 2.0 ** -10, 447.0]])
    x = x[np.abs(x) <= 448].astype(np.float32)
    mine = np.array([oracle.e4m3_encode(v, lib=lib) for v in x], dtype=np.uint8)
    assert np.array_equal(mine, _torch_e4m3(x))
    assert oracle.e4m3_encode(1e6, lib=lib) == 0x7E and oracle.e4m3_encode(-500.0, lib=lib) == 0xFE


def pin_fp8_layout_examples(lib):
    """Where one element lands inside an FP8 (block, head) tile, against
    positions worked out by hand from the layout contract (K columns
    interleaved in groups of 16 and 16-byte chunks swizzled by the row; V
    stored transposed with keys interleaved): a single token whose element d
    is 1.0 (code 0x38) and every other element 0."""
    cases_k = {(16, 128): [((0, 0), 0), ((0, 1), 1), ((0, 8), 2), ((0, 9), 3), ((0, 2), 16),
                           ((0, 16), 4), ((0, 64), 64), ((3, 0), 432), ((5, 18), 708)],
               (32, 64): [((0, 2), 16), ((1, 0), 64 + 16), ((6, 33), 6 * 64 + 16 * (0 ^ 2) + 4 * 2 + 1)]}
    cases_v = {(16, 128): [((0, 0), 0), ((1, 0), 1), ((8, 0), 2), ((2, 0), 4), ((10, 0), 6),
                           ((3, 5), 85)],
               (32, 64): [((17, 2), 69), ((31, 0), 8 * 3 + 4 + 3)]}
    for (bs, D), cases in cases_k.items():
        for (r, d), want in cases:
            kc = np.zeros((1, 1, bs, D), np.uint8)
            vc = np.zeros((1, 1, bs, D), np.uint8)
            key = np.zeros((1, 1, D), np.float32)
            key[0, 0, d] = 1.0
            oracle.reshape_and_cache_fp8(kc, vc, key, np.zeros_like(key), "f32",
                                         np.array([r], np.int64), 1.0, 1.0, lib=lib)
            assert np.flatnonzero(kc.reshape(-1)).tolist() == [want], (bs, D, r, d)
            assert kc.reshape(-1)[want] == 0x38
    for (bs, D), cases in cases_v.items():
        for (r, d), want in cases:
            kc = np.zeros((1, 1, bs, D), np.uint8)
            vc = np.zeros((1, 1, bs, D), np.uint8)
            val = np.zeros((1, 1, D), np.float32)
            val[0, 0, d] = 1.0
            oracle.reshape_and_cache_fp8(kc, vc, np.zeros_like(val), val, "f32",
                                         np.array([r], np.int64), 1.0, 1.0, lib=lib)
            assert np.flatnonzero(vc.reshape(-1)).tolist() == [want], (bs, D, r, d)


def pin_fp8_reshape(lib):
    """Quantising scatter: each token's K row lands in row (slot mod
    block_size) of its slot's (block, head) tile as exactly torch's E4M3
    codes of the float32 quotients x / k_scale -- the same bytes, in the
    tile's column order; tiles that no slot addresses keep their bytes, and a
    padding slot writes nothing.  (Where V bytes land is pinned by the worked
    layout examples and by attention over the written codes.)"""
    import torch
    rng = np.random.default_rng(23)
    nb, Hk, bs, D = 6, 2, 16, 64
    for dt in ("f32", "bf16"):
        key = _bits(rng.standard_normal((5, Hk, D)) * 3, dt)
        val = _bits(rng.standard_normal((5, Hk, D)) * 3, dt)
        kc = rng.integers(0, 256, (nb, Hk, bs, D), dtype=np.uint8)
        vc = rng.integers(0, 256, (nb, Hk, bs, D), dtype=np.uint8)
        k0, v0 = kc.copy(), vc.copy()
        slots = np.array([5, -1, 40, 95, 33], dtype=np.int64)   # blocks 0, -, 2, 5, 2
        ks, vs = 0.0517, 0.0391
        oracle.reshape_and_cache_fp8(kc, vc, key, val, dt, slots, ks, vs, lib=lib)
        kf = _as_f64(key, dt).astype(np.float32)
        qk = _torch_e4m3(torch.from_numpy(kf).div(np.float32(ks)).numpy())
        for b in (1, 3, 4):
            assert np.array_equal(kc[b], k0[b]) and np.array_equal(vc[b], v0[b])
        for t, sl in enumerate(slots):
            if sl < 0:
                continue
            for h in range(Hk):
                row = kc[sl // bs, h, sl % bs]
                assert sorted(row.tolist()) == sorted(qk[t, h].tolist())
        for b, used in ((0, {5}), (2, {8, 1}), (5, {15})):   # rows other than the written ones
            for r in set(range(bs)) - used:
                assert np.array_equal(kc[b, :, r], k0[b, :, r])


def pin_fp8_decode(lib):
    """Write tokens with the E4M3 reshape, then attend over the codes: the
    result is bit-identical to the pinned float32 path (natural layout) over
    the dequantised values code * scale written by the plain reshape -- for
    scales whose products are exact in float32 (powers of two, 3/8, 5/16) --
    with q in bf16; a one-key context returns that key's dequantised value
    row exactly; the value scale enters linearly."""
    import torch
    rng = np.random.default_rng(24)
    Hk, H = 2, 8
    deq = np.array([oracle.e4m3_decode(c, lib=lib) for c in range(256)])
    for bs, D in ((16, 64), (32, 128)):
        nb = 10
        lens = np.array([1, 16, 33, 70], dtype=np.int32)
        need = [-(-int(L) // bs) for L in lens]
        perm = rng.permutation(nb)
        bt = np.zeros((len(lens), 5), np.int32)
        pos = 0
        for i, n in enumerate(need):            # distinct physical blocks per sequence
            bt[i, :n] = perm[pos:pos + n]
            pos += n
        slots = []
        for i, L in enumerate(lens):
            for p in range(L):
                slots.append(int(bt[i, p // bs]) * bs + p % bs)
        slots = np.asarray(slots, np.int64)
        T = slots.shape[0]
        key = _bits(rng.standard_normal((T, Hk, D)) * 2, "bf16")
        val = _bits(rng.standard_normal((T, Hk, D)) * 2, "bf16")
        for ks, vs in ((0.25, 4.0), (0.375, 0.3125)):
            kc = rng.integers(0, 256, (nb, Hk, bs, D), dtype=np.uint8)
            vc = rng.integers(0, 256, (nb, Hk, bs, D), dtype=np.uint8)
            oracle.reshape_and_cache_fp8(kc, vc, key, val, "bf16", slots, ks, vs, lib=lib)
            kq = _torch_e4m3(torch.from_numpy(_as_f64(key, "bf16").astype(np.float32)).div(np.float32(ks)).numpy())
            vq = _torch_e4m3(torch.from_numpy(_as_f64(val, "bf16").astype(np.float32)).div(np.float32(vs)).numpy())
            kf = np.zeros((nb, Hk, bs, D), np.float32)
            vf = np.zeros((nb, Hk, bs, D), np.float32)
            oracle.reshape_and_cache(kf, vf, (deq[kq] * ks).astype(np.float32),
                                     (deq[vq] * vs).astype(np.float32), slots, "f32", lib=lib)
            q = _bits(rng.standard_normal((4, H, D)), "bf16")
            qf = _as_f64(q, "bf16").astype(np.float32)
            got = oracle.decode_fp8(q, "bf16", kc, vc, ks, vs, bt, lens, 0.125, lib=lib)
            want = oracle.decode(qf, kf, vf, bt, lens, 0.125, "f32", lib=lib)
            assert np.array_equal(got, want)
            one = deq[vq[0]] * vs                    # sequence 0 holds token 0 only
            assert np.array_equal(got[0].reshape(H, D), np.repeat(one, H // Hk, axis=0))
            got2 = oracle.decode_fp8(q, "bf16", kc, vc, ks, 2 * vs, bt, lens, 0.125, lib=lib)
            assert np.allclose(got2, 2 * got, rtol=1e-12, atol=0)


ALL_PINS = [
    pin_brute_force, pin_decode_without_qsl, pin_identical_keys_mean, pin_single_key,
    pin_dominant_logit, pin_v_linearity, pin_scale_zero_mean, pin_hand_example,
    pin_gqa_equals_replicated_mha, pin_placement_invariance, pin_shared_equals_duplicated,
    pin_causal_truncation, pin_empty_context, pin_dtype_decoding, pin_worked_block_table,
    pin_block_counts, pin_reshape_then_gather, pin_copy_blocks, pin_swap_blocks,
    pin_e4m3_codec, pin_fp8_layout_examples, pin_fp8_reshape, pin_fp8_decode,
]
