"""Seeded synthetic workloads for paged KV-cache attention.

This module is shared by the CUDA path's tests/benchmark and by the CPU oracle.
It holds only random draws and the *shape* of each batch (which sequences,
their lengths, which tokens are new, the order of the free pool).  It computes
none of the method: no block tables, no slots, no attention.

Recipe (per workload, seed = 1000 + config number for the full-size configs):
  * integer structure from ``numpy.random.default_rng(seed)``, drawn in the
    order lengths -> pool permutation -> tails -> sequence order;
  * values from ``torch.Generator('cpu').manual_seed(seed)``: standard normal
    fp32, drawn in the order q, whole K pool, whole V pool, new keys, new
    values (pools in slabs of 2**24 elements), then cast to the cache dtype.

The five full-size workloads follow the configuration list of the build:
  1 tiny fp32 decode            2 Llama-2-7B-shaped MHA fp16 decode
  3 Llama-3-8B-shaped GQA bf16   4 shared-prefix parallel sampling (70B layer)
  5 long-context ragged batch with chunked-prefill rows (block size 16 and 32)
Pool size is 1.25x the blocks the batch needs (a sizing rule of the
configurations); the free list is a seeded permutation of the pool.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

DTYPE_NAMES = ("f32", "f16", "bf16")


@dataclass
class Workload:
    name: str
    kind: str                 # 'decode' | 'shared_prefix' | 'mixed'
    seed: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    num_blocks: int
    free_order: np.ndarray    # int64 permutation of range(num_blocks)
    # 'decode' / 'mixed': one entry per sequence, in batch order
    context_lens: list = field(default_factory=list)  # tokens incl. the new ones
    query_lens: list = field(default_factory=list)    # new (query) tokens per sequence
    # 'shared_prefix'
    num_prompts: int = 0
    samples: int = 0
    prompt_len: int = 0
    tails: list = field(default_factory=list)         # per sample, tokens after the prompt

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def num_seqs(self) -> int:
        if self.kind == "shared_prefix":
            return self.num_prompts * self.samples
        return len(self.context_lens)

    @property
    def num_q_tokens(self) -> int:
        if self.kind == "shared_prefix":
            return self.num_seqs
        return int(sum(self.query_lens))

    @property
    def num_new_tokens(self) -> int:
        """Tokens whose K/V are written by this step (reshape_and_cache)."""
        if self.kind == "shared_prefix":
            return int(sum(self.tails))
        return int(sum(self.query_lens))

    def seq_context_lens(self) -> list:
        if self.kind == "shared_prefix":
            return [self.prompt_len + t for t in self.tails]
        return list(self.context_lens)

    @property
    def max_context_len(self) -> int:
        return int(max(self.seq_context_lens()) if self.num_seqs else 0)

    @property
    def max_query_len(self) -> int:
        if self.kind == "shared_prefix":
            return 1
        return int(max(self.query_lens) if self.query_lens else 0)


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def _pool(rng, needed_blocks: int, exact: int | None = None):
    nb = exact if exact is not None else int(math.ceil(1.25 * needed_blocks))
    return nb, rng.permutation(nb).astype(np.int64)


def decode_workload(name, seed, lengths, H, Hk, D, bs, dtype, num_blocks=None,
                    rng=None) -> Workload:
    rng = rng if rng is not None else np.random.default_rng(seed)
    lengths = [int(x) for x in lengths]
    need = sum(_ceil_div(L, bs) for L in lengths)
    nb, perm = _pool(rng, need, num_blocks)
    return Workload(name, "decode", seed, H, Hk, D, bs, dtype, nb, perm,
                    context_lens=lengths, query_lens=[1] * len(lengths))


def shared_prefix_workload(name, seed, prompts, samples, prompt_len, tail_max,
                           H, Hk, D, bs, dtype) -> Workload:
    rng = np.random.default_rng(seed)
    # lengths: the prompt length is fixed; pool sizing uses an upper bound on
    # the tails (each sample may also take one private copy of a shared block).
    need = prompts * _ceil_div(prompt_len, bs) + prompts * samples * (_ceil_div(tail_max, bs) + 1)
    nb, perm = _pool(rng, need)
    tails = rng.integers(1, tail_max + 1, size=prompts * samples).tolist()
    return Workload(name, "shared_prefix", seed, H, Hk, D, bs, dtype, nb, perm,
                    num_prompts=prompts, samples=samples, prompt_len=prompt_len,
                    tails=[int(t) for t in tails])


def mixed_workload(name, seed, n_decode, dec_lo, dec_hi, n_chunk, prefix, chunk,
                   H, Hk, D, bs, dtype) -> Workload:
    rng = np.random.default_rng(seed)
    dec = rng.integers(dec_lo, dec_hi + 1, size=n_decode).tolist()
    lens = [int(x) for x in dec] + [prefix + chunk] * n_chunk
    qls = [1] * n_decode + [chunk] * n_chunk
    need = sum(_ceil_div(L, bs) for L in lens)
    nb, perm = _pool(rng, need)
    order = rng.permutation(len(lens))
    return Workload(name, "mixed", seed, H, Hk, D, bs, dtype, nb, perm,
                    context_lens=[lens[i] for i in order],
                    query_lens=[qls[i] for i in order])


def _reseed(config, seed):
    """The named workload drawn again from another seed (same shapes/recipe)."""
    global _SEED_OVERRIDE
    _SEED_OVERRIDE = seed
    try:
        return make(config)
    finally:
        _SEED_OVERRIDE = None


_SEED_OVERRIDE = None


def _seed(default):
    return default if _SEED_OVERRIDE is None else _SEED_OVERRIDE


def lognormal_lengths(rng, n, median, sigma, cap):
    z = rng.standard_normal(n)
    return np.clip(np.rint(np.exp(np.log(median) + sigma * z)), 1, cap).astype(np.int64).tolist()


def make(config: str, replica: int = 0) -> Workload:
    """Named workloads: the five full-size configurations and small variants
    ('s' suffix) of the same shapes that the oracle finishes in seconds.
    ``replica`` > 0 gives an independent batch of the same shape (seeds offset
    by 100000 * replica) -- one per rank when N GPUs each run their own batch."""
    if replica:
        return _reseed(config, make(config).seed + 100000 * replica)
    c = config
    if c == "1":
        return decode_workload("cfg1_tiny_fp32", _seed(1001), [17, 33, 64, 100], 4, 4, 64, 16,
                               "f32", num_blocks=64)
    if c == "2":
        rng = np.random.default_rng(_seed(1002))
        lens = rng.integers(128, 2048 + 1, size=64).tolist()
        return decode_workload("cfg2_llama2_7b_mha_fp16", _seed(1002), lens, 32, 32, 128, 16, "f16",
                               rng=rng)
    if c == "3":
        rng = np.random.default_rng(_seed(1003))
        lens = lognormal_lengths(rng, 256, 800, 0.8, 4096)
        return decode_workload("cfg3_llama3_8b_gqa_bf16", _seed(1003), lens, 32, 8, 128, 16, "bf16",
                               rng=rng)
    if c == "4":
        return shared_prefix_workload("cfg4_shared_prefix_70b_bf16", _seed(1004), 32, 8, 1024, 512,
                                      64, 8, 128, 16, "bf16")
    if c == "4cow":
        return shared_prefix_workload("cfg4cow_shared_prefix_1016_bf16", _seed(1014), 32, 8, 1016, 512,
                                      64, 8, 128, 16, "bf16")
    if c == "5":
        return mixed_workload("cfg5_long_mixed_bf16_bs16", _seed(1005), 8, 32768, 131072, 4, 16384,
                              512, 32, 8, 128, 16, "bf16")
    if c == "5bs32":
        return mixed_workload("cfg5_long_mixed_bf16_bs32", _seed(1005), 8, 32768, 131072, 4, 16384,
                              512, 32, 8, 128, 32, "bf16")
    # ---- small variants: same head shapes, dtypes and structure ----
    if c == "2s":
        rng = np.random.default_rng(_seed(2002))
        lens = rng.integers(1, 700 + 1, size=12).tolist()
        return decode_workload("cfg2s_mha_fp16_small", _seed(2002), lens, 32, 32, 128, 16, "f16", rng=rng)
    if c == "3s":
        rng = np.random.default_rng(_seed(2003))
        lens = lognormal_lengths(rng, 40, 200, 0.8, 1100)
        return decode_workload("cfg3s_gqa_bf16_small", _seed(2003), lens, 32, 8, 128, 16, "bf16", rng=rng)
    if c == "3s32":
        rng = np.random.default_rng(_seed(2013))
        lens = lognormal_lengths(rng, 24, 200, 0.8, 1100)
        return decode_workload("cfg3s_gqa_bf16_bs32_small", _seed(2013), lens, 32, 8, 128, 32, "bf16",
                               rng=rng)
    if c == "4s":
        return shared_prefix_workload("cfg4s_shared_prefix_small", _seed(2004), 2, 8, 128, 70,
                                      64, 8, 128, 16, "bf16")
    if c == "4cows":
        return shared_prefix_workload("cfg4cows_shared_prefix_cow_small", _seed(2014), 2, 8, 120, 70,
                                      64, 8, 128, 16, "bf16")
    if c == "5s":
        return mixed_workload("cfg5s_mixed_bf16_bs16_small", _seed(2005), 3, 1500, 5000, 2, 700, 96,
                              32, 8, 128, 16, "bf16")
    if c == "5s32":
        return mixed_workload("cfg5s_mixed_bf16_bs32_small", _seed(2005), 3, 1500, 5000, 2, 700, 96,
                              32, 8, 128, 32, "bf16")
    raise KeyError(config)


FULL_CONFIGS = ("1", "2", "3", "4", "4cow", "5", "5bs32")
SMALL_CONFIGS = ("1", "2s", "3s", "3s32", "4s", "4cows", "5s", "5s32")


def torch_dtype(name: str):
    import torch
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[name]


def values(wl: Workload, slab: int = 1 << 24):
    """Seeded N(0,1) values cast to the cache dtype (torch CPU tensors).

    Returns dict with q [Tq,H,D], k_pool/v_pool [NB,Hk,bs,D],
    new_key/new_value [T_new,Hk,D].
    """
    import torch
    g = torch.Generator("cpu").manual_seed(wl.seed)
    dt = torch_dtype(wl.dtype)

    def draw(shape):
        n = int(np.prod(shape))
        out = torch.empty(n, dtype=dt)
        for s in range(0, n, slab):
            e = min(n, s + slab)
            out[s:e] = torch.randn(e - s, generator=g, dtype=torch.float32).to(dt)
        return out.view(*shape)

    H, Hk, D, bs = wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size
    q = draw((wl.num_q_tokens, H, D))
    k_pool = draw((wl.num_blocks, Hk, bs, D))
    v_pool = draw((wl.num_blocks, Hk, bs, D))
    new_key = draw((wl.num_new_tokens, Hk, D))
    new_value = draw((wl.num_new_tokens, Hk, D))
    return {"q": q, "k_pool": k_pool, "v_pool": v_pool, "new_key": new_key,
            "new_value": new_value}


def to_numpy_raw(t):
    """torch CPU tensor -> numpy array the oracle accepts (bf16 as uint16 bits)."""
    import torch
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)
    return t.contiguous().numpy()
