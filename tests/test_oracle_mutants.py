"""Plant plausible mistakes in copies of the oracle and check that each one
fails at least one pin -- evidence that the pins would catch a real slip.

Every mutant is a one-line text edit of oracle/pa_oracle.c compiled into a
temporary library; the real oracle is never modified.
"""
import os
import subprocess

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "pa_oracle.c")

MUTANTS = {
    "gqa_modulo_mapping": ("int h_kv = h / group;", "int h_kv = h % num_kv_heads;"),
    "logical_not_physical_block": ("int32_t pb = table[p / block_size];", "int32_t pb = p / block_size;"),
    "offset_reversed": ("int off = p % block_size;", "int off = block_size - 1 - p % block_size;"),
    "scale_dropped": ("s *= scale;", "s *= 1.0;"),
    "no_max_shift": ("sbuf[p] = exp(sbuf[p] - m);", "sbuf[p] = exp(sbuf[p]);"),
    "causal_off_by_one": ("int n_vis = (int)(context_lens[seq] - qlen + tq + 1);",
                          "int n_vis = (int)(context_lens[seq] - qlen + tq);"),
    "no_normalisation": ("out_row[d] = acc / denom;", "out_row[d] = acc;"),
    "q_row_of_wrong_head": ("int64_t qbase = (row * num_heads + h) * (int64_t)head_dim;",
                            "int64_t qbase = (row * num_heads + h_kv) * (int64_t)head_dim;"),
    "k_and_v_swapped_in_reshape": (
        "memcpy((char *)k_cache + dst, (const char *)key + src, (size_t)row_bytes);",
        "memcpy((char *)k_cache + dst, (const char *)value + src, (size_t)row_bytes);"),
    "reshape_offset_from_block_count": ("off = slot % block_size;", "off = slot % num_blocks % block_size;"),
    "copy_without_staging": (
        "memcpy(stage_k + i * blk_bytes, (const char *)k_cache + s * blk_bytes, (size_t)blk_bytes);",
        "memcpy((char *)k_cache + block_mapping[2 * i + 1] * blk_bytes, (const char *)k_cache + s * blk_bytes, (size_t)blk_bytes); memcpy(stage_k + i * blk_bytes, (const char *)k_cache + s * blk_bytes, (size_t)blk_bytes);"),
    "swap_k_and_v_crossed": (
        "memcpy((char *)dst_k + d * blk_bytes, (const char *)src_k + s * blk_bytes, (size_t)blk_bytes);",
        "memcpy((char *)dst_k + d * blk_bytes, (const char *)src_v + s * blk_bytes, (size_t)blk_bytes);"),
    "swap_half_block": (
        "memcpy((char *)dst_v + d * blk_bytes, (const char *)src_v + s * blk_bytes, (size_t)blk_bytes);",
        "memcpy((char *)dst_v + d * blk_bytes, (const char *)src_v + s * blk_bytes, (size_t)(blk_bytes / 2));"),
    "e4m3_exponent_bias": ("v = ldexp((double)(8 + mant), expo - 10);",
                           "v = ldexp((double)(8 + mant), expo - 9);"),
    "e4m3_ties_to_odd": ("(d == best_d && (c & 1) == 0 && (best & 1) == 1)",
                         "(d == best_d && (c & 1) == 1 && (best & 1) == 0)"),
    "fp8_value_scale_from_key": ("elem(v_cache, tile + fp8_v_pos(off, d, block_size), dtype) * v_scale;",
                                 "elem(v_cache, tile + fp8_v_pos(off, d, block_size), dtype) * k_scale;"),
    "fp8_quantise_value_with_key_scale": ("fp8_v_pos((int)off, d, block_size)] = e4m3_from_float(vx / v_scale);",
                                          "fp8_v_pos((int)off, d, block_size)] = e4m3_from_float(vx / k_scale);"),
    "fp8_key_layout_unswizzled": ("int chunk = (4 * j + t) ^ (r % (head_dim / 16));",
                                  "int chunk = (4 * j + t);"),
    "f16_exponent_bias": ("v = ldexp((double)(mant | 0x400), expo - 25);",
                          "v = ldexp((double)(mant | 0x400), expo - 24);"),
    "f16_subnormal_scale": ("v = ldexp((double)mant, -24);", "v = ldexp((double)mant, -25);"),
    "bf16_wrong_half": ("uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    msrc = tmp_path / f"m_{name}.c"
    msrc.write_text(src.replace(old, new), encoding="utf-8")
    so = tmp_path / f"m_{name}.so"
    oracle.build(str(msrc), str(so), force=True)
    lib = oracle.load(str(so))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError) as e:  # noqa: PERF203
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
