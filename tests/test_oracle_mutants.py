"""Mutation check of the oracle's pins: each plausible mistake, planted in a copy of
the C oracle compiled here on the CPU, must make at least one pin fail."""
import os

import pytest

import oracle
from oracle import build_oracle
from tests import pins

# (name, original text, mutated text) -- each a mistake someone could plausibly make.
MUTANTS = [
    ("gqa_map", "int g = h / (num_q_heads / num_kv_heads);", "int g = h % num_kv_heads;"),
    ("wrong_page_index", "int blk = table[t / block_size];",
     "int blk = table[(t / block_size) / 2];"),
    ("row_in_page", "+ (t % block_size)) * d;", "+ (block_size - 1 - t % block_size)) * d;"),
    ("dropped_scale", "z[t] = scale * acc;", "z[t] = acc;"),
    ("k_for_v", "out[i] += z[t] * Vc[(size_t)t * d + i];",
     "out[i] += z[t] * Kc[(size_t)t * d + i];"),
    ("no_normalise", "out[i] /= denom;", "out[i] /= 1.0;"),
    ("drops_last_token", "if (L <= 0) return 0;", "if (L <= 0) return 0;\n    if (L > 1) --L;"),
    ("fp16_bias", "e - 25", "e - 24"),
    ("bf16_shift", "(uint32_t)h << 16", "(uint32_t)h << 15"),
    ("q_head", "((size_t)s * num_q_heads + h) * head_dim", "((size_t)s * num_q_heads + 0) * head_dim"),
    ("write_skips_slot0", "if (slot < 0) continue;", "if (slot <= 0) continue;"),
    ("write_head0", "(size_t)t * key_token_stride + (size_t)h * head_dim",
     "(size_t)t * key_token_stride + (size_t)0 * head_dim"),
    ("copy_reversed", "int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];",
     "int64_t dst = pairs[2 * p], src = pairs[2 * p + 1];"),
    ("softmax_no_exp", "z[t] = exp(z[t] - m);", "z[t] = (z[t] - m) + 1000.0;"),
    ("window_one_short", "int t_lo = (window > 0 && L > window) ? L - window : 0;",
     "int t_lo = (window > 0 && L > window) ? L - window + 1 : 0;"),
    ("window_one_long", "int t_lo = (window > 0 && L > window) ? L - window : 0;",
     "int t_lo = (window > 0 && L > window) ? L - window - 1 : 0;"),
    ("window_ignored", "int t_lo = (window > 0 && L > window) ? L - window : 0;", "int t_lo = 0;"),
    ("prefill_pos_early", "int pos = L - n + (tok - query_start_loc[s]);",
     "int pos = L - n + (tok - query_start_loc[s]) - 1;"),
    ("prefill_pos_late", "int pos = L - n + (tok - query_start_loc[s]);",
     "int pos = L - n + (tok - query_start_loc[s]) + (n < L);"),
    ("prefill_wrong_seq", "query_start_loc[s] <= tok && tok < query_start_loc[s + 1]",
     "query_start_loc[s] <= tok && tok <= query_start_loc[s + 1]"),
    ("prefill_not_causal", "pos + 1, h,", "L, h,"),
    ("prefill_q_head", "q + ((size_t)tok * num_q_heads + h) * head_dim",
     "q + ((size_t)tok * num_q_heads + 0) * head_dim"),
    ("prefill_window_ignored", "dtype,\n                    window) != 0)",
     "dtype,\n                    0) != 0)"),
    ("softmax_skips_first", "for (int t = t_lo; t < L; ++t) {\n            z[t] = exp",
     "for (int t = t_lo + 1; t < L; ++t) {\n            z[t] = exp"),
    ("fp16_subnormal", "ldexp((double)f, -24)", "ldexp((double)f, -23)"),
    ("copy_v_from_k", "v_cache[(size_t)dst * blk + i] = v_cache[(size_t)src * blk + i];",
     "v_cache[(size_t)dst * blk + i] = k_cache[(size_t)src * blk + i];"),
    ("write_v_from_key", "v_cache[dst + i] = vs[i];", "v_cache[dst + i] = ks[i];"),
    ("copy_rows_whole_block", "for (int64_t r = 0; r < rows; ++r) {",
     "for (int64_t r = 0; r < block_size; ++r) {"),
    ("copy_rows_head0", "size_t from = (((size_t)src * num_kv_heads + h) * block_size + r)",
     "size_t from = (((size_t)src * num_kv_heads + 0) * block_size + r)"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = open(build_oracle.SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mpath = tmp_path / f"mut_{name}.c"
    mpath.write_text(src.replace(old, new))
    lib_path = build_oracle.build(force=True, src=str(mpath), out=str(tmp_path / f"lib_{name}.so"))
    lib = oracle.load(lib_path)
    failed = pins.run_all(lib)
    assert failed, f"mutant {name} passed every pin"


def test_unmutated_passes_all(oracle_lib):
    assert pins.run_all(oracle_lib) == []
