"""Plant plausible mistakes in a copy of the oracle and show that the pins catch them.

Each mutant is built from ``oracle/oracle.c`` with one textual replacement
(the replaced text must occur, or the test fails), compiled with gcc into a
temporary directory and run through every check in ``tests/oracle_pins.py``.
A mutant that passes every check would mean the pins cannot see that
mistake.  CPU only.
"""
import ctypes
import shutil
import subprocess

import pytest

import oracle
from tests import oracle_pins

# (name, text in oracle.c, replacement, occurrence: 0 = first only, -1 = all)
MUTANTS = [
    ("mask_drops_own_row", "int n = seq_lens[b] + i + 1;\n        const uint16_t* Kb",
     "int n = seq_lens[b] + i;\n        const uint16_t* Kb", 0),
    ("mask_sees_next_row", "int n = seq_lens[b] + i + 1;\n        const uint16_t* Kb",
     "int n = seq_lens[b] + i + 2;\n        const uint16_t* Kb", 0),
    ("mask_ignores_chunk_row", "int n = seq_lens[b] + i + 1;\n        const uint16_t* Kb",
     "int n = seq_lens[b] + T_new;\n        const uint16_t* Kb", 0),
    ("gqa_modulo_mapping", "int g = h / group;", "int g = h % H_kv;", 0),
    ("scale_dropped", "s[j] = scale * dot;", "s[j] = dot;", 0),
    ("denominator_is_count", "double pj = s[j] / denom;", "double pj = s[j] / (double)n;", 0),
    ("exp_sign_flipped", "s[j] = exp(s[j] - mx);", "s[j] = exp(mx - s[j]);", 0),
    ("values_read_from_K", "const uint16_t* vrow = Vbase + (int64_t)j * D;",
     "const uint16_t* vrow = Kbase + (int64_t)j * D;", 0),
    ("keys_reversed", "const uint16_t* krow = Kbase + (int64_t)j * D;",
     "const uint16_t* krow = Kbase + (int64_t)(n - 1 - j) * D;", 0),
    ("q_rows_transposed", "attend_row(D, n, q + r * D,",
     "attend_row(D, n, q + (((int64_t)b * T_new + i) * H_q + h) * D,", 0),
    ("dot_drops_last_dim", "for (int d = 0; d < D; ++d)\n            dot += qd[d]",
     "for (int d = 0; d < D - 1; ++d)\n            dot += qd[d]", 0),
    ("append_contig_off_by_one", "int64_t pos = (int64_t)seq_lens[b] + i;",
     "int64_t pos = (int64_t)seq_lens[b] + i + 1;", 0),
    ("append_paged_slot_swapped",
     "int64_t page = block_table[(int64_t)b * max_pages + pos / P];\n                int64_t slot = pos % P;\n                const uint16_t* src = new_kv",
     "int64_t page = block_table[(int64_t)b * max_pages + pos % P];\n                int64_t slot = pos / P;\n                const uint16_t* src = new_kv", 0),
    ("gather_ignores_table",
     "int64_t page = block_table[(int64_t)b * max_pages + pos / P];\n                int64_t slot = pos % P;\n                const uint16_t* src = pool",
     "int64_t page = pos / P;\n                int64_t slot = pos % P;\n                const uint16_t* src = pool", 0),
    ("fp16_bias_wrong", "expo - 25", "expo - 24", 0),
    ("fp16_subnormal_scale", "ldexp((double)mant, -24)", "ldexp((double)mant, -25)", 0),
    ("rounding_ties_away", "nearbyint(a / quantum)", "round(a / quantum)", 0),
    ("kv_bytes_without_k_and_v", "return (uint64_t)2 *", "return (uint64_t)1 *", 0),
    ("chunked_no_rescale_of_sum", "l *= alpha;", "l *= 1.0;", 0),
    ("chunked_no_rescale_of_acc", "acc[d] *= alpha;", "acc[d] *= 1.0;", 0),
    ("commit_one_too_far", "seq_lens[b] = (int32_t)grown;", "seq_lens[b] = (int32_t)grown + 1;", 0),
    ("commit_accepts_past_chunk", "accepted[b] > T_new ||", "accepted[b] > T_new + 1 ||", 0),
    ("rollback_adds", "seq_lens[b] -= drop[b];", "seq_lens[b] += drop[b];", 0),
    ("copy_pages_reversed",
     "const uint16_t* from = pool + (int64_t)src[i] * page_elems;\n        uint16_t* to = pool + (int64_t)dst[i] * page_elems;",
     "const uint16_t* from = pool + (int64_t)dst[i] * page_elems;\n        uint16_t* to = pool + (int64_t)src[i] * page_elems;", 0),
    ("copy_pages_half_page", "for (int64_t e = 0; e < page_elems; ++e)",
     "for (int64_t e = 0; e < page_elems / 2; ++e)", 0),
    ("window_one_short", "seen[j] = (W == 0 || j >= n - W || j < S);",
     "seen[j] = (W == 0 || j > n - W || j < S);", 0),
    ("window_drops_sinks", "seen[j] = (W == 0 || j >= n - W || j < S);",
     "seen[j] = (W == 0 || j >= n - W);", 0),
    ("window_one_sink_too_many", "seen[j] = (W == 0 || j >= n - W || j < S);",
     "seen[j] = (W == 0 || j >= n - W || j <= S);", 0),
    ("e4m3_exponent_bias", "ldexp((double)(8 + m), e - 10)", "ldexp((double)(8 + m), e - 11)", 0),
    ("e4m3_subnormal_scale", "ldexp((double)m, -9)", "ldexp((double)m, -10)", 0),
    ("e4m3_ties_to_odd", "(c & 1) == 0 && (best & 1) == 1", "(c & 1) == 1 && (best & 1) == 0", 0),
    ("fp8_scale_447", "amax / 448.0f", "amax / 447.0f", 0),
    ("fp8_attend_drops_v_scale", "* (double)Vs[j])", "* 1.0)", 0),
    ("fp8_attend_k_scale_from_v", "(double)Ks[j])", "(double)Vs[j])", 0),
    ("gather_rows_page_slot_swapped",
     "int64_t page = block_table[(int64_t)b * max_pages + pos / P];\n                int64_t slot = pos % P;\n                const uint8_t* src = pool",
     "int64_t page = block_table[(int64_t)b * max_pages + pos % P];\n                int64_t slot = pos / P;\n                const uint8_t* src = pool", 0),
    ("gather_rows_ignores_table",
     "int64_t page = block_table[(int64_t)b * max_pages + pos / P];\n                int64_t slot = pos % P;\n                const uint8_t* src = pool",
     "int64_t page = pos / P;\n                int64_t slot = pos % P;\n                const uint8_t* src = pool", 0),
    ("gather_rows_head_dropped", "const uint8_t* src = pool + ((page * H_kv + g) * P + slot)",
     "const uint8_t* src = pool + ((page * H_kv) * P + slot)", 0),
    ("fp8_append_contig_off_by_one",
     "int64_t pos = (int64_t)seq_lens[b] + i;\n                const uint16_t* src = new_kv + (((int64_t)b * H_kv + g) * T_new + i) * D;\n                int64_t code_row",
     "int64_t pos = (int64_t)seq_lens[b] + i + 1;\n                const uint16_t* src = new_kv + (((int64_t)b * H_kv + g) * T_new + i) * D;\n                int64_t code_row", 0),
    ("fp8_append_contig_scale_stride", "int64_t scale_at = ((int64_t)b * H_kv + g) * T_pad + pos;",
     "int64_t scale_at = ((int64_t)b * H_kv + g) * T_cap + pos;", 0),
    ("fp8_append_paged_off_by_one",
     "int64_t pos = (int64_t)seq_lens[b] + i;\n                int64_t page = block_table[(int64_t)b * max_pages + pos / P];\n                int64_t slot = pos % P;\n                const uint16_t* src = new_kv + (((int64_t)b * H_kv + g) * T_new + i) * D;\n                int64_t row",
     "int64_t pos = (int64_t)seq_lens[b] + i + 1;\n                int64_t page = block_table[(int64_t)b * max_pages + pos / P];\n                int64_t slot = pos % P;\n                const uint16_t* src = new_kv + (((int64_t)b * H_kv + g) * T_new + i) * D;\n                int64_t row", 0),
    ("fp8_append_paged_slot_swapped",
     "int64_t page = block_table[(int64_t)b * max_pages + pos / P];\n                int64_t slot = pos % P;\n                const uint16_t* src = new_kv + (((int64_t)b * H_kv + g) * T_new + i) * D;\n                int64_t row",
     "int64_t page = block_table[(int64_t)b * max_pages + pos % P];\n                int64_t slot = pos / P;\n                const uint16_t* src = new_kv + (((int64_t)b * H_kv + g) * T_new + i) * D;\n                int64_t row", 0),
    ("fp8_append_scale_in_logical_page", "quantize_row(src, D, codes + row * D, &scales[row]);",
     "quantize_row(src, D, codes + row * D, &scales[((pos / P) * H_kv + g) * P + slot]);", 0),
]


def _mutate(src: str, old: str, new: str, occurrence: int) -> str:
    assert old in src, f"mutation target not found: {old!r}"
    if occurrence == -1:
        return src.replace(old, new)
    return src.replace(old, new, 1)


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new, occ):
    src = oracle.SRC.read_text()
    mutated = _mutate(src, old, new, occ)
    assert mutated != src
    c = tmp_path / f"oracle_{name}.c"
    c.write_text(mutated)
    so = oracle.build(c, tmp_path / f"liboracle_{name}.so")
    o = oracle.Oracle(oracle.load(so))
    caught = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(o)
        except (AssertionError, FloatingPointError, ValueError, ZeroDivisionError) as e:
            caught.append(check.__name__)
    assert caught, f"mutant {name} passed every pin"


def test_unmutated_copy_passes(tmp_path):
    c = tmp_path / "oracle_copy.c"
    shutil.copy(oracle.SRC, c)
    o = oracle.Oracle(oracle.load(oracle.build(c, tmp_path / "liboracle_copy.so")))
    for check in oracle_pins.ALL_CHECKS:
        check(o)
