"""The pins must catch plausible mistakes in the oracle.

Each case below plants one mistake in a copy of the oracle's C source (on the
CPU), builds it, and runs the pin suite against it in a subprocess; the suite
has to fail.  The committed oracle itself is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dsa_oracle.c")

MUTATIONS = {
    "relu_dropped": ("int64_t relu = dot > 0 ? dot : 0;", "int64_t relu = dot;"),
    "relu_is_abs": ("int64_t relu = dot > 0 ? dot : 0;", "int64_t relu = dot > 0 ? dot : -dot;"),
    "logical_not_physical_page": ("const int8_t *kc = kc_pool + (long)page * idx_dim;",
                                  "const int8_t *kc = kc_pool + (long)b * idx_dim;"),
    "visibility_off_by_one": ("int n_vis = p / block_size + 1;\n        if (n_vis > max_blocks) return ORC_BAD_POS;\n"
                              "        for (int b = 0; b < max_blocks; ++b) scores[(long)t * max_blocks + b] = INT64_MIN;\n"
                              "        for (int b = 0; b < n_vis; ++b) {\n"
                              "            int page = block_table[(long)s * max_blocks + b];\n"
                              "            if (page < 0 || page >= num_pages) return ORC_BAD_PAGE;\n"
                              "            const int8_t *kc",
                              "int n_vis = p / block_size;\n        if (n_vis > max_blocks) return ORC_BAD_POS;\n"
                              "        for (int b = 0; b < max_blocks; ++b) scores[(long)t * max_blocks + b] = INT64_MIN;\n"
                              "        for (int b = 0; b < n_vis; ++b) {\n"
                              "            int page = block_table[(long)s * max_blocks + b];\n"
                              "            if (page < 0 || page >= num_pages) return ORC_BAD_PAGE;\n"
                              "            const int8_t *kc"),
    "fp8_visibility_off_by_one": ("int n_vis = p / block_size + 1;\n        if (n_vis > max_blocks) return ORC_BAD_POS;\n"
                                  "        for (int b = 0; b < max_blocks; ++b) scores[(long)t * max_blocks + b] = INT64_MIN;\n"
                                  "        for (int b = 0; b < n_vis; ++b) {\n"
                                  "            int page = block_table[(long)s * max_blocks + b];\n"
                                  "            if (page < 0 || page >= num_pages) return ORC_BAD_PAGE;\n"
                                  "            const uint8_t *kc",
                                  "int n_vis = p / block_size;\n        if (n_vis > max_blocks) return ORC_BAD_POS;\n"
                                  "        for (int b = 0; b < max_blocks; ++b) scores[(long)t * max_blocks + b] = INT64_MIN;\n"
                                  "        for (int b = 0; b < n_vis; ++b) {\n"
                                  "            int page = block_table[(long)s * max_blocks + b];\n"
                                  "            if (page < 0 || page >= num_pages) return ORC_BAD_PAGE;\n"
                                  "            const uint8_t *kc"),
    "weight_index_transposed": ("total += (int64_t)w[(long)t * num_idx_heads + h] * relu;",
                                "total += (int64_t)w[(long)h * num_idx_heads + t % num_idx_heads] * relu;"),
    "tie_break_reversed": ("return (x->block > y->block) - (x->block < y->block);",
                           "return (x->block < y->block) - (x->block > y->block);"),
    "own_block_not_forced": ("for (int i = 0; i < k - 1; ++i) out[n++] = cand[i].block;\n            out[n++] = own;",
                             "cand[own].score = scores[(long)t * max_blocks + own]; cand[own].block = own;\n"
                             "            qsort(cand, (size_t)own + 1, sizeof(orc_cand), cand_rank_order);\n"
                             "            for (int i = 0; i < k; ++i) out[n++] = cand[i].block;"),
    "gqa_modulo_mapping": ("int kvh = h / group;", "int kvh = h % num_kv_heads;"),
    "causal_excludes_self": ("if (pos <= p) tok_row", "if (pos < p || pos == 0) tok_row"),
    "scale_dropped": ("logit[j] = dot * sm_scale;", "logit[j] = dot;"),
    "kc_first_not_last": ("int last_in_block = (i == cu_new[s + 1] - 1) || (slot == block_size - 1);",
                          "int last_in_block = (i == cu_new[s]) || (slot == 0);"),
    "kv_swapped": ("k_pool[dst + e] = k_new[(long)i * row + e];\n                v_pool[dst + e] = v_new[(long)i * row + e];",
                   "k_pool[dst + e] = v_new[(long)i * row + e];\n                v_pool[dst + e] = k_new[(long)i * row + e];"),
    "lse_base2": ("n_tok > 0 ? m + log(denom) : -INFINITY;", "n_tok > 0 ? m + log2(denom) : -INFINITY;"),
    "lse_max_dropped": ("n_tok > 0 ? m + log(denom) : -INFINITY;", "n_tok > 0 ? log(denom) : -INFINITY;"),
    "v_rows_from_k": ("const uint16_t *vj = v_pool + (tok_row[j] * num_kv_heads + kvh) * head_dim;",
                      "const uint16_t *vj = k_pool + (tok_row[j] * num_kv_heads + kvh) * head_dim;"),
    "ids_not_sorted": ("qsort(out, (size_t)n, sizeof(int32_t), int_ascending);", "(void)int_ascending;"),
    "one_candidate_short": ("for (int i = 0; i < k - 1; ++i) out[n++] = cand[i].block;",
                            "for (int i = 0; i < k - 2; ++i) out[n++] = cand[i].block;"),
    "append_one_slot_late": ("return seq_lens[s] - n + (i - cu_new[s]);", "return seq_lens[s] - n + (i - cu_new[s]) + 1;"),
    "fp8_subnormal_as_normal": ("(e == 0) ? (int64_t)f :", "(e == 0) ? (int64_t)(8 + f) :"),
    "fp8_exponent_bias_off": ("((int64_t)(8 + f) << (e - 1))", "((int64_t)(8 + f) << e)"),
    "fp8_sign_ignored": ("return sign ? -mag : mag;", "return mag;"),
    "fp8_relu_dropped": ("__int128 relu = dot > 0 ? dot : 0;", "__int128 relu = dot;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-o", str(lib),
                           str(mutated), "-lm"])
    env = dict(os.environ, DSA_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutation {name} survived the pins:\n{r.stdout[-2000:]}"
