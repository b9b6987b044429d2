"""The oracle's pins must catch plausible mistakes.

Each case copies oracle.c, plants one mistake with a text substitution,
builds the copy with gcc and runs the pin suite (tests/test_oracle.py)
against it in a subprocess; the suite has to fail.  Nothing here touches a
GPU or the CUDA library.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "scale_dropped": ("s_out[i] = sc * acc;", "s_out[i] = acc;"),
    "gqa_head_map_modulo": ("int G = Hq / Hkv, kvh = h / G;", "int G = Hq / Hkv, kvh = h % Hkv; (void)G;"),
    "ties_to_higher_position": ("return (x->i > y->i) - (x->i < y->i);", "return (x->i < y->i) - (x->i > y->i);"),
    "tail_over_kept_mass": ("*tail_r = z_tail / (z_k + z_tail);", "*tail_r = z_tail / z_k;"),
    "softmax_over_all_keys": ("double p = exp(sp[j].s - m) / z_k;", "double p = exp(sp[j].s - m) / (z_k + z_tail);"),
    "causal_off_by_one": ("return seq_len - Q + qpos + 1;", "return seq_len - Q + qpos + (qpos > 0);"),
    "values_from_keys": ("attend_prefix(sp, vis, kk, v_cache, dtype, voff, d, out + (size_t)r * d, tail ? tail + r : NULL,\n"
                         "                          idx + (size_t)r * k, k, sel);",
                         "attend_prefix(sp, vis, kk, k_cache, dtype, voff, d, out + (size_t)r * d, tail ? tail + r : NULL,\n"
                         "                          idx + (size_t)r * k, k, sel);"),
    "q_index_transposed": ("size_t qoff = (((size_t)b * Q + qpos) * Hq + h) * d;",
                           "size_t qoff = (((size_t)b * Hq + h) * Q + qpos) * d;"),
    "block_mean_over_full_size": ("bk[(size_t)j * d + c] = hi > lo ? acc / (double)(hi - lo) : 0.0;",
                                  "bk[(size_t)j * d + c] = hi > lo ? acc / (double)block_size : 0.0;"),
    "certified_k_one_too_many": ("                    kk = j + 1;\n", "                    kk = j + 1 < cap ? j + 2 : cap;\n"),
    "certified_mass_of_capped_prefix": ("for (int j = 0; j < vis; j++) z += exp(sp[j].s - m);",
                                        "for (int j = 0; j < (k_max < vis ? k_max : vis); j++) z += exp(sp[j].s - m);"),
    "hisa_first_blocks_not_best": ("for (int j = 0; j < nk; j++) kept[j] = sb[j].i;\n            qsort(kept, (size_t)nk",
                                   "for (int j = 0; j < nk; j++) kept[j] = j;\n            qsort(kept, (size_t)nk"),
    "hisa_candidates_all_blocks": ("            for (int j = 0; j < nk; j++) {\n                int lo = kept[j] * block_size, hi = lo + block_size;\n                if (hi > Lb) hi = Lb;\n                for (int i = lo; i < hi; i++) {\n                    sp[nc]",
                                   "            for (int j = 0; j < nblk; j++) {\n                int lo = j * block_size, hi = lo + block_size;\n                if (hi > Lb) hi = Lb;\n                for (int i = lo; i < hi; i++) {\n                    sp[nc]"),
    "indexer_relu_dropped": ("(dot > 0.0 ? dot : 0.0)", "dot"),
    "indexer_weights_ignored": ("acc += (double)w_idx[(size_t)u * H_I + j] * (dot > 0.0 ? dot : 0.0);",
                                "acc += (dot > 0.0 ? dot : 0.0);"),
    "current_block_not_forced": ("kept[nk] = nblk - 1; /* the current block */",
                                 "kept[nk] = nk < nblk - 1 ? sp[nk].i : nblk - 1;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mut_c = tmp_path / "oracle_mutant.c"
    mut_c.write_text(src.replace(old, new))
    so = tmp_path / "oracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
                           "-o", str(so), str(mut_c), "-lm"])
    env = dict(os.environ, ORACLE_LIB_OVERRIDE=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
