"""The oracle pins must catch plausible mistakes in the oracle.

Each case compiles a copy of ``oracle/attention_oracle.c`` with one planted
mistake (a dropped term, a wrong sign or index, a transposed operand, a wrong
dropout scale ...) and runs the pin suite against it in a subprocess; the
suite has to fail.  Mistakes are planted only in the oracle, on the CPU.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "attention_oracle.c")

MUTANTS = {
    "drop_minus_D_in_dS": ("double ds = p * (dp - D);", "double ds = p * dp;"),
    "causal_mask_transposed": ("(pb->causal && j > i) || block_masked(pb, bh, i, j)) {",
                               "(pb->causal && j < i) || block_masked(pb, bh, i, j)) {"),
    "causal_mask_off_by_one": ("(pb->causal && j > i) || block_masked(pb, bh, i, j)) {",
                               "(pb->causal && j >= i) || block_masked(pb, bh, i, j)) {"),
    "length_mask_off_by_one": ("if (i >= L || j >= L ||", "if (i >= L || j > L ||"),
    "padding_queries_see_keys": ("if (i >= L || j >= L ||", "if (j >= L ||"),
    "padding_keys_get_gradients": ("if (j >= L) continue; /* a padding key", "if (j > L) continue; /* a padding key"),
    "lse_without_max": ("*lse = l > 0.0 ? m + log(l) : -INFINITY;", "*lse = l > 0.0 ? log(l) : -INFINITY;"),
    "dropout_scale_inverted": ("const double inv_keep = 1.0 / (1.0 - pb->p_drop);\n    for (int c = 0; c < pb->d; ++c) o[c] = 0.0;",
                               "const double inv_keep = (1.0 - pb->p_drop);\n    for (int c = 0; c < pb->d; ++c) o[c] = 0.0;"),
    "dq_missing_scale": ("for (int c = 0; c < pb->d; ++c) dq[c] *= pb->scale;", ""),
    "dk_uses_k_not_q": ("dkj[c] += ds * elem(qi, c);", "dkj[c] += ds * elem(kj, c);"),
    "dv_without_dropout_mask": ("double pd = p * z;", "double pd = p;"),
    "softmax_not_normalised": ("return l > 0.0 ? exp(s - m) / l : 0.0;", "return l > 0.0 ? exp(s - m) : 0.0;"),
    "block_mask_transposed": ("(size_t)(i / pb->bmask_tile)) * nt + (size_t)(j / pb->bmask_tile)]",
                              "(size_t)(j / pb->bmask_tile)) * nt + (size_t)(i / pb->bmask_tile)]"),
    "block_mask_head_ignored": ("const int hm = pb->bmask_heads == 1 ? 0 : bh % pb->H;", "const int hm = 0;"),
    "key_pass_ignores_block_mask": ("if (block_masked(&pb, bh, i, j)) continue;", ""),
    "empty_row_lse_zero": ("*lse = l > 0.0 ? m + log(l) : -INFINITY;", "*lse = l > 0.0 ? m + log(l) : 0.0;"),
    "hash_constant_typo": ("C2 = (uint32_t)(uint64_t)floor((sqrt(3.0) - 1.0) * two32);",
                           "C2 = (uint32_t)(uint64_t)floor((sqrt(3.0) - 1.0) * two32) + 2u;"),
    "threshold_floor": ("double t = ceil(p * 65536.0);", "double t = floor(p * 65536.0);"),
    "pair_same_half": ("uint32_t h16 = (j & 1) ? (w >> 16) : (w & 0xffffu);", "uint32_t h16 = w & 0xffffu;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    before, after = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(before) == 1, f"mutation anchor for {name} not found exactly once"
    mutant_c = tmp_path / "mutant.c"
    mutant_c.write_text(text.replace(before, after))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so),
                    str(mutant_c), "-lm"], check=True)
    env = dict(os.environ, ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
