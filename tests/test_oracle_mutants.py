"""The pins must catch plausible mistakes in the oracle.  Each case plants one
mistake in a copy of oracle/pa_oracle.c (in-bounds edits only), builds it,
points the oracle at it and runs the pin suite, which must fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "pa_oracle.c")

MUTANTS = {
    "dropped_scale": ("scores[t] = scale * dot;", "scores[t] = dot;"),
    "softmax_sign": ("scores[t] = exp(scores[t] - m);", "scores[t] = exp(m - scores[t]);"),
    "row_off_by_one": ("((p * H + h) * bs + t % bs) * D;\n        double dot",
                       "((p * H + h) * bs + (t + 1) % bs) * D;\n        double dot"),
    "first_block_only": ("int64_t p = table[t / bs];\n        if (p < 0", "int64_t p = table[0];\n        if (p < 0"),
    "context_one_short": ("scores, q + u * D, k_cache, v_cache,\n                            block_tables + (int64_t)b * max_blocks_per_seq, len,",
                          "scores, q + u * D, k_cache, v_cache,\n                            block_tables + (int64_t)b * max_blocks_per_seq, len > 1 ? len - 1 : len,"),
    "fp16_exponent_bias": ("ldexp((double)(frac + 1024), expo - 25)", "ldexp((double)(frac + 1024), expo - 24)"),
    "no_normalisation": ("        out[d] /= l;\n", "        out[d] /= 1.0;\n"),
    "write_offset_dropped": ("uint16_t *kd = k_cache + ((block * H + h) * bs + offset) * D;",
                             "uint16_t *kd = k_cache + ((block * H + h) * bs) * D;"),
    "copy_direction": ("memmove(k_cache + dst * block_elems, k_cache + src * block_elems,",
                       "memmove(k_cache + src * block_elems, k_cache + dst * block_elems,"),
    "size_formula_factor": ("return 2 * batch * seq_len * layers * d_model * bytes_per_elem;",
                            "return batch * seq_len * layers * d_model * bytes_per_elem;"),
    "head_stride": ("const uint16_t *v = v_cache + ((p * H + h) * bs + t % bs) * D;",
                    "const uint16_t *v = v_cache + ((p * H + (h + 1) % H) * bs + t % bs) * D;"),
    "quant_levels": ("const float qmax = (float)((1 << bits) - 1);",
                     "const float qmax = (float)(1 << bits);"),
    "quant_zero_point_unrounded": ("const float z = rintf(-rmin / s);", "const float z = -rmin / s;"),
    "causal_off_by_one": ("block_tables + (int64_t)b * max_blocks_per_seq, pos + 1, h, H, D,",
                          "block_tables + (int64_t)b * max_blocks_per_seq, pos, h, H, D,"),
    "query_position": ("const int pos = context_lens[b] - n + (int)(tok - query_start_loc[b]);",
                       "const int pos = context_lens[b] - n;"),
    "dequant_sign": ("dot += h2d(q[u * D + d]) * (s * ((double)k_codes[row * D + d] - z));",
                     "dot += h2d(q[u * D + d]) * (s * ((double)k_codes[row * D + d] + z));"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mutant_c = tmp_path / "mutant.c"
    mutant_c.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-pthread",
                    "-o", str(lib), str(mutant_c), "-lm"], check=True)
    env = dict(os.environ, PA_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        os.path.join(ROOT, "tests", "test_quant_pins.py"),
                        os.path.join(ROOT, "tests", "test_prefill_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, f"pins did not catch {name}:\n{r.stdout[-2000:]}"
