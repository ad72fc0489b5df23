"""Pin strength: plant one plausible mistake at a time in a copy of the oracle's C
source, build it, and check that the pin suite (tests/test_oracle_pins.py) fails.

Each mutant is a dropped term, a wrong sign, index or constant, or a wrong
rounding rule -- the kinds of slip that would otherwise let the oracle agree with
a CUDA kernel carrying the same slip.
"""
import os
import subprocess
import sys

import pytest

from oracle import build as obuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "fwht_no_stage_scale": ("row[j] = (u + v) * c;", "row[j] = (u + v);"),
    "fwht_wrong_sign": ("row[j + h] = (u - v) * c;", "row[j + h] = (v - u) * c;"),
    "fwht_skips_first_stage": ("for (int64_t h = 1; h < K; h *= 2) {", "for (int64_t h = 2; h < K; h *= 2) {"),
    "rmsnorm_sum_not_mean": ("float mean = ss / (float)K;", "float mean = ss;"),
    "rmsnorm_no_gain": ("yr[k] = g ? v * g[k] : v;", "yr[k] = v;"),
    "int8_q_is_128": ("static float q_int8(void) { return 127.0f; }", "static float q_int8(void) { return 128.0f; }"),
    "int4_sum_not_mean": ("float beta = sum / (float)K;", "float beta = sum;"),
    "int4_q_is_8": ("return (float)sqrt(7.0); }", "return 8.0f; }"),
    "round_half_away": ("static float rne(float v) { return nearbyintf(v); }",
                        "static float rne(float v) { return roundf(v); }"),
    "int4_clip_low": ("lo = -8.0f;", "lo = -7.0f;"),
    "pack_wrong_bit_index": ("packed[n * row_bytes + 4 * w + i / 2] |= (uint8_t)(code << (4 * (i % 2) + 2 * h));",
                             "packed[n * row_bytes + 4 * w + i / 2] |= (uint8_t)(code << (2 * (i % 2) + 4 * h));"),
    "gemm_packed_no_offset": ("s += (int32_t)q[m * K + k] * (int32_t)(code - 1);",
                              "s += (int32_t)q[m * K + k] * (int32_t)(code);"),
    "alpha_sum_not_mean": ("return (float)(sum / (double)count);", "return (float)(sum);"),
    "dequant_times_q": ("float f = (alpha * scale_x[m]) / Q;", "float f = (alpha * scale_x[m]) * Q;"),
    "swiglu_sigmoid_only": ("float silu = gv / den;", "float silu = 1.0f / den;"),
    "swiglu_wrong_exp_sign": ("float den = 1.0f + expf(-gv);", "float den = 1.0f + expf(gv);"),
    "swiglu_drops_up": ("out[i] = silu * up[i];", "out[i] = silu;"),
    "kv_bos_not_int8": ("const int rbits = (r % S == 0) ? 8 : bits;\n        float stat",
                        "const int rbits = bits;\n        float stat"),
    "kv_3bit_q_is_4": ("else { Q = 3.0f; lo = -4.0f; hi = 3.0f; }", "else { Q = 4.0f; lo = -4.0f; hi = 3.0f; }"),
    "kv_step_without_eps": ("float scale = stat + eps;\n        float s = Q / scale;",
                            "float scale = stat;\n        float s = Q / (stat + eps);"),
    "bf16_truncates": ("if (dropped > 0x8000u) r = kept + 1;", "if (0) r = kept + 1;"),
    "tl2_sign_inverted": ("const unsigned idx = (unsigned)(v < 0 ? -v : v), sign = v < 0 ? 1u : 0u;",
                          "const unsigned idx = (unsigned)(v < 0 ? -v : v), sign = v > 0 ? 1u : 0u;"),
    "tl2_digits_reversed": ("v = 9 * w[0] + 3 * w[1] + w[2];", "v = w[0] + 3 * w[1] + 9 * w[2];"),
    "tl2_sign_word_offset": ("grp[16 + jj / 8] |= (uint8_t)(sign << (jj % 8));",
                             "grp[12 + jj / 8] |= (uint8_t)(sign << (jj % 8));"),
    "bf16_ties_away": ("else if (dropped == 0x8000u && (kept & 1u)) r = kept + 1;",
                       "else if (dropped == 0x8000u) r = kept + 1;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(obuild.SRC).read()
    assert src.count(before) == 1, f"mutation site for {name} not unique/absent"
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(src.replace(before, after))
    lib = obuild.build(force=True, src=str(mut_src), out=str(tmp_path / "libmutant.so"))
    env = dict(os.environ, ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not slow",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
