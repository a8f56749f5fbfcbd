"""The oracle's pins catch plausible mistakes.

Each case copies ``oracle/oracle.c``, plants one mistake of the kind a
restatement of the definition could contain (a dropped term, a wrong sign,
index or operand, an off-by-one mask, a wrong page address), builds it, and
runs the pin suite against that build.  The suite must fail for every
mutant; the unmodified source must pass it (``test_oracle_pins.py``).
Everything runs on the CPU.
"""
import os
import subprocess
import sys

import pytest

from oracle import build as oracle_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = [os.path.join(ROOT, "tests", "test_oracle_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_variant_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_append_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_fp8_pins.py")]

MUTANTS = {
    "scale_dropped": ("s[j] = scale * dot;", "s[j] = dot;"),
    "causal_excludes_diagonal": ("if (causal && j > i)", "if (causal && j >= i)"),
    "gqa_head_modulo": ("int kh = h / group;\n", "int kh = h % Hkv;\n"),
    "lse_without_max": ("*lse_out = m + log(z);", "*lse_out = log(z);"),
    "no_normalisation": ("p[j] = p[j] / z;", "p[j] = p[j];"),
    "scores_transposed_operands": ("dot += elem(q, qrow + (size_t)c, qdtype) * elem(k, krows[j] + (size_t)c, dtype);",
                                   "dot += elem(q, krows[j] + (size_t)c, qdtype) * elem(k, qrow + (size_t)c, dtype);"),
    "exp_sign_flipped": ("p[j] = exp(s[j] - m);", "p[j] = exp(m - s[j]);"),
    "wrong_query_head": ("size_t qrow = ((size_t)t * (size_t)Hq + (size_t)h) * (size_t)d;",
                         "size_t qrow = ((size_t)t * (size_t)Hq + (size_t)(Hq - 1 - h)) * (size_t)d;"),
    "page_slot_wrong": ("int64_t slot = t % page_size;", "int64_t slot = (t / page_size) % page_size;"),
    "decode_drops_last_token": ("int64_t n = seq_lens[b];", "int64_t n = seq_lens[b] - (seq_lens[b] > 1);"),
    "values_reversed": ("acc += p[j] * elem(v, vrows[j] + (size_t)c, dtype);",
                        "acc += p[j] * elem(v, vrows[n - 1 - j] + (size_t)c, dtype);"),
    "keys_ignore_sequence_start": ("kr[n] = ((size_t)(start + j) * (size_t)Hkv + (size_t)kh) * (size_t)d;",
                                   "kr[n] = ((size_t)(j) * (size_t)Hkv + (size_t)kh) * (size_t)d;"),
    # mask variants (skill page, section 3.3)
    "window_left_off_by_one": ("if (window_left >= 0 && j < i - window_left)",
                               "if (window_left >= 0 && j <= i - window_left)"),
    "window_right_off_by_one": ("if (window_right >= 0 && j > i + window_right)",
                                "if (window_right >= 0 && j > i + window_right + 1)"),
    "window_sides_swapped": ("if (window_left >= 0 && j < i - window_left)",
                             "if (window_right >= 0 && j < i - window_right)"),
    "softcap_without_outer_factor": ("s[j] = softcap * tanh(s[j] / softcap);",
                                     "s[j] = tanh(s[j] / softcap);"),
    "softcap_before_scale": ("s[j] = scale * dot;\n        if (softcap > 0.0)\n            s[j] = softcap * tanh(s[j] / softcap);",
                             "s[j] = dot;\n        if (softcap > 0.0)\n            s[j] = softcap * tanh(s[j] / softcap);\n        s[j] *= scale;"),
    "alibi_sign_flipped": ("bias[n] = -slope * fabs((double)(i - j));",
                                 "bias[n] = slope * fabs((double)(i - j));"),
    "alibi_without_abs": ("bias[n] = -slope * fabs((double)(i - j));",
                          "bias[n] = -slope * ((double)(i - j));"),
    "alibi_slope_of_kv_head": ("double slope = alibi ? alibi_slope(alibi, alibi_stride, b, h) : 0.0;",
                               "double slope = alibi ? alibi_slope(alibi, alibi_stride, b, kh) : 0.0;"),
    "alibi_batch_rows_ignored": ("return (double)alibi[(size_t)b * (size_t)stride + (size_t)h];",
                                 "return (double)alibi[(size_t)h];"),
    "alibi_before_cap": ("        if (softcap > 0.0)\n            s[j] = softcap * tanh(s[j] / softcap);\n        if (bias)\n            s[j] += bias[j];",
                         "        if (bias)\n            s[j] += bias[j];\n        if (softcap > 0.0)\n            s[j] = softcap * tanh(s[j] / softcap);"),
    # decode with cache append and RoPE (skill page, section 3.5)
    "rope_sin_sign": ("out[a] = x[a] * co - x[b] * si;", "out[a] = x[a] * co + x[b] * si;"),
    "rope_half_pairs_adjacent": ("int b = interleaved ? 2 * i + 1 : i + rd / 2;",
                                 "int b = interleaved ? 2 * i + 1 : i + 1;"),
    "rope_interleaved_pairs_half": ("int a = interleaved ? 2 * i : i;", "int a = i;"),
    "append_one_slot_late": ("int64_t slot = pos % page_size;", "int64_t slot = (pos + 1) % page_size;"),
    "append_not_attended": ("int64_t n = (int64_t)cache_seqlens[b] + 1;",
                            "int64_t n = (int64_t)cache_seqlens[b] + (cache_seqlens[b] == 0);"),
    "query_not_rotated": ("            if (co)\n                rope_vec(tmp, rot, d, rotary_dim, interleaved, co, si);\n            else\n                memcpy(rot, tmp, (size_t)d * sizeof(double));\n            for (int c = 0; c < d; ++c)\n                qr[",
                          "            memcpy(rot, tmp, (size_t)d * sizeof(double));\n            for (int c = 0; c < d; ++c)\n                qr["),
    "value_rotated_like_key": ("v_pages[dst + (size_t)c] = v_new[src + (size_t)c];",
                               "v_pages[dst + (size_t)c] = bf16_bits(round_bf16(rot[c]));"),
    "bf16_rounding_truncates": ("double r = nearbyint(scaled);", "double r = trunc(scaled);"),
    # FP8 inputs
    "e4m3_bias_off_by_one": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_subnormal_scale": ("v = ldexp((double)m / 8.0, -6);", "v = ldexp((double)m / 8.0, -7);"),
    "e4m3_mantissa_width": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 16.0, e - 7);"),
    "fp8_value_descale_dropped": ("vd[i] = v_descale * oracle_e4m3_value(v[i]);", "vd[i] = oracle_e4m3_value(v[i]);"),
    "fp8_key_descale_on_query": ("kd[i] = k_descale * oracle_e4m3_value(k[i]);", "kd[i] = q_descale * oracle_e4m3_value(k[i]);"),
}


@pytest.fixture(scope="module")
def source():
    with open(oracle_build.SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, source, tmp_path):
    old, new = MUTANTS[name]
    # the first occurrence is the main path (attend_one_row / prefill_rows come
    # first in the file; oracle_prefill_probs repeats some lines further down)
    assert source.count(old) >= 1, f"mutation site for {name} not found"
    src = tmp_path / "oracle_mutant.c"
    src.write_text(source.replace(old, new, 1))
    lib = oracle_build.compile_oracle(str(src), str(tmp_path / "liboracle_mutant.so"))
    env = dict(os.environ, ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins accepted mutant {name}:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout, r.stdout[-2000:]
