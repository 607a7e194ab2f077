"""Each plausible mistake planted in a copy of the oracle must fail at least one pin.

The copies are built from ``oracle/oracle.c`` by replacing one exact snippet,
compiled with gcc into a temporary directory and run on the CPU only.
"""
import os
import subprocess
import sys

import pytest

import oracle
from oracle_pins import ALL_CHECKS

MUTANTS = {
    "head_grouping_interleaved": ("const int h = g / group;", "const int h = g % num_kv_heads;"),
    "block_index_swapped": ("block_tables[(size_t)s * max_blocks_per_seq + t / block_size];\n                const int off = t % block_size;\n                if",
                            "block_tables[(size_t)s * max_blocks_per_seq + t % block_size];\n                const int off = t / block_size;\n                if"),
    "scale_dropped": ("x[t] = scale * dot;", "x[t] = dot;"),
    "v_read_from_k": ("o[i] += w * elem(v_cache, kv_dtype, voff + i, vsc);",
                      "o[i] += w * elem(k_cache, kv_dtype, voff + i, vsc);"),
    "head_scale_of_wrong_head": ("const double ksc = k_head_scales ? (double)k_head_scales[h] : k_scale;",
                                 "const double ksc = k_head_scales ? (double)k_head_scales[0] : k_scale;"),
    "last_token_dropped": ("const int L = seq_lens[s];", "const int L = seq_lens[s] > 1 ? seq_lens[s] - 1 : seq_lens[s];"),
    "no_normalisation": ("o[i] /= denom;", "o[i] /= 1.0;"),
    "no_max_subtraction": ("const double w = exp(x[t] - m);", "const double w = exp(x[t]);"),
    "e4m3_sign_dropped": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);\n    return s ? -v : v;",
                          "v = ldexp(1.0 + (double)m / 8.0, e - 7);\n    return v;"),
    "e4m3_ties_to_odd": ("double vlo = e4m3_pos[lo], vhi = e4m3_pos[hi];\n    double midpoint = 0.5 * (vlo + vhi); "
                         "/* exact: both are short binary fractions */\n    int code;\n    if (a < midpoint)\n"
                         "        code = lo;\n    else if (a > midpoint)\n        code = hi;\n    else\n"
                         "        code = (lo & 1) ? hi : lo;",
                         "double vlo = e4m3_pos[lo], vhi = e4m3_pos[hi];\n    double midpoint = 0.5 * (vlo + vhi); "
                         "/* exact: both are short binary fractions */\n    int code;\n    if (a < midpoint)\n"
                         "        code = lo;\n    else if (a > midpoint)\n        code = hi;\n    else\n"
                         "        code = (lo & 1) ? lo : hi;"),
    "e5m2_sign_dropped": ("v = ldexp(1.0 + (double)m / 4.0, e - 15);\n    return s ? -v : v;",
                          "v = ldexp(1.0 + (double)m / 4.0, e - 15);\n    return v;"),
    "e5m2_bias_off_by_one": ("v = ldexp(1.0 + (double)m / 4.0, e - 15);", "v = ldexp(1.0 + (double)m / 4.0, e - 14);"),
    "e5m2_ties_to_odd": ("double vlo = e5m2_pos[lo], vhi = e5m2_pos[hi];\n    double midpoint = 0.5 * (vlo + vhi);\n"
                         "    int code;\n    if (a < midpoint)\n        code = lo;\n    else if (a > midpoint)\n"
                         "        code = hi;\n    else\n        code = (lo & 1) ? hi : lo;",
                         "double vlo = e5m2_pos[lo], vhi = e5m2_pos[hi];\n    double midpoint = 0.5 * (vlo + vhi);\n"
                         "    int code;\n    if (a < midpoint)\n        code = lo;\n    else if (a > midpoint)\n"
                         "        code = hi;\n    else\n        code = (lo & 1) ? lo : hi;"),
    "int8_ties_away_from_zero": ("if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0))", "if (frac >= 0.5)"),
    "int8_clamps_at_128": ("    if (x >= 127.0f)\n        return 127;", "    if (x >= 128.0f)\n        return 127;"),
    "causal_limit_off_by_one": ("const int Lq = L - q_len + 1 + j;", "const int Lq = L - q_len + j;"),
    "e5m2_saturates_to_infinity": ("if (a >= e5m2_pos[123])\n        return sign | 123;",
                                   "if (a >= e5m2_pos[123])\n        return sign | 124;"),
    "e4m3_bias_off_by_one": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "fp8_scale_multiplied": ("const float ky = kx / (k_head_scales ? k_head_scales[h] : k_scale);",
                             "const float ky = kx * (k_head_scales ? k_head_scales[h] : k_scale);"),
    "append_offset_wrong": ("const int64_t blk = slot / block_size, off = slot % block_size;",
                            "const int64_t blk = slot / block_size, off = (slot + 1) % block_size;"),
    "negative_slot_written": ("if (slot < 0)\n            continue;", "if (slot < -1000)\n            continue;"),
    "lse_without_max": ("= m + log(denom);", "= log(denom);"),
    "lse_of_weights_not_scores": ("= m + log(denom);", "= m + log(denom / Lq);"),
    "dequant_scale_ignored": ("return orc_e4m3_value(((const uint8_t*)base)[i]) * scale;",
                              "return orc_e4m3_value(((const uint8_t*)base)[i]);"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, f"snippet for {name} not found exactly once"
    msrc = tmp_path / f"oracle_{name}.c"
    msrc.write_text(src.replace(old, new))
    return oracle.build(str(msrc), str(tmp_path / f"liboracle_{name}.so"), force=True)


RUNNER = """
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle
from oracle_pins import ALL_CHECKS
lib = oracle.load({so!r})
failed = []
for check in ALL_CHECKS:
    try:
        check(lib)
    except (AssertionError, oracle.OracleError):
        failed.append(check.__name__)
print("FAILED:" + ",".join(failed))
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    so = _build_mutant(tmp_path, name, old, new)
    here = os.path.dirname(os.path.abspath(__file__))
    code = RUNNER.format(root=os.path.dirname(here), tests=here, so=so)
    # a separate process: a planted indexing mistake may corrupt memory or abort
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    if r.returncode != 0:
        return  # the planted mistake crashed the oracle: caught
    line = [l for l in r.stdout.splitlines() if l.startswith("FAILED:")][-1]
    failed = [f for f in line[len("FAILED:"):].split(",") if f]
    assert failed, f"planted mistake {name} passed every pin"
