"""Plant plausible mistakes in a copy of the oracle and check a pin catches each.

Every mutant is the oracle's C source with one textual edit (a dropped term,
a wrong sign, a wrong index, a transposed mapping), compiled into a temporary
directory.  The real oracle is never modified.  A mutant that passes every
pin would mean the pins cannot tell that mistake from the correct oracle.
"""
import os
import subprocess

import pytest

import oracle
from oracle_checks import ALL_CHECKS

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "drop_scale": ("s[j - j0] = scale * dot;", "s[j - j0] = dot;"),
    "exp_sign": ("double w = exp(s[j - j0] - m);", "double w = exp(m - s[j - j0]);"),
    "gqa_mapping": ("hq = (int)(r % H_q), g = hq / G;", "hq = (int)(r % H_q), g = hq % H_kv;"),
    "no_normalise": ("for (int i = 0; i < d; ++i) o[i] /= den;", ""),
    "row_in_page": ("ORC_PAGE_TOKENS + (j % ORC_PAGE_TOKENS)) * (size_t)d",
                    "ORC_PAGE_TOKENS + (j / ORC_PAGE_TOKENS)) * (size_t)d"),
    "ignore_block_table": ("int phys = block_table[(size_t)b * max_blocks + logical];\n    if (phys < 0 || phys >= num_blocks) return -1;",
                           "int phys = logical; (void)block_table; (void)num_blocks;"),
    "lse_without_max": ("if (lse) lse[r] = m + log(den);", "if (lse) lse[r] = log(den);"),
    "merge_weight": ("double w = exp(L[s] - LSE);", "double w = exp(L[s] - M);"),
    "f16_bias": ("ldexp((double)(1024 + frac), expo - 25)", "ldexp((double)(1024 + frac), expo - 24)"),
    "f16_subnormal": ("ldexp((double)frac, -24)", "ldexp((double)frac, -25)"),
    "bf16_shift": ("((uint32_t)b) << 16", "((uint32_t)b) << 15"),
    "append_row": ("int row = pos % ORC_PAGE_TOKENS;", "int row = pos / ORC_PAGE_TOKENS;"),
    "append_head_stride": ("size_t src = ((size_t)b * H_kv + h) * (size_t)d;",
                           "size_t src = ((size_t)h * B + b) * (size_t)d;"),
    "tiled_no_rescale": ("ssum = ssum * exp_old + tile_sum;", "ssum = ssum + tile_sum;"),
    "kv_bytes_no_kv_factor": ("return 2LL * (long long)dtype_size * layers * heads * d_head;",
                              "return (long long)dtype_size * layers * heads * d_head;"),
    "fp8_scale_max": ("volatile float s = mx / 448.0f;", "volatile float s = mx / 240.0f;"),
    "fp8_group_index": ("const float *sk = ks + off / d * ng;", "const float *sk = ks + off / d;"),
    "fp8_round_down": ("double r = rint(a / ldexp(1.0, E - 3));", "double r = floor(a / ldexp(1.0, E - 3));"),
    "fp8_decode_bias": ("else v = ldexp((double)(8 + m), e - 10);", "else v = ldexp((double)(8 + m), e - 9);"),
    "int8_scale_max": ("volatile float s = mx / 127.0f;", "volatile float s = mx / 128.0f;"),
    "int8_round_floor": ("double r = rint((double)x);", "double r = floor((double)x);"),
    "int8_decode_unsigned": ("return (double)(int8_t)c;", "return (double)c;"),
    "int8_clamp": ("if (r > 127.0) r = 127.0;", "if (r > 128.0) r = 128.0;"),
    "int8_nan_code": ("if (isnan(x)) return 0;", "if (isnan(x)) return 0x7F;"),
    "int4_scale_max": ("volatile float s = mx / 7.0f;", "volatile float s = mx / 8.0f;"),
    "int4_clamp": ("if (r > 7.0) r = 7.0;", "if (r > 8.0) r = 8.0;"),
    "int4_round_floor": ("double r = rint((double)x);               /* nearest, ties to even */\n    if (r > 7.0)",
                         "double r = floor((double)x);               /* nearest, ties to even */\n    if (r > 7.0)"),
    "int4_nibble_order": ("if (ch % 2 == 0) *byte = (uint8_t)((*byte & 0xF0) | nib);",
                          "if (ch % 2 == 1) *byte = (uint8_t)((*byte & 0xF0) | nib);"),
    "int4_decode_unsigned": ("return (double)(v >= 8 ? v - 16 : v);", "return (double)v;"),
    "int4_value_nibble": ("return dec((uint8_t)((i % 2 == 0) ? (byte & 15) : (byte >> 4)));",
                          "return dec((uint8_t)((i % 2 == 0) ? (byte >> 4) : (byte & 15)));"),
    "max_skips_first": ("for (int t = 0; t < n; ++t) if (s[t] > m) m = s[t];",
                        "for (int t = 1; t < n; ++t) if (s[t] > m) m = s[t];"),
}


@pytest.fixture(scope="module")
def source():
    with open(SRC, encoding="utf-8") as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    # the first occurrence is the plain attention's (the 8-bit path repeats a
    # few lines after it); one planted mistake per mutant
    assert source.count(old) >= 1, f"mutation site for {name} not found in oracle.c"
    src = tmp_path / "mutant.c"
    src.write_text(source.replace(old, new, 1), encoding="utf-8")
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                    "-ffp-contract=off", str(src), "-o", str(lib), "-lm"], check=True)
    caught = []
    with oracle.using_library(str(lib)):
        for check in ALL_CHECKS:
            try:
                check()
            except AssertionError:
                caught.append(check.__name__)
                break
            except oracle.OracleError:
                caught.append(check.__name__ + " (error)")
                break
    assert caught, f"no pin detects the planted mistake {name!r}"
