"""The oracle's pins must catch plausible mistakes.  Each case below plants
one mistake in a copy of the oracle's C source (dropped term, wrong sign,
wrong index, transposed operand, wrong tie-break), builds it on the CPU and
checks that at least one pin from test_oracle_pins fails against it."""
import pytest

import oracle
import test_oracle_pins as pins
from mixture_experts_layer_43_b200 import synth

MUTANTS = {
    "no_renormalisation": ("w[j] = p[ids[j]] / psel;", "w[j] = p[ids[j]];"),
    "silu_sign": ("return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    "gate_up_swapped": ("h[f] = silu(g) * u;", "h[f] = silu(u) * g;"),
    "down_transposed": (
        "load_row(down_fmt(wfmt), wd, m, d, Fh, j, row);\n"
        "            for (int f = 0; f < Fh; ++f) acc += row[f] * h[f];",
        "for (int f = 0; f < Fh; ++f) {\n"
        "                load_row(down_fmt(wfmt), wd, m, Fh, d, f, row);\n"
        "                acc += row[j] * h[f];\n            }"),
    "shared_dropped": ("for (int i = 0; i < d; ++i) o[i] += y[i];",
                       "for (int i = 0; i < d; ++i) o[i] += 0.0 * y[i];"),
    "shared_weighted_half": ("for (int i = 0; i < d; ++i) o[i] += y[i];",
                             "for (int i = 0; i < d; ++i) o[i] += 0.5 * y[i];"),
    "tie_to_higher_index": ("l[e] > l[best]) best = e;", "l[e] >= l[best]) best = e;"),
    "bias_dropped": ("if (br) acc += (double)br[e];", ""),
    "logit_sign": ("for (int i = 0; i < d; ++i) acc += xt[i] * (double)row[i];\n        if (br)",
                   "for (int i = 0; i < d; ++i) acc -= xt[i] * (double)row[i];\n        if (br)"),
    "q4_nibbles_swapped": ("int lo = blk[2 + j] & 0x0f;\n            int hi = blk[2 + j] >> 4;",
                           "int hi = blk[2 + j] & 0x0f;\n            int lo = blk[2 + j] >> 4;"),
    "q4_offset_7": ("dsc * (double)(lo - 8);", "dsc * (double)(lo - 7);"),
    "q8_codes_unsigned": ("int q = blk[2 + j] < 128 ? (int)blk[2 + j] : (int)blk[2 + j] - 256;",
                          "int q = (int)blk[2 + j];"),
    "q8_scale_bytes_not_skipped": ("int q = blk[2 + j] < 128 ? (int)blk[2 + j] : (int)blk[2 + j] - 256;",
                                   "int q = blk[j] < 128 ? (int)blk[j] : (int)blk[j] - 256;"),
    "q5_fifth_bits_swapped_halves": ("int lo = (blk[6 + j] & 0x0f) | (int)(((qh >> j) & 1u) << 4);",
                                     "int lo = (blk[6 + j] & 0x0f) | (int)(((qh >> (j + 16)) & 1u) << 4);"),
    "q5_offset_15": ("out[b * 32 + j] = dsc * (double)(lo - 16);", "out[b * 32 + j] = dsc * (double)(lo - 15);"),
    "q5_qh_bytes_not_skipped": ("int lo = (blk[6 + j] & 0x0f)", "int lo = (blk[2 + j] & 0x0f)"),
    "fp16_exponent_bias": ("ldexp(1024.0 + (double)m, e - 25)", "ldexp(1024.0 + (double)m, e - 24)"),
    "bucket_unstable": ("for (int64_t p = 0; p < n; ++p) {\n            int e = ids[p];",
                        "for (int64_t p = n - 1; p >= 0; --p) {\n            int e = ids[p];"),
    "softmax_temperature": ("p[e] = exp(l[e] - mx); z += p[e];",
                            "p[e] = exp(0.5 * (l[e] - mx)); z += p[e];"),
    "q6_nibble_halves_swapped": ("int low = (c >= 2) ? (byte >> 4) : (byte & 0x0f);",
                                 "int low = (c >= 2) ? (byte & 0x0f) : (byte >> 4);"),
    "q6_high_bits_shift": ("int high = (qh[32 * h + l] >> (2 * c)) & 3;",
                           "int high = (qh[32 * h + l] >> c) & 3;"),
    "q6_offset_31": ("out[b * 256 + i] = dsc * (double)s8 * (double)(q - 32);",
                     "out[b * 256 + i] = dsc * (double)s8 * (double)(q - 31);"),
    "q6_sub_scales_unsigned": ("int s8 = sc[i / 16] < 128 ? (int)sc[i / 16] : (int)sc[i / 16] - 256;",
                               "int s8 = (int)sc[i / 16];"),
    "q6_sub_scale_index": ("int s8 = sc[i / 16] < 128", "int s8 = sc[i / 32] < 128"),
    "q6_odd_quarter_offset": ("ql[64 * h + ((c & 1) ? 32 : 0) + l]", "ql[64 * h + ((c & 1) ? 16 : 0) + l]"),
    "f16_down_read_as_bf16": ("static int down_fmt(int wfmt) { return wfmt == ORACLE_WFMT_BF16_F16DOWN ? ORACLE_ROWS_F16 : wfmt; }",
                              "static int down_fmt(int wfmt) { return wfmt == ORACLE_WFMT_BF16_F16DOWN ? ORACLE_WFMT_BF16 : wfmt; }"),
    "routed_weight_ignored": ("o[i] += w[(int64_t)n * k + j] * y[i];", "o[i] += y[i];"),
    "routed_shared_dropped": (
        "expert_ffn(wfmt, d, Fs, sg, su, sd, s2, xt, y);\n"
        "            for (int i = 0; i < d; ++i) o[i] += y[i];",
        "expert_ffn(wfmt, d, Fs, sg, su, sd, s2, xt, y);\n"
        "            for (int i = 0; i < d; ++i) o[i] += 0.0 * y[i];"),
}


def _pins():
    yield lambda: pins.test_q4_0_golden_blocks()
    yield lambda: pins.test_q8_0_golden_blocks()
    yield lambda: pins.test_q5_0_golden_blocks()
    yield lambda: pins.test_q6_k_golden_blocks()
    yield lambda: pins.test_fp16_decode_matches_numpy_all_patterns()
    yield lambda: pins.test_softmax_renormalisation_closed_form()
    yield lambda: pins.test_swiglu_closed_form()
    yield lambda: pins.test_tie_break_lower_index()
    for sh in pins.TINY:
        yield (lambda sh=sh: pins.test_brute_force_tiny(sh))
    yield lambda: pins.test_buckets_match_sort(37, 6, 64, 2)
    yield lambda: pins.test_k_equals_E_is_dense_softmax_mixture(synth.WFMT_BF16)
    yield lambda: pins.test_k_equals_E_is_dense_softmax_mixture(synth.WFMT_BF16_F16DOWN)
    yield lambda: pins.test_single_expert_is_plain_swiglu()
    yield lambda: pins.test_shared_only_when_routed_down_is_zero()
    yield lambda: pins.test_forward_routed_is_weighted_sum_of_ffns(synth.WFMT_BF16)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.source()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    path = oracle.build_variant(src.replace(old, new, 1), str(tmp_path / f"m_{name}.so"))
    oracle.use(path)
    try:
        caught = False
        for pin in _pins():
            try:
                pin()
            except (AssertionError, ValueError):
                caught = True
                break
        assert caught, f"no pin caught the planted mistake {name}"
    finally:
        oracle.use(None)
