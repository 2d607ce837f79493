"""Plants plausible mistakes in copies of the oracle source (on the CPU) and
checks that at least one pin catches each: a dropped term, a wrong sign, a
wrong index, a transposed operand, an off-by-one window, a wrong log base.
The committed oracle source is never modified."""
import os

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "window_off_by_one": ("int64_t lo = i - (int64_t)W + 1;", "int64_t lo = i - (int64_t)W;"),
    "distance_not_deduplicated": ("if (j >= lo) continue;", "if (j > i) continue;"),
    "scale_dropped": ("s[e] = scale * dot;", "s[e] = dot;"),
    "max_not_subtracted": ("for (int64_t e = 0; e < deg; ++e) l += exp(s[e] - m);",
                           "for (int64_t e = 0; e < deg; ++e) l += exp(s[e]);"),
    "lse_log2": ("*lse = m + log(l);", "*lse = m + log2(l);"),
    "delta_sign": ("double ds = p * (dp - delta);", "double ds = p * (dp + delta);"),
    "dk_transposed_operand": ("dk[j * D + d] += scale * ds * qd[i * D + d];",
                              "dk[j * D + d] += scale * ds * kd[i * D + d];"),
    "dq_scale_dropped": ("dq[i * D + d] += scale * ds * kd[j * D + d];",
                         "dq[i * D + d] += ds * kd[j * D + d];"),
    "dv_prob_dropped": ("dv[j * D + d] += p * dod[i * D + d];",
                        "dv[j * D + d] += dod[i * D + d];"),
    "dv_wrong_row": ("dv[j * D + d] += p * dod[i * D + d];",
                     "dv[i * D + d] += p * dod[i * D + d];"),
    "delta_from_values": ("delta += dod[i * D + d] * o[d];",
                          "delta += dod[i * D + d] * vd[i * D + d];"),
    "reverse_stores_key": ("rev_colidx[fill[j]++] = (int32_t)i;",
                           "rev_colidx[fill[j]++] = (int32_t)j;"),
    "normalize_keeps_repeats": ("if (u == 0 || row[u - 1] != row[e]) row[u++] = row[e];",
                                "row[u++] = row[e];"),
    "lookahead_accepted": ("if ((int64_t)colidx[e] > i) return OR_LOOKAHEAD;",
                           "if ((int64_t)colidx[e] > i + 1) return OR_LOOKAHEAD;"),
    "negative_key_accepted": ("if (colidx[e] < 0) return OR_NEGATIVE;",
                              "if (colidx[e] < -1) return OR_NEGATIVE;"),
    "link_before_start_clamped": ("if (j < 0) continue;          /* no position before the start */",
                                  "if (j < 0) j = 0;"),
    "repeated_exponent_counted": ("if (dup) continue;", "(void)dup;"),
    "structured_row_unsorted": ("if (buf) qsort(buf, (size_t)cnt, sizeof(int32_t), cmp_i32);", ""),
    "normalize_row_unsorted": ("qsort(row, (size_t)n, sizeof(int32_t), cmp_i32);", ""),
    "reverse_descending": ("for (int64_t i = 0; i < T; ++i) /* ascending i keeps each list sorted */",
                           "for (int64_t i = T - 1; i >= 0; --i)"),
    "empty_row_lse_zero": ("*lse = -INFINITY;", "*lse = 0.0;"),
    "lse_max_dropped": ("*lse = m + log(l);", "*lse = log(l);"),
    "output_not_normalized": ("double p = exp(s[e] - m) / l;", "double p = exp(s[e] - m);"),
    "delta_dropped": ("double ds = p * (dp - delta);", "double ds = p * dp;"),
    "dq_value_for_key": ("dq[i * D + d] += scale * ds * kd[j * D + d];",
                         "dq[i * D + d] += scale * ds * vd[j * D + d];"),
    "dk_scale_dropped": ("dk[j * D + d] += scale * ds * qd[i * D + d];",
                         "dk[j * D + d] += ds * qd[i * D + d];"),
    "bwd_prob_without_lse": ("double p = exp(s[e] - lse);", "double p = exp(s[e]);"),
    "dist_sign_flipped": ("w[e] = -scale * dist2;", "w[e] = scale * dist2;"),
    "dist_not_squared": ("dist2 += diff * diff;", "dist2 += fabs(diff);"),
    "dist_grad_factor_two_dropped": ("double g = dse * (-2.0 * scale * (ad[i * 3 + x] - cd[j * 3 + x]));",
                                     "double g = dse * (-scale * (ad[i * 3 + x] - cd[j * 3 + x]));"),
    "dist_key_grad_sign": ("dc[j * 3 + x] -= g;", "dc[j * 3 + x] += g;"),
    "dist_key_grad_wrong_row": ("dc[j * 3 + x] -= g;", "dc[i * 3 + x] -= g;"),
    "dist_delta_dropped": ("double dse = pe * (dpe - dlt);", "double dse = pe * dpe;"),
    "dist_scale_dropped": ("w[e] = -scale * dist2;", "w[e] = -dist2;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, "mutation site not found: " + name
    mpath = tmp_path / "oracle_mutant.c"
    mpath.write_text(src.replace(before, after))
    lib = oracle.build(str(mpath), str(tmp_path / "liboracle_mutant.so"))
    o = oracle.Oracle(lib)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, oracle.OracleError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, "no pin caught mutant " + name
