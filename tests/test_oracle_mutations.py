"""Plant plausible mistakes in a copy of the oracle's C source (on the CPU)
and check that the pins reject every one of them."""
import pytest

import oracle
import oracle_pins as P

# (name, text in the oracle source, replacement)
MUTATIONS = [
    ("window_off_by_one", "p - J->window > 0) lo = p - J->window;", "p - J->window + 1 > 0) lo = p - J->window + 1;"),
    ("rope_sign", "y[i] = x[i] * c - x[i + half] * s;", "y[i] = x[i] * c + x[i + half] * s;"),
    ("rope_pairing_interleaved", "y[i + half] = x[i + half] * c + x[i] * s;", "y[i + half] = x[i + half] * c - x[i] * s;"),
    ("rope_theta_denominator", "-2.0 * (double)i / (double)rope_dims", "-2.0 * (double)i / (double)dim"),
    ("sink_dropped_from_sum", "double Z = has_sink ? exp(sigma - M) : 0.0;\n      for (int64_t j = lo; j <= p; ++j) Z += exp(s[j - lo] - M);\n      /* step 6 */",
     "double Z = 0.0;\n      for (int64_t j = lo; j <= p; ++j) Z += exp(s[j - lo] - M);\n      /* step 6 */"),
    ("v_scale_dropped", "o[d] += w * (J->v_scale * ld(J->v, vbase + d, J->f64));", "o[d] += w * ld(J->v, vbase + d, J->f64);"),
    ("softmax_scale_dv", "1.0 / sqrt((double)J->dqk)", "1.0 / sqrt((double)J->dv)"),
    ("gqa_modulo_mapping", "int32_t g = h / group;\n      const size_t qbase", "int32_t g = h % J->hkv;\n      const size_t qbase"),
    ("key_position_global", "oracle_rope(x, pos, j->rope_base", "oracle_rope(x, t, j->rope_base"),
    ("lse_without_max", "double L = M + log(Z);\n      J->lse", "double L = log(Z);\n      J->lse"),
    ("causal_excludes_self", "for (int64_t j = lo; j <= p; ++j) {\n        const double* kr = J->k_rot",
     "for (int64_t j = lo; j < p; ++j) {\n        const double* kr = J->k_rot"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = oracle.source()
    assert src.count(old) == 1, f"mutation anchor not found once: {name}"
    mutant = oracle.Variant(src.replace(old, new), str(tmp_path))
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, ZeroDivisionError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {name}"
