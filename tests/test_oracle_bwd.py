"""The oracle's backward against its pins, and planted mistakes in a copy of
its C source that the pins must reject (CPU only)."""
import pytest

import oracle
import oracle_bwd_pins as B


@pytest.mark.parametrize("pin", B.BWD_PINS, ids=[p.__name__ for p in B.BWD_PINS])
def test_bwd_pin(pin):
    pin(oracle)


# (name, text in the oracle source, replacement)
MUTATIONS = [
    ("row_dot_term_dropped", "double ds = pj * (dpj - D + gl);", "double ds = pj * (dpj + gl);"),
    ("lse_gradient_dropped", "double ds = pj * (dpj - D + gl);", "double ds = pj * (dpj - D);"),
    ("dv_without_v_scale", "dvv[vrow + d] += v_scale * pj * go[d];", "dvv[vrow + d] += pj * go[d];"),
    ("dk_without_softmax_scale", "dkr[d] += ds * qr[d] * inv_sqrt_d;", "dkr[d] += ds * qr[d];"),
    ("dq_not_rotated_back", "oracle_rope_transpose(dqr, p, rope_base, rope_dims, dqk, dq + (t * hq + h) * dqk);",
     "oracle_rope(dqr, p, rope_base, rope_dims, dqk, dq + (t * hq + h) * dqk);"),
    ("dk_rotated_at_query_position",
     "oracle_rope_transpose(dk_rot + (t * hkv + g) * dqk, p, rope_base",
     "oracle_rope_transpose(dk_rot + (t * hkv + g) * dqk, 0, rope_base"),
    ("dsink_sign", "if (has_sink) dsink[h] += exp(sigma - L) * (gl - D);", "if (has_sink) dsink[h] += exp(sigma - L) * (D - gl);"),
    ("transpose_same_direction", "oracle_rope(x, -pos, base, rope_dims, dim, y);", "oracle_rope(x, pos, base, rope_dims, dim, y);"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_bwd_mutant_is_caught(name, old, new, tmp_path):
    src = oracle.source()
    assert src.count(old) == 1, f"mutation anchor not found once: {name}"
    mutant = oracle.Variant(src.replace(old, new), str(tmp_path))
    caught = []
    for pin in B.BWD_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, ZeroDivisionError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {name}"
