"""The oracle of the steps beside the attention kernel (FP8 blockwise dequant,
fused-QKV split, MoE router) against its pins, and planted mistakes in copies
of it (on the CPU) against the same pins."""
import os
import types

import pytest

import neighbors_pins as P
from oracle import neighbors

SRC = os.path.join(os.path.dirname(neighbors.__file__), "neighbors.py")


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=[p.__name__ for p in P.ALL_PINS])
def test_pin(pin):
    pin(neighbors)


# (name, text in the oracle source, replacement)
MUTATIONS = [
    ("e4m3_bias_8", "np.exp2(e.astype(np.float64) - 7.0)", "np.exp2(e.astype(np.float64) - 8.0)"),
    ("e4m3_no_subnormals", "out = np.where(e == 0, sub, normal)", "out = normal"),
    ("e4m3_mantissa_16ths", "normal = sign * (1.0 + m / 8.0)", "normal = sign * (1.0 + m / 16.0)"),
    ("dequant_block_transposed", "s[rows[:, None], cols[None, :]]", "s[np.minimum(np.arange(M) // b1, s.shape[0] - 1)[:, None], np.minimum(np.arange(N) // b0, s.shape[1] - 1)[None, :]]"),
    ("split_k_before_q", "q = x[:, :, :group * dqk]", "q = x[:, :, dqk:dqk + group * dqk]"),
    ("split_v_k_swapped", "k = x[:, :, group * dqk:group * dqk + dqk]", "k = x[:, :, group * dqk + dv:group * dqk + dv + dqk]"),
    ("split_heads_transposed", ".reshape(T, hkv, group, dqk).reshape(T, hq, dqk)", ".reshape(T, hkv, group, dqk).transpose(0, 2, 1, 3).reshape(T, hq, dqk)"),
    ("route_bias_ignored", "key = (s64.astype(np.float32) + bias[None, :])", "key = (s64.astype(np.float32) + 0 * bias[None, :])"),
    ("route_bias_subtracted", "key = (s64.astype(np.float32) + bias[None, :])", "key = (s64.astype(np.float32) - bias[None, :])"),
    ("route_ascending", "key=lambda e: (-float(key[t, e]), e)", "key=lambda e: (float(key[t, e]), e)"),
    ("route_weights_with_bias", "sel = s64[t, order]", "sel = s64[t, order] + bias[order]"),
    ("route_no_normalise", "w[t] = sel / sel.sum() if normalize else sel", "w[t] = sel"),
    ("route_softmax_scores", "s64 = sigmoid_f64(logits)", "s64 = np.exp(logits.astype(np.float64)) / np.exp(logits.astype(np.float64)).sum(1, keepdims=True)"),
    ("route_ties_to_higher_index", "key=lambda e: (-float(key[t, e]), e)", "key=lambda e: (-float(key[t, e]), -e)"),
    ("proj_weight_not_transposed", "return xf @ wf.T", "return xf @ wf.reshape(wf.shape[1], wf.shape[0])"),
    ("proj_drops_last_feature", "return xf @ wf.T", "return xf[:, :-1] @ wf[:, :-1].T"),
    ("proj_rounds_to_fp32", "return xf @ wf.T", "return (xf @ wf.T).astype(np.float32).astype(np.float64)"),
    ("proj_bf16_decoded_as_fp16", "b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)\n    return b.view(np.float32).astype(np.float64)",
     "return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutant_is_caught(name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {name}"
    mutant = types.ModuleType(f"neighbors_{name}")
    exec(compile(src.replace(old, new), f"<{name}>", "exec"), mutant.__dict__)
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, IndexError, ZeroDivisionError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {name}"
