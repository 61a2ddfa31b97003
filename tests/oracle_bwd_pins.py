"""Pins of the oracle's backward (gradients of the attention forward).

None retypes the gradient formulas: the gradients are checked against
central finite differences of the FP64 forward oracle, against invariances of
the forward (a common shift of every key's pass-through dims or of every V
row), and against the closed forms of a one-key window.  Each pin takes an
oracle-like object (the module, or a Variant built from a mutated copy)."""
from __future__ import annotations

import numpy as np

import oracle
from global_attention_moe_b200 import synth


def _case(lengths, hq, hkv, seed, window, base, sink):
    rng = np.random.default_rng(seed)
    T = int(sum(lengths))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    # BF16-representable values, so the FP64 and BF16 forms see the same numbers
    f = lambda shape, s: synth.bf16_bits_to_f32(synth.f32_to_bf16_bits((rng.standard_normal(shape) * s).astype(np.float32))).astype(np.float64)
    q, k, v = f((T, hq, 192), 1.0), f((T, hkv, 192), 1.0), f((T, hkv, 128), 1.0)
    # sinks on a 1/8 grid: sink +- 2^-12 is exact in FP32
    sk = (np.round(rng.standard_normal(hq) * 8) / 8).astype(np.float32) if sink else None
    return q, k, v, sk, cu, window, base


def _loss(O, q, k, v, sk, cu, window, base, go, gl):
    out, lse = O.attn_fwd_f64(q, k, v, sk, cu, window, base, 64, 0.707, threads=1)
    return float(np.sum(out * go) + (np.sum(lse * gl) if gl is not None else 0.0))


def _fd_check(O, case, seed, n_coords=24, with_dlse=True):
    q, k, v, sk, cu, window, base = case
    rng = np.random.default_rng(seed)
    out, lse = O.attn_fwd_f64(q, k, v, sk, cu, window, base, 64, 0.707, threads=1)
    go = rng.standard_normal(out.shape)
    gl = rng.standard_normal(lse.shape) if with_dlse else None
    dq, dk, dv, ds = O.attn_bwd(q, k, v, sk, cu, window, base, 64, 0.707, go, gl)
    eps = 1e-5
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        flat = arr.reshape(-1)
        idx = rng.choice(flat.size, size=n_coords, replace=False)
        # include rotated dims and pass-through dims of Q/K
        for i in idx:
            old = flat[i]
            flat[i] = old + eps
            lp = _loss(O, q, k, v, sk, cu, window, base, go, gl)
            flat[i] = old - eps
            lm = _loss(O, q, k, v, sk, cu, window, base, go, gl)
            flat[i] = old
            fd = (lp - lm) / (2 * eps)
            an = grad.reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), f"d{name}[{i}]: analytic {an:.10g} vs numeric {fd:.10g}"
    if sk is not None:
        h_eps = np.float32(2.0 ** -12)
        for h in range(len(sk)):
            sp, sm = sk.copy(), sk.copy()
            sp[h] += h_eps
            sm[h] -= h_eps
            fd = (_loss(O, q, k, v, sp, cu, window, base, go, gl) - _loss(O, q, k, v, sm, cu, window, base, go, gl)) / (2 * float(h_eps))
            assert abs(fd - ds[h]) <= 1e-6 * max(1.0, abs(fd)), f"dsink[{h}]: analytic {ds[h]:.10g} vs numeric {fd:.10g}"


def pin_bwd_finite_differences_swa_sink(O):
    """Sliding window 5 (masked rows and a window edge), a sink, GQA 4:2, two sequences, dL/dlse != 0."""
    _fd_check(O, _case([30, 17], 4, 2, 21, 5, 1e4, True), 22)


def pin_bwd_finite_differences_global(O):
    """Global causal layer, base 1e7, no sink, GQA 4:1."""
    _fd_check(O, _case([20, 9], 4, 1, 23, -1, 1e7, False), 24, with_dlse=True)


def pin_bwd_shift_invariance(O):
    """No sink and dL/dlse = 0: adding one vector to the pass-through dims of every key of a
    sequence shifts every score of each row by the same amount, so L does not move and those
    dk sum to zero; adding c to every V row adds v_scale c to every output row, so the dv of a
    sequence and KV head sum to v_scale times the summed dO of its query heads."""
    q, k, v, sk, cu, window, base = _case([25, 40], 6, 2, 25, 7, 1e4, False)
    rng = np.random.default_rng(26)
    out, _ = O.attn_fwd_f64(q, k, v, None, cu, window, base, 64, 0.707, threads=1)
    go = rng.standard_normal(out.shape)
    dq, dk, dv, _ = O.attn_bwd(q, k, v, None, cu, window, base, 64, 0.707, go, None)
    group = 6 // 2
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        for g in range(2):
            assert np.allclose(dk[s:e, g, 64:].sum(axis=0), 0.0, atol=1e-9), "pass-dim key shift changes L"
            want = 0.707 * go[s:e, g * group:(g + 1) * group, :].sum(axis=(0, 1))
            assert np.allclose(dv[s:e, g].sum(axis=0), want, atol=1e-9), "V shift rule"


def pin_bwd_one_key_window(O):
    """Window 0: every query sees only its own key.  Without a sink out = v_scale v, so dq = dk = 0
    and dv = v_scale * (sum of dO over the group's query heads).  With a sink the weight is the
    logistic of (s - sigma) and dL/dsigma = -sum over rows of P (1 - P) (dO . v_scale v)."""
    q, k, v, _, cu, _, base = _case([9, 4], 4, 2, 27, 0, 1e4, False)
    rng = np.random.default_rng(28)
    go = rng.standard_normal((13, 4, 128))
    dq, dk, dv, _ = O.attn_bwd(q, k, v, None, cu, 0, base, 64, 0.707, go, None)
    assert np.allclose(dq, 0.0, atol=1e-12) and np.allclose(dk, 0.0, atol=1e-12)
    assert np.allclose(dv, 0.707 * go.reshape(13, 2, 2, 128).sum(axis=2), atol=1e-12)
    sk = np.array([0.5, -1.25, 2.0, 0.0], dtype=np.float32)
    dq, dk, dv, ds = O.attn_bwd(q, k, v, sk, cu, 0, base, 64, 0.707, go, None)
    want = np.zeros(4)
    for t in range(13):
        pos = t if t < 9 else t - 9
        for h in range(4):
            g = h // 2
            qr = oracle.rope(q[t, h], pos, base)
            kr = oracle.rope(k[t, g], pos, base)
            s = float(qr @ kr) / np.sqrt(192.0)
            p = 1.0 / (1.0 + np.exp(float(sk[h]) - s))
            want[h] -= p * (1 - p) * float(go[t, h] @ (0.707 * v[t, g]))
    assert np.allclose(ds, want, rtol=1e-9, atol=1e-12), (ds, want)


def pin_bwd_bf16_inputs_match_f64(O):
    """The BF16-bit entry and the FP64 entry give the same gradients for the same values."""
    q, k, v, sk, cu, window, base = _case([12, 5], 2, 1, 29, 3, 1e4, True)
    rng = np.random.default_rng(30)
    go = rng.standard_normal((17, 2, 128))
    a = O.attn_bwd(q, k, v, sk, cu, window, base, 64, 0.707, go, None)
    bits = lambda x: synth.f32_to_bf16_bits(x.astype(np.float32))
    b = O.attn_bwd(bits(q), bits(k), bits(v), sk, cu, window, base, 64, 0.707, go, None)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


BWD_PINS = [pin_bwd_finite_differences_swa_sink, pin_bwd_finite_differences_global, pin_bwd_shift_invariance,
            pin_bwd_one_key_window, pin_bwd_bf16_inputs_match_f64]
