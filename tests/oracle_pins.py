"""Pins for the FP64 oracle: checks against what the pages and mathematics fix.

Each ``pin_*`` takes an oracle handle ``O`` (with ``attn_fwd`` and ``rope``)
and raises AssertionError when the handle disagrees with a closed form, an
invariant, an independent brute force or a library routine.  The same pins run
against the real oracle (test_oracle_pins.py) and against deliberately broken
copies of it (test_oracle_mutations.py), which shows that each plausible
mistake is caught by at least one pin.
"""
from __future__ import annotations

import cmath
import json
import math
import os

import numpy as np

from global_attention_moe_b200 import synth

FACTS = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))
DQK = FACTS["head_dim_qk"]["value"]
DV = FACTS["head_dim_v"]["value"]
R = FACTS["rope_dims"]["value"]
VS = FACTS["v_scale"]["value"]
W_SWA = FACTS["swa_window"]["value"]
BASE_SWA = FACTS["rope_base_swa"]["value"]
BASE_GLOBAL = FACTS["rope_base_global"]["value"]


def bf16(x) -> np.ndarray:
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def f64(bits) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def rand_inputs(seed, lengths, hq, hkv, sink=True, dqk=DQK, dv=DV):
    T = int(sum(lengths))
    q = synth.normal_bf16(seed, 1, (T, hq, dqk))
    k = synth.normal_bf16(seed, 2, (T, hkv, dqk))
    v = synth.normal_bf16(seed, 3, (T, hkv, dv))
    s = synth.normal_f32(seed, 4, hq) if sink else None
    cu = synth.cu_seqlens_from_lengths(lengths)
    return q, k, v, s, cu


# ----------------------------------------------------------------------------- RoPE
def rope_complex(x, pos, base, rope_dims=R):
    """Textbook complex form: (x_i + i x_{i+R/2}) * exp(i pos base^(-2i/R))."""
    x = [float(t) for t in x]
    y = list(x)
    half = rope_dims // 2
    for i in range(half):
        z = complex(x[i], x[i + half]) * cmath.exp(1j * pos * base ** (-2.0 * i / rope_dims))
        y[i], y[i + half] = z.real, z.imag
    return np.array(y)


def pin_rope(O):
    rng = np.random.default_rng(1)
    x = rng.standard_normal(DQK)
    # position 0 is the identity
    assert np.array_equal(O.rope(x, 0, BASE_SWA), x)
    for base in (BASE_SWA, BASE_GLOBAL):
        for pos in (1, 5, 127, 128, 4095, 131071):
            y = O.rope(x, pos, base)
            # dims past the rotary part are untouched
            assert np.array_equal(y[R:], x[R:])
            # rotation preserves the norm
            assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12 * np.linalg.norm(x)
            # equals the complex-multiplication form
            assert np.max(np.abs(y - rope_complex(x, pos, base))) < 1e-9, (base, pos)
    # relative-position invariance of the rotated dot product
    q, k = rng.standard_normal(DQK), rng.standard_normal(DQK)
    for (m, n, c) in ((3, 1, 7), (200, 17, 1000), (5000, 4990, 123)):
        a = O.rope(q, m, BASE_SWA) @ O.rope(k, n, BASE_SWA)
        b = O.rope(q, m + c, BASE_SWA) @ O.rope(k, n + c, BASE_SWA)
        assert abs(a - b) < 1e-9
    # the first pair rotates by exactly pos radians (theta_0 = 1) and pair i by pos*base^(-2i/R)
    e = np.zeros(DQK)
    for i in (0, 1, 17, R // 2 - 1):
        e[:] = 0.0
        e[i] = 1.0
        y = O.rope(e, 3, BASE_SWA)
        ang = math.atan2(y[i + R // 2], y[i])
        want = math.remainder(3 * BASE_SWA ** (-2.0 * i / R), 2 * math.pi)
        assert abs(ang - want) < 1e-12, (i, ang, want)


# ------------------------------------------------------------------ window / key set
def pin_key_counts(O):
    """Q = 0 makes every score 0, so with no sink lse = ln(#keys) and out is the
    plain mean of the attended v rows.  Pins the exact key set A(p)."""
    L = 300
    hq = hkv = 1
    q = np.zeros((L, hq, DQK), dtype=np.uint16)  # bf16 +0.0
    k = synth.normal_bf16(9, 2, (L, hkv, DQK))
    j = np.arange(L)
    vf = np.zeros((L, hkv, DV), dtype=np.float32)
    vf[:, 0, 0] = j // 16
    vf[:, 0, 1] = j % 16
    vf[:, 0, 2] = 1.0
    v = bf16(vf)
    cu = np.array([0, L], dtype=np.int32)
    cases = [(FACTS["swa_window"]["value"], FACTS["swa_keys_per_query"]["value"]),
             (FACTS["hf_variant_keys_per_query"]["window"], FACTS["hf_variant_keys_per_query"]["value"]),
             (0, 1), (5, 6), (1000, None), (-1, None)]
    for W, full_keys in cases:
        out, lse = O.attn_fwd(q, k, v, None, cu, W, BASE_SWA, v_scale=1.0)
        p = np.arange(L)
        lo = np.zeros(L, dtype=np.int64) if W < 0 else np.maximum(0, p - W)
        count = p - lo + 1
        if full_keys is not None:
            assert count[-1] == full_keys
        assert np.allclose(lse[0], np.log(count), rtol=0, atol=1e-12), W
        mean_j = 16 * out[:, 0, 0] + out[:, 0, 1]
        assert np.allclose(mean_j, (lo + p) / 2.0, rtol=0, atol=1e-9), W
        assert np.allclose(out[:, 0, 2], 1.0, atol=1e-12)


def pin_window_large_equals_global(O):
    q, k, v, _, cu = rand_inputs(3, [200, 77], 2, 1, sink=False)
    o1, l1 = O.attn_fwd(q, k, v, None, cu, 10 ** 6, BASE_GLOBAL)
    o2, l2 = O.attn_fwd(q, k, v, None, cu, -1, BASE_GLOBAL)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    o3, l3 = O.attn_fwd(q, k, v, None, cu, 199, BASE_GLOBAL)
    assert np.array_equal(o1, o3) and np.array_equal(l1, l3)


# ----------------------------------------------------------------------------- sink
def pin_sink_limits(O):
    q, k, v, s, cu = rand_inputs(4, [150], 4, 2)
    o0, l0 = O.attn_fwd(q, k, v, None, cu, W_SWA, BASE_SWA)
    neg = np.full(4, -np.inf, dtype=np.float32)
    o1, l1 = O.attn_fwd(q, k, v, neg, cu, W_SWA, BASE_SWA)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    big = np.full(4, 1e4, dtype=np.float32)
    o2, l2 = O.attn_fwd(q, k, v, big, cu, W_SWA, BASE_SWA)
    assert np.all(o2 == 0.0) and np.all(l2 == 1e4)
    # sink identities: lse_s = logaddexp(lse, sigma), out_s = out * exp(lse - lse_s)
    o3, l3 = O.attn_fwd(q, k, v, s, cu, W_SWA, BASE_SWA)
    want_l = np.logaddexp(l0, s.astype(np.float64)[:, None])
    assert np.max(np.abs(l3 - want_l)) < 1e-12
    want_o = o0 * np.exp(l0 - want_l).T[:, :, None]
    assert np.max(np.abs(o3 - want_o)) < 1e-12


def pin_weights_sum(O):
    """With every v = 1 and v_scale = 1 each output is the total key weight,
    1 - sink weight = 1 - exp(sigma - lse)."""
    q, k, _, s, cu = rand_inputs(5, [64, 190], 4, 1)
    v = bf16(np.ones((254, 1, DV), dtype=np.float32))
    out, lse = O.attn_fwd(q, k, v, s, cu, W_SWA, BASE_SWA, v_scale=1.0)
    want = 1.0 - np.exp(s.astype(np.float64)[:, None] - lse)
    assert np.max(np.abs(out - want.T[:, :, None])) < 1e-12
    assert np.all(lse >= s.astype(np.float64)[:, None])


def pin_first_row_closed_form(O):
    """At p = 0 RoPE is the identity and the only key is the query's own:
    out = v_scale v0 e^{s00} / (e^{s00} + e^{sigma}), lse = ln(e^{s00} + e^{sigma})."""
    q, k, v, s, cu = rand_inputs(6, [40, 33], 4, 2)
    out, lse = O.attn_fwd(q, k, v, s, cu, W_SWA, BASE_SWA, v_scale=VS)
    outn, lsen = O.attn_fwd(q, k, v, None, cu, W_SWA, BASE_SWA, v_scale=VS)
    for t0 in cu[:-1]:
        for h in range(4):
            g = h // 2
            s00 = float(f64(q[t0, h]) @ f64(k[t0, g])) / math.sqrt(DQK)
            sig = float(s[h])
            w = math.exp(s00) / (math.exp(s00) + math.exp(sig))
            assert np.max(np.abs(out[t0, h] - VS * f64(v[t0, g]) * w)) < 1e-12
            assert abs(lse[h, t0] - math.log(math.exp(s00) + math.exp(sig))) < 1e-12
            assert np.max(np.abs(outn[t0, h] - VS * f64(v[t0, g]))) < 1e-12
            assert abs(lsen[h, t0] - s00) < 1e-12


def pin_v_scale_linear(O):
    q, k, v, s, cu = rand_inputs(7, [200], 2, 1)
    o1, l1 = O.attn_fwd(q, k, v, s, cu, W_SWA, BASE_SWA, v_scale=1.0)
    o2, l2 = O.attn_fwd(q, k, v, s, cu, W_SWA, BASE_SWA, v_scale=VS)
    assert np.array_equal(l1, l2)
    assert np.max(np.abs(o2 - VS * o1)) < 1e-13


# ------------------------------------------------------------------- brute force
def brute_row(q, k, v, sink, cu, t, h, window, base, v_scale, hq, hkv):
    """Independent per-query softmax: explicit logits list, complex-form RoPE,
    Python floats with math.fsum."""
    b = int(np.searchsorted(cu, t, side="right") - 1)
    sb = int(cu[b])
    p = t - sb
    g = h * hkv // hq
    qr = rope_complex(f64(q[t, h]), p, base)
    keys = [j for j in range(0, p + 1) if window < 0 or p - j <= window]
    logits = []
    for j in keys:
        kr = rope_complex(f64(k[sb + j, g]), j, base)
        logits.append(math.fsum(float(a) * float(c) for a, c in zip(qr, kr)) / math.sqrt(DQK))
    all_logits = logits + ([float(sink[h])] if sink is not None else [])
    m = max(all_logits)
    z = math.fsum(math.exp(x - m) for x in all_logits)
    lse = m + math.log(z)
    vv = f64(v)
    out = [math.fsum(math.exp(logits[i] - lse) * v_scale * float(vv[sb + j, g, d]) for i, j in enumerate(keys))
           for d in range(vv.shape[2])]
    return np.array(out), lse


def pin_brute_force(O):
    cases = [([37], 4, 1, W_SWA, BASE_SWA, True),
             ([140, 9], 4, 2, W_SWA, BASE_SWA, True),
             ([70, 1, 60], 6, 3, 5, BASE_SWA, False),
             ([90], 4, 4, -1, BASE_GLOBAL, False),
             ([30, 44], 8, 2, -1, BASE_GLOBAL, True)]
    for ci, (lengths, hq, hkv, W, base, has_sink) in enumerate(cases):
        q, k, v, s, cu = rand_inputs(20 + ci, lengths, hq, hkv, sink=has_sink)
        out, lse = O.attn_fwd(q, k, v, s, cu, W, base, v_scale=VS)
        T = int(sum(lengths))
        rows = sorted({0, T - 1, T // 2, int(cu[-2]), min(T - 1, 129), min(T - 1, 131)})
        for t in rows:
            for h in range(hq):
                bo, bl = brute_row(q, k, v, s, cu, t, h, W, base, VS, hq, hkv)
                assert abs(lse[h, t] - bl) < 1e-12, (ci, t, h)
                assert np.max(np.abs(out[t, h] - bo)) < 1e-12, (ci, t, h)


def pin_library_sdpa(O):
    """Special case that reduces to a library routine: torch's float64
    scaled_dot_product_attention with an explicit boolean mask on RoPE'd
    inputs (rotated here with torch complex ops), plus torch.logsumexp."""
    import torch
    lengths, hq, hkv = [180, 75], 4, 2
    q, k, v, s, cu = rand_inputs(31, lengths, hq, hkv)
    for W, base, use_sink in ((W_SWA, BASE_SWA, True), (-1, BASE_GLOBAL, False), (17, BASE_SWA, False)):
        out, lse = O.attn_fwd(q, k, v, s if use_sink else None, cu, W, base, v_scale=VS)
        for b in range(len(lengths)):
            sb, L = int(cu[b]), lengths[b]
            pos = torch.arange(L, dtype=torch.float64)
            inv = base ** (-torch.arange(R // 2, dtype=torch.float64) * 2.0 / R)
            rot = torch.polar(torch.ones(L, R // 2, dtype=torch.float64), pos[:, None] * inv[None, :])

            def rope_t(x):  # x [L, H, D]
                z = torch.complex(x[..., :R // 2], x[..., R // 2:R]) * rot[:, None, :]
                return torch.cat([z.real, z.imag, x[..., R:]], dim=-1)

            qt = rope_t(torch.from_numpy(f64(q[sb:sb + L]))).permute(1, 0, 2)
            kt = rope_t(torch.from_numpy(f64(k[sb:sb + L]))).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)
            vt = torch.from_numpy(VS * f64(v[sb:sb + L])).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)
            i = torch.arange(L)[:, None]
            j = torch.arange(L)[None, :]
            mask = (j <= i) if W < 0 else ((j <= i) & (i - j <= W))
            ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
            scores = (qt @ kt.transpose(1, 2)) / math.sqrt(DQK)
            ref_lse = torch.logsumexp(scores.masked_fill(~mask, float("-inf")), dim=-1)
            if use_sink:
                sig = torch.from_numpy(s.astype(np.float64))[:, None]
                new_lse = torch.logaddexp(ref_lse, sig.expand_as(ref_lse))
                ref = ref * torch.exp(ref_lse - new_lse)[..., None]
                ref_lse = new_lse
            assert np.max(np.abs(out[sb:sb + L].transpose(1, 0, 2) - ref.numpy())) < 1e-11, (W, b)
            assert np.max(np.abs(lse[:, sb:sb + L] - ref_lse.numpy())) < 1e-11, (W, b)


# --------------------------------------------------------------- structure
def pin_packing_independent(O):
    lengths = [130, 1, 257, 0, 64]
    q, k, v, s, cu = rand_inputs(8, lengths, 4, 2)
    out, lse = O.attn_fwd(q, k, v, s, cu, W_SWA, BASE_SWA)
    for b, L in enumerate(lengths):
        if L == 0:
            continue
        sb = int(cu[b])
        sl = slice(sb, sb + L)
        o1, l1 = O.attn_fwd(q[sl], k[sl], v[sl], s, np.array([0, L], dtype=np.int32), W_SWA, BASE_SWA)
        assert np.array_equal(o1, out[sl]) and np.array_equal(l1, lse[:, sl])


def pin_gqa_equals_mha(O):
    hq, hkv = 8, 2
    q, k, v, s, cu = rand_inputs(10, [150], hq, hkv)
    o1, l1 = O.attn_fwd(q, k, v, s, cu, W_SWA, BASE_SWA)
    kr = np.repeat(k, hq // hkv, axis=1)
    vr = np.repeat(v, hq // hkv, axis=1)
    o2, l2 = O.attn_fwd(q, kr, vr, s, cu, W_SWA, BASE_SWA)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def pin_rows_subset(O):
    q, k, v, s, cu = rand_inputs(11, [300, 20], 4, 1)
    o, l = O.attn_fwd(q, k, v, s, cu, W_SWA, BASE_SWA)
    rows = np.array([319, 0, 128, 129, 300, 5], dtype=np.int64)
    o2, l2 = O.attn_fwd(q, k, v, s, cu, W_SWA, BASE_SWA, rows=rows)
    assert np.array_equal(o2, o[rows]) and np.array_equal(l2, l[:, rows])


ALL_PINS = [pin_rope, pin_key_counts, pin_window_large_equals_global, pin_sink_limits, pin_weights_sum,
            pin_first_row_closed_form, pin_v_scale_linear, pin_brute_force, pin_library_sdpa,
            pin_packing_independent, pin_gqa_equals_mha, pin_rows_subset]
