"""Pins for the oracle of the steps beside the attention kernel (FP8 blockwise
dequant, fused-QKV split, output projection, MoE router), against what the pages and mathematics
fix: a library decoder of the FP8 format, closed forms, an independent
construction of the fused layout, brute force over expert subsets, invariants.

Each ``pin_*`` takes a handle ``N`` with ``e4m3_to_f64``,
``dequant_fp8_blockwise``, ``split_qkv``, ``linear_proj`` and ``route``, and raises
AssertionError on a disagreement.  The same pins run against the real module
and against deliberately broken copies of it.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch

FACTS = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))
E = FACTS["moe_routed_experts"]["value"]
K = FACTS["moe_top_k"]["value"]
DQK = FACTS["head_dim_qk"]["value"]
DV = FACTS["head_dim_v"]["value"]


# ---------------------------------------------------------------- FP8


def pin_e4m3_all_codes_match_torch(N):
    """Every one of the 256 codes decodes as torch's float8_e4m3fn does (a library decoder)."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = N.e4m3_to_f64(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "NaN codes"
    assert np.array_equal(got[~nan], ref[~nan]), "decoded values"


def pin_e4m3_closed_forms(N):
    """Values the format's definition fixes: 1, -1, the largest finite (448), the smallest
    normal (2^-6), the smallest subnormal (2^-9), zero and negative zero."""
    v = N.e4m3_to_f64(np.array([0x38, 0xB8, 0x7E, 0x08, 0x01, 0x00, 0x80], dtype=np.uint8))
    assert list(v[:5]) == [1.0, -1.0, 448.0, 2.0 ** -6, 2.0 ** -9]
    assert v[5] == 0.0 and v[6] == 0.0 and math.copysign(1.0, v[6]) == -1.0


def pin_dequant_blocks_by_kron(N):
    """Blockwise scaling equals the scale grid expanded by a Kronecker product with a block of
    ones (a library routine), cropped at ragged edges; non-square blocks catch a transposed
    block index."""
    rng = np.random.default_rng(5)
    for (M, Nn), blk in (((300, 200), (128, 128)), ((70, 130), (32, 64)), ((5, 7), (4, 2))):
        codes = rng.integers(0, 256, size=(M, Nn)).astype(np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x00  # no NaN codes here
        gs = (-(-M // blk[0]), -(-Nn // blk[1]))
        s = rng.uniform(0.5, 4.0, size=gs)
        want = N.e4m3_to_f64(codes) * np.kron(s, np.ones(blk))[:M, :Nn]
        got = N.dequant_fp8_blockwise(codes, s, block=blk)
        assert got.shape == (M, Nn)
        assert np.array_equal(got, want), f"blockwise scaling {M}x{Nn} {blk}"


def pin_dequant_identity_scale(N):
    """With scale_inv = 1 the dequant is the plain decode; with code 1.0 it is the scale grid."""
    codes = np.full((256, 384), 0x38, dtype=np.uint8)
    s = np.arange(2 * 3, dtype=np.float64).reshape(2, 3) + 1.0
    got = N.dequant_fp8_blockwise(codes, s)
    for i, j in itertools.product(range(2), range(3)):
        assert np.all(got[128 * i:128 * (i + 1), 128 * j:128 * (j + 1)] == s[i, j])
    one = N.dequant_fp8_blockwise(codes, np.ones((2, 3)))
    assert np.all(one == 1.0)


# ---------------------------------------------------------------- fused QKV


def _fused_from_parts(q, k, v):
    """The page's layout built element by element: KV group g holds its query heads, then its
    K head, then its V head."""
    T, hq, dqk = q.shape
    hkv, dv = k.shape[1], v.shape[2]
    group = hq // hkv
    rows = []
    for t in range(T):
        row = []
        for g in range(hkv):
            for j in range(group):
                row.extend(q[t, g * group + j].tolist())
            row.extend(k[t, g].tolist())
            row.extend(v[t, g].tolist())
        rows.append(row)
    return np.array(rows, dtype=q.dtype)


def pin_split_inverts_the_fused_layout(N):
    """Splitting a fused row built from known q/k/v (distinct values everywhere) returns them
    exactly, for the layer shapes and for degenerate groupings."""
    rng = np.random.default_rng(6)
    for hq, hkv, dqk, dv in ((64, 8, DQK, DV), (64, 4, DQK, DV), (4, 4, 6, 4), (6, 2, 5, 3), (3, 1, 4, 2)):
        T = 3
        vals = rng.permutation(T * (hq * dqk + hkv * dqk + hkv * dv)).astype(np.int64)
        q = vals[:T * hq * dqk].reshape(T, hq, dqk)
        k = vals[T * hq * dqk:T * (hq + hkv) * dqk].reshape(T, hkv, dqk)
        v = vals[T * (hq + hkv) * dqk:].reshape(T, hkv, dv)
        fq, fk, fv = N.split_qkv(_fused_from_parts(q, k, v), hq, hkv, dqk, dv)
        assert np.array_equal(fq, q) and np.array_equal(fk, k) and np.array_equal(fv, v), (hq, hkv)


# ---------------------------------------------------------------- router


def pin_route_zero_bias_is_logit_topk(N):
    """Without a bias the choice is the k largest logits (sigmoid is increasing), in order: a
    library sort of the logits."""
    rng = np.random.default_rng(7)
    logits = rng.standard_normal((32, E)).astype(np.float32) * 3
    ids, w, _ = N.route(logits, np.zeros(E, np.float32), K)
    want = np.argsort(-logits, axis=1, kind="stable")[:, :K]
    assert np.array_equal(ids, want)


def pin_route_brute_force_subsets(N):
    """On a small expert count, the chosen set maximises the summed score + bias over all
    subsets of size k (brute force), with a bias large enough to change the choice."""
    rng = np.random.default_rng(8)
    e, k = 9, 3
    for _ in range(20):
        logits = rng.standard_normal((1, e)).astype(np.float32)
        bias = rng.uniform(-0.5, 0.5, e).astype(np.float32)
        score = 1.0 / (1.0 + np.exp(-logits[0].astype(np.float64)))
        key = score + bias
        best = max(itertools.combinations(range(e), k), key=lambda c: sum(key[list(c)]))
        ids, _, _ = N.route(logits, bias, k)
        assert sorted(ids[0].tolist()) == sorted(best)


def pin_route_weights_closed_form(N):
    """sigmoid(0) = 1/2 and sigmoid(ln 3) = 3/4: the chosen weights are 0.6 and 0.4 after
    normalisation; a bias that promotes expert 2 leaves the bias out of its weight."""
    ln3 = math.log(3.0)
    ids, w, _ = N.route(np.array([[0.0, ln3, -5.0, -5.0]], np.float32), np.zeros(4, np.float32), 2)
    assert ids[0].tolist() == [1, 0]
    assert np.allclose(w[0], [0.6, 0.4], rtol=0, atol=1e-7)
    ids, w, _ = N.route(np.array([[0.0, ln3, 0.0, -5.0]], np.float32), np.array([0, 0, 0.3, 0], np.float32), 2)
    assert ids[0].tolist() == [2, 1]  # keys 0.8 and 0.75
    assert np.allclose(w[0], [0.4, 0.6], rtol=0, atol=1e-7)


def pin_route_invariants(N):
    """At the layer's shape: distinct experts, keys non-increasing along the choice, every
    unchosen key at most the smallest chosen key, weights positive and summing to one; equal
    keys go to the lower expert index."""
    rng = np.random.default_rng(9)
    logits = rng.standard_normal((64, E)).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.1).astype(np.float32)
    ids, w, key = N.route(logits, bias, K)
    for t in range(64):
        assert len(set(ids[t].tolist())) == K
        kk = key[t, ids[t]]
        assert np.all(np.diff(kk.astype(np.float64)) <= 0)
        rest = np.setdiff1d(np.arange(E), ids[t])
        assert key[t, rest].max() <= kk.min()
        assert np.all(w[t] > 0) and abs(w[t].sum() - 1.0) < 1e-12
    ids, _, _ = N.route(np.zeros((1, E), np.float32), np.zeros(E, np.float32), K)
    assert ids[0].tolist() == list(range(K))


# ---------------------------------------------------------------- output projection


def _bf16_exact(v):
    """BF16 bits of FP32 values that are exactly representable (at most 8 significant bits)."""
    f = np.asarray(v, dtype=np.float32)
    bits = (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    assert np.array_equal((bits.astype(np.uint32) << np.uint32(16)).view(np.float32), f)
    return bits


def pin_linear_proj_brute_force(N):
    """Against a pure-Python sum over the input features (math.fsum, exactly rounded), with the BF16
    values decoded bit by bit, on a tiny ragged shape."""
    rng = np.random.default_rng(21)
    T, Kf, Nf = 3, 24, 5
    # full 8-bit BF16 significands over a spread of exponents: the sums need far more than 24 bits
    x = (rng.standard_normal((T, Kf)).astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    w = (rng.standard_normal((Nf, Kf)).astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)

    def dec(b):
        sign = -1.0 if b >> 15 else 1.0
        e, m = (b >> 7) & 0xFF, b & 0x7F
        return sign * (m / 128.0) * 2.0 ** -126 if e == 0 else sign * (1 + m / 128.0) * 2.0 ** (e - 127)

    y = N.linear_proj(x, w)
    assert y.shape == (T, Nf)
    for t in range(T):
        for n in range(Nf):
            want = math.fsum(dec(int(x[t, k])) * dec(int(w[n, k])) for k in range(Kf))
            assert abs(y[t, n] - want) <= 1e-12 * max(1.0, abs(want)), (t, n)


def pin_linear_proj_selector_weights(N):
    """A weight with a single 1 per output row picks that input feature: output n equals input
    feature perm[n] exactly (catches a transposed or shifted operand)."""
    rng = np.random.default_rng(22)
    T, Kf, Nf = 4, DV * 2, 7
    x = _bf16_exact(np.round(rng.standard_normal((T, Kf)) * 8) / 8)
    perm = rng.permutation(Kf)[:Nf]
    wf = np.zeros((Nf, Kf), np.float32)
    wf[np.arange(Nf), perm] = 1.0
    y = N.linear_proj(x, _bf16_exact(wf))
    xv = (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    assert np.array_equal(y, xv[:, perm])


ALL_PINS = [pin_e4m3_all_codes_match_torch, pin_e4m3_closed_forms, pin_dequant_blocks_by_kron,
            pin_dequant_identity_scale, pin_split_inverts_the_fused_layout, pin_route_zero_bias_is_logit_topk,
            pin_route_brute_force_subsets, pin_route_weights_closed_form, pin_route_invariants,
            pin_linear_proj_brute_force, pin_linear_proj_selector_weights]
