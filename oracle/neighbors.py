"""Plain CPU definitions of the steps on either side of the MiMo-V2 attention
kernel -- TEST INFRASTRUCTURE (same rule as the rest of ``oracle``: only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU legs may use it).

numpy only, FP64 unless a page fixes the precision.  Sources (page title and
section):

* FP8 block-quantized weights and the fused, kv-head-interleaved qkv_proj:
  miles docs "MiMo-V2.6-Flash", section 1 Model Introduction (compressed
  checkpoint) and section 3.1 (the converter dequantizes each kv-head shard of
  the fused qkv_proj with its own FP8 block scales and splits it into q/k/v in
  head order); Megatron-Bridge API doc "mimo_v2_flash_bridge",
  ``_dequant_fp8_blockwise`` (out = fp8 value times scale_inv) and
  ``MiMoV2FlashQKVMapping`` (192-dim Q/K, 128-dim V).
* Output projection (linear_proj): miles PR #3648 "add MiMo-V2.6-Flash-RL
  support", commit message on MiMoV2SelfAttention (the layer's linear_qkv and
  linear_proj are built for the 128-dim V heads: linear_proj takes the
  Hq x 128 attention output of a token).
* MoE router: miles docs section 1 (256 routed experts, top-8 sigmoid routing
  with a fixed score-correction bias); miles PR #3648 review (no group-limited
  routing in this checkpoint); SGLang cookbook "MiMo-V2.6", section 2
  Configuration tips, Parallelism and precision (router logits computed in
  FP32).

Readings where the pages are silent:

* FP8 element format: OCP E4M3 ("fn": no infinities, S.1111.111 is NaN).
  The block size of the scales is not given: 128 x 128 blocks here, a
  parameter.  The block size is therefore a reading, not a page fact
  (``dequant_fp8_blockwise``: parity unpinned as to the block size).
* kv-head-interleaved layout: along the fused output dimension, KV group g
  holds its Hq/Hkv query heads (192 each), then its K head (192), then its V
  head (128), groups in order.
* linear_proj: y = x W^T with W stored as a Linear weight [out, in], no bias
  (the pages name no bias anywhere in the layer); the output width (the
  model's hidden size) is not on the pages, a parameter here.
* Router: scores are sigmoid(logit); the correction bias enters the choice of
  experts only (top-8 of score + bias); the weights are the chosen experts'
  scores, normalised to sum to one (``normalize``) -- both parts of this
  reading are unpinned by the pages.  Ties in score + bias go to the lower
  expert index.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------- FP8 E4M3


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Decode FP8 E4M3 bytes by the format's definition: sign bit, 4 exponent
    bits with bias 7, 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6);
    S.1111.111 is NaN; there are no infinities."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = sign * (m / 8.0) * 2.0 ** -6
    out = np.where(e == 0, sub, normal)
    return np.where((e == 0xF) & (m == 0x7), np.nan, out)


def dequant_fp8_blockwise(codes: np.ndarray, scale_inv: np.ndarray, block=(128, 128)) -> np.ndarray:
    """out[i, j] = e4m3(codes[i, j]) * scale_inv[i // block[0], j // block[1]] (FP64).
    codes: uint8 [M, N]; scale_inv: [ceil(M / b0), ceil(N / b1)]."""
    codes = np.asarray(codes, dtype=np.uint8)
    M, N = codes.shape
    b0, b1 = block
    s = np.asarray(scale_inv, dtype=np.float64)
    assert s.shape == (-(-M // b0), -(-N // b1)), "one scale per block"
    rows = np.arange(M) // b0
    cols = np.arange(N) // b1
    return e4m3_to_f64(codes) * s[rows[:, None], cols[None, :]]


# ---------------------------------------------------------------- fused QKV


def qkv_layout(hq: int, hkv: int, dqk: int = 192, dv: int = 128):
    """Offsets of the kv-head-interleaved fused output: for KV group g, its
    Hq/Hkv query heads, then its K head, then its V head."""
    group = hq // hkv
    per_group = group * dqk + dqk + dv
    return group, per_group


def split_qkv(fused: np.ndarray, hq: int, hkv: int, dqk: int = 192, dv: int = 128):
    """fused [T, Hkv * (group*dqk + dqk + dv)] -> q [T, Hq, dqk], k [T, Hkv, dqk], v [T, Hkv, dv].
    A pure permutation: values are copied unchanged (any dtype)."""
    assert hq % hkv == 0
    group, per_group = qkv_layout(hq, hkv, dqk, dv)
    T = fused.shape[0]
    assert fused.shape[1] == hkv * per_group
    x = fused.reshape(T, hkv, per_group)
    q = x[:, :, :group * dqk].reshape(T, hkv, group, dqk).reshape(T, hq, dqk)
    k = x[:, :, group * dqk:group * dqk + dqk]
    v = x[:, :, group * dqk + dqk:]
    return np.ascontiguousarray(q), np.ascontiguousarray(k), np.ascontiguousarray(v)


# ---------------------------------------------------------------- MoE router


def sigmoid_f64(x):
    x = np.asarray(x, dtype=np.float64)
    return np.where(x >= 0, 1.0 / (1.0 + np.exp(-np.abs(x))), np.exp(-np.abs(x)) / (1.0 + np.exp(-np.abs(x))))


def route(logits: np.ndarray, bias: np.ndarray, top_k: int = 8, normalize: bool = True):
    """Top-k sigmoid routing with a score-correction bias.

    logits [T, E] (FP32 on the pages), bias [E].  The choice is taken in FP32,
    the precision the pages give the router output: key = fp32(sigmoid) + fp32(bias)
    rounded to FP32.  Returns ids [T, k] int32 in descending key order (ties:
    lower expert first), weights [T, k] FP64 (the chosen experts' sigmoid
    scores, normalised to sum to one when ``normalize``), and the FP32 keys [T, E].
    """
    logits = np.asarray(logits, dtype=np.float32)
    bias = np.asarray(bias, dtype=np.float32)
    T, E = logits.shape
    assert bias.shape == (E,) and 1 <= top_k <= E
    s64 = sigmoid_f64(logits)
    key = (s64.astype(np.float32) + bias[None, :]).astype(np.float32)
    ids = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k), dtype=np.float64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(key[t, e]), e))[:top_k]
        ids[t] = order
        sel = s64[t, order]
        w[t] = sel / sel.sum() if normalize else sel
    return ids, w, key


# ---------------------------------------------------------------- output projection


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) to their exact FP64 values (the top half of an FP32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def linear_proj(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """The attention's output projection y = x W^T, exactly in FP64.

    x: BF16 bits [T, K], the attention output of each token with its Hq heads of 128 dims side by
    side (K = Hq x 128); w: BF16 bits [N, K], a Linear weight (out_features x in_features).
    Returns FP64 [T, N]; no bias."""
    xf = bf16_bits_to_f64(x)
    wf = bf16_bits_to_f64(w)
    assert xf.ndim == 2 and wf.ndim == 2 and xf.shape[1] == wf.shape[1]
    return xf @ wf.T
