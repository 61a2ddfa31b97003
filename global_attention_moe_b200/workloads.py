"""Named synthetic workloads shaped like the MiMo-V2 attention layers.

Every workload is drawn by :mod:`global_attention_moe_b200.synth` with seed 0
unless a caller passes another seed.  Q/K/V are i.i.d. N(0,1) rounded to BF16;
the sink (sliding-window layers only) is N(0,1) per query head in FP32.

Layer facts (miles docs "MiMo-V2.6-Flash", section 1 Model Introduction and
section 5.4 Notable quirks; miles PR #3648 "add MiMo-V2.6-Flash-RL support",
Design Notes): sliding-window layers attend the query plus 128 previous keys
with a learnable sink, 8 KV heads and RoPE base 1e4; global layers are causal
with 4 KV heads, RoPE base 1e7 and no sink; Q/K are 192-dim, V is 128-dim and
scaled by 0.707; RoPE covers 64 of the 192 Q/K dims.  The query-head count
is not stated there; 64 query heads (8 per KV head on the sliding layer) is a chosen value.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import synth

LAYER_SWA = 0
LAYER_GLOBAL = 1
HEAD_DIM_QK = 192
HEAD_DIM_V = 128
ROPE_DIMS = 64
V_SCALE = 0.707
SWA_WINDOW = 128
ROPE_BASE_SWA = 1e4
ROPE_BASE_GLOBAL = 1e7


@dataclass
class Workload:
    name: str
    layer_kind: int
    lengths: list
    num_q_heads: int
    num_kv_heads: int
    window: int  # -1 for the global (causal) layer
    rope_base: float
    has_sink: bool
    seed: int = 0
    head_dim_qk: int = HEAD_DIM_QK
    head_dim_v: int = HEAD_DIM_V
    rope_dims: int = ROPE_DIMS
    v_scale: float = V_SCALE
    meta: dict = field(default_factory=dict)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))

    @property
    def num_seqs(self) -> int:
        return len(self.lengths)

    @property
    def max_seqlen(self) -> int:
        return int(max(self.lengths)) if self.lengths else 0

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "layer": "swa_sink" if self.layer_kind == LAYER_SWA else "global_causal",
            "num_seqs": self.num_seqs,
            "total_tokens": self.total_tokens,
            "max_seqlen": self.max_seqlen,
            "q_heads": self.num_q_heads,
            "kv_heads": self.num_kv_heads,
            "head_dim_qk": self.head_dim_qk,
            "head_dim_v": self.head_dim_v,
            "window": self.window,
            "rope_base": self.rope_base,
            "rope_dims": self.rope_dims,
            "v_scale": self.v_scale,
            "sink": self.has_sink,
            "seed": self.seed,
        }


def attended_pairs(lengths, window: int, num_q_heads: int) -> int:
    """(query head, query, key) triples attended: sum over queries of min(p+1, W+1)."""
    total = 0
    for L in lengths:
        L = int(L)
        if window < 0:
            total += L * (L + 1) // 2
        else:
            w1 = window + 1
            if L <= w1:
                total += L * (L + 1) // 2
            else:
                total += w1 * (w1 + 1) // 2 + (L - w1) * w1
    return total * num_q_heads


def tiny_swa(seed: int = 0) -> Workload:
    return Workload("tiny_swa_sink_T512_h4_kv1", LAYER_SWA, [512], 4, 1, SWA_WINDOW, ROPE_BASE_SWA, True, seed)


def swa_4096(seed: int = 0) -> Workload:
    return Workload("swa_sink_T4096_h64_kv8", LAYER_SWA, [4096], 64, 8, SWA_WINDOW, ROPE_BASE_SWA, True, seed)


def swa_varlen(seed: int = 0) -> Workload:
    lengths = synth.seq_lengths(seed, 16, 256, 2048).tolist()
    return Workload("swa_sink_varlen_B16_U256_2048_h64_kv8", LAYER_SWA, lengths, 64, 8, SWA_WINDOW,
                    ROPE_BASE_SWA, True, seed)


def global_2x8192(seed: int = 0) -> Workload:
    return Workload("global_causal_B2_L8192_h64_kv4", LAYER_GLOBAL, [8192, 8192], 64, 4, -1,
                    ROPE_BASE_GLOBAL, False, seed)


def swa_131072(seed: int = 0) -> Workload:
    return Workload("swa_sink_T131072_h64_kv8", LAYER_SWA, [131072], 64, 8, SWA_WINDOW, ROPE_BASE_SWA, True, seed)


WORKLOADS = {
    "tiny": tiny_swa,
    "swa4096": swa_4096,
    "swa_varlen": swa_varlen,
    "global": global_2x8192,
    "swa_long": swa_131072,
}


@dataclass
class Inputs:
    q: np.ndarray          # uint16 BF16 bits [T, Hq, 192]
    k: np.ndarray          # uint16 BF16 bits [T, Hkv, 192]
    v: np.ndarray          # uint16 BF16 bits [T, Hkv, 128]
    sink: np.ndarray | None  # float32 [Hq] or None
    cu_seqlens: np.ndarray  # int32 [B+1]


def make_inputs(w: Workload, threads: int | None = None) -> Inputs:
    """Draw the workload's tensors in the order q, k, v, sink (separate streams)."""
    T = w.total_tokens
    q = synth.normal_bf16(w.seed, synth.STREAM_Q, (T, w.num_q_heads, w.head_dim_qk), threads)
    k = synth.normal_bf16(w.seed, synth.STREAM_K, (T, w.num_kv_heads, w.head_dim_qk), threads)
    v = synth.normal_bf16(w.seed, synth.STREAM_V, (T, w.num_kv_heads, w.head_dim_v), threads)
    sink = synth.normal_f32(w.seed, synth.STREAM_SINK, w.num_q_heads) if w.has_sink else None
    cu = synth.cu_seqlens_from_lengths(w.lengths)
    return Inputs(q, k, v, sink, cu)


def custom(name, layer_kind, lengths, hq, hkv, window, rope_base, has_sink, seed=0, v_scale=V_SCALE) -> Workload:
    return Workload(name, layer_kind, list(lengths), hq, hkv, window, rope_base, has_sink, seed, v_scale=v_scale)


# ---------------------------------------------------------------- KV-cache attention
@dataclass
class DecodeInputs:
    """One batch of new tokens against a page-size-1 KV cache (host arrays).

    Sequence b has kv_lens[b] cached tokens (the last q_lens[b] of them new), whose
    cache rows are kv_indices[kv_indptr[b]:kv_indptr[b+1]] in position order; q holds
    the new tokens' queries, THD-packed by cu_q."""
    q: np.ndarray          # uint16 BF16 bits [Tq, Hq, 192]
    k_cache: np.ndarray    # uint16 [rows, Hkv, 192]
    v_cache: np.ndarray    # uint16 [rows, Hkv, 128]
    kv_indices: np.ndarray  # int32 [total_kv]
    kv_indptr: np.ndarray   # int32 [B+1]
    cu_q: np.ndarray        # int32 [B+1]
    sink: np.ndarray | None
    q_lens: list
    kv_lens: list


def make_decode_inputs(kv_lens, q_lens, hq, hkv, has_sink, seed, spare_rows=64, threads=None) -> DecodeInputs:
    """Seeded decode problem: cache rows are a random permutation (page size 1), with spare rows
    that no sequence uses."""
    kv_lens = [int(x) for x in kv_lens]
    q_lens = [int(x) for x in q_lens]
    total_kv = sum(kv_lens)
    rows = total_kv + spare_rows
    q = synth.normal_bf16(seed, synth.STREAM_Q, (sum(q_lens), hq, 192), threads)
    k = synth.normal_bf16(seed, synth.STREAM_K, (rows, hkv, 192), threads)
    v = synth.normal_bf16(seed, synth.STREAM_V, (rows, hkv, 128), threads)
    perm = np.argsort(synth.uniforms(seed, synth.STREAM_PAGES, rows), kind="stable").astype(np.int32)
    kv_indices = perm[:total_kv].copy()
    kv_indptr = np.concatenate([[0], np.cumsum(kv_lens)]).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    sink = synth.normal_f32(seed, synth.STREAM_SINK, hq) if has_sink else None
    return DecodeInputs(q, k, v, kv_indices, kv_indptr, cu_q, sink, q_lens, kv_lens)


DECODE_KINDS = ("swa", "global")


def decode_batch(kind: str, seed: int = 0, num_seqs: int = 64, q_len: int = 8, kv_lo: int = 1024,
                 kv_hi: int = 8192, threads=None, contiguous: bool = False):
    """A serving-shaped batch for the KV-cache path: num_seqs requests (SGLang's cap of 64 running
    requests), q_len = 8 new tokens each (8 speculative draft tokens), context lengths uniform in
    [kv_lo, kv_hi].  The sliding-window layer (64 Q / 8 KV heads, window 128, sink, base 1e4) keeps
    only each request's last window + q_len rows in its cache, as a sliding-window pool does; the
    index entries of older positions point at row 0 and are never read.  The global layer (64 Q /
    4 KV heads, base 1e7) keeps every row.  Cache rows are a seeded random permutation (a
    fragmented page-size-1 pool), or, with ``contiguous``, each request's rows in order (a pool
    filled request by request).  Returns (DecodeInputs, layer_kind, window, rope_base)."""
    assert kind in DECODE_KINDS
    kv = [int(x) for x in synth.seq_lengths(seed, num_seqs, kv_lo, kv_hi)]
    ql = [min(q_len, x) for x in kv]
    if kind == "swa":
        hq, hkv, window, base, has_sink = 64, 8, SWA_WINDOW, ROPE_BASE_SWA, True
        stored = [min(x, window + q) for x, q in zip(kv, ql)]
    else:
        hq, hkv, window, base, has_sink = 64, 4, -1, ROPE_BASE_GLOBAL, False
        stored = list(kv)
    rows = sum(stored) + 1
    q = synth.normal_bf16(seed, synth.STREAM_Q, (sum(ql), hq, 192), threads)
    k = synth.normal_bf16(seed, synth.STREAM_K, (rows, hkv, 192), threads)
    v = synth.normal_bf16(seed, synth.STREAM_V, (rows, hkv, 128), threads)
    if contiguous:
        perm = np.arange(1, rows, dtype=np.int32)
    else:
        perm = (1 + np.argsort(synth.uniforms(seed, synth.STREAM_PAGES, rows - 1), kind="stable")).astype(np.int32)
    idx, used = [], 0
    for x, st in zip(kv, stored):
        idx.append(np.zeros(x - st, dtype=np.int32))
        idx.append(perm[used:used + st])
        used += st
    kv_indices = np.concatenate(idx).astype(np.int32)
    kv_indptr = np.concatenate([[0], np.cumsum(kv)]).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)
    sink = synth.normal_f32(seed, synth.STREAM_SINK, hq) if has_sink else None
    layer = LAYER_SWA if kind == "swa" else LAYER_GLOBAL
    return DecodeInputs(q, k, v, kv_indices, kv_indptr, cu_q, sink, ql, kv), layer, window, base


def decode_subset(x: DecodeInputs, seqs) -> DecodeInputs:
    """The same problem restricted to the given sequences (for bounded reference checks)."""
    qs, idx, kv, ql = [], [], [], []
    for b in seqs:
        qs.append(x.q[x.cu_q[b]:x.cu_q[b + 1]])
        idx.append(x.kv_indices[x.kv_indptr[b]:x.kv_indptr[b + 1]])
        kv.append(x.kv_lens[b])
        ql.append(x.q_lens[b])
    return DecodeInputs(np.concatenate(qs), x.k_cache, x.v_cache, np.concatenate(idx).astype(np.int32),
                        np.concatenate([[0], np.cumsum(kv)]).astype(np.int32),
                        np.concatenate([[0], np.cumsum(ql)]).astype(np.int32), x.sink, ql, kv)
