"""Reference for the KV-cache path: a decode step equals selected rows of the
forward over each whole sequence.  The oracle is run on that forward problem
(the cached K/V rows gathered in position order, the new queries placed at
their positions, every other query row zero and not selected)."""
from __future__ import annotations

import numpy as np

import oracle
from global_attention_moe_b200 import workloads


def decode_reference(x: workloads.DecodeInputs, window, rope_base, rope_dims=64, v_scale=0.707):
    """Oracle out [Tq, Hq, 128] and lse [Hq, Tq] (FP64) for a DecodeInputs batch."""
    hq = x.q.shape[1]
    qs, ks, vs, rows = [], [], [], []
    off = 0
    for b, (kv_len, q_len) in enumerate(zip(x.kv_lens, x.q_lens)):
        idx = x.kv_indices[x.kv_indptr[b]:x.kv_indptr[b + 1]]
        ks.append(x.k_cache[idx])
        vs.append(x.v_cache[idx])
        qf = np.zeros((kv_len, hq, 192), dtype=np.uint16)
        qf[kv_len - q_len:] = x.q[x.cu_q[b]:x.cu_q[b + 1]]
        qs.append(qf)
        rows.extend(range(off + kv_len - q_len, off + kv_len))
        off += kv_len
    cu = np.concatenate([[0], np.cumsum(x.kv_lens)]).astype(np.int32)
    return oracle.attn_fwd(np.concatenate(qs), np.concatenate(ks), np.concatenate(vs), x.sink, cu, window,
                           rope_base, rope_dims, v_scale, rows=np.asarray(rows, dtype=np.int64))


def decode_gpu(x: workloads.DecodeInputs, layer_kind, window, rope_base, rope_dims=64, v_scale=0.707, dev="cuda"):
    import torch
    from global_attention_moe_b200 import mimo_attn
    t = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    sink = None if x.sink is None else torch.from_numpy(x.sink).to(dev)
    out, lse = mimo_attn.decode(t(x.q), t(x.k_cache), t(x.v_cache), i32(x.kv_indices), i32(x.kv_indptr),
                                i32(x.cu_q), sink, max(x.q_lens), max(x.kv_lens), layer_kind, window, rope_base,
                                rope_dims, v_scale)
    st = mimo_attn.check()
    assert st == mimo_attn.OK, mimo_attn.status_string(st)
    return out, lse
