"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
run the CUDA path through the C-ABI binding, run the oracle on the same
inputs and compare with the tolerances the method states."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from global_attention_moe_b200 import workloads

# Tolerances (on BF16 out vs the FP64 oracle, and FP32 LSE): max-abs, rel-L2, LSE abs.
TOL_MAX_ABS = 2e-2
TOL_REL_L2 = 5e-3
TOL_LSE = 1e-3


def to_device(x: workloads.Inputs, dev="cuda"):
    q = torch.from_numpy(x.q.view(np.int16)).to(dev).view(torch.bfloat16)
    k = torch.from_numpy(x.k.view(np.int16)).to(dev).view(torch.bfloat16)
    v = torch.from_numpy(x.v.view(np.int16)).to(dev).view(torch.bfloat16)
    s = None if x.sink is None else torch.from_numpy(x.sink).to(dev)
    cu = torch.from_numpy(x.cu_seqlens).to(dev)
    return q, k, v, s, cu


def run_gpu(w: workloads.Workload, x: workloads.Inputs, dev_inputs=None, out=None, lse=None):
    from global_attention_moe_b200 import mimo_attn
    q, k, v, s, cu = dev_inputs if dev_inputs is not None else to_device(x)
    out, lse = mimo_attn.fwd(q, k, v, s, cu, w.max_seqlen, w.layer_kind, w.window, w.rope_base, w.rope_dims,
                             w.v_scale, out=out, lse=lse)
    st = mimo_attn.check()
    assert st == mimo_attn.OK, mimo_attn.status_string(st)
    return out, lse


def out_to_f64(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy().astype(np.float64)


def run_oracle(w: workloads.Workload, x: workloads.Inputs, rows=None):
    return oracle.attn_fwd(x.q, x.k, x.v, x.sink, x.cu_seqlens, w.window, w.rope_base, w.rope_dims, w.v_scale,
                           rows=rows)


def errors(gpu_out: np.ndarray, gpu_lse: np.ndarray, ref_out: np.ndarray, ref_lse: np.ndarray) -> dict:
    diff = gpu_out - ref_out
    return {
        "max_abs": float(np.max(np.abs(diff))) if diff.size else 0.0,
        "rel_l2": float(np.linalg.norm(diff) / max(np.linalg.norm(ref_out), 1e-300)) if diff.size else 0.0,
        "lse_max_abs": float(np.max(np.abs(gpu_lse - ref_lse))) if gpu_lse.size else 0.0,
        "finite": bool(np.all(np.isfinite(gpu_out)) and np.all(np.isfinite(gpu_lse))),
    }


def assert_within(err: dict, what: str = ""):
    assert err["finite"], f"{what}: non-finite output"
    assert err["max_abs"] <= TOL_MAX_ABS, f"{what}: max-abs {err['max_abs']:.3e}"
    assert err["rel_l2"] <= TOL_REL_L2, f"{what}: rel-L2 {err['rel_l2']:.3e}"
    assert err["lse_max_abs"] <= TOL_LSE, f"{what}: LSE {err['lse_max_abs']:.3e}"


def sample_rows(w: workloads.Workload, n_random=48, seed=123) -> np.ndarray:
    """Rows the oracle computes one by one at full size: each sequence's first
    rows, rows around the 128-row tile and window boundaries, its last rows,
    plus seeded random rows."""
    cu = np.concatenate([[0], np.cumsum(w.lengths)])
    rows = set()
    for b, L in enumerate(w.lengths):
        s = int(cu[b])
        for p in (0, 1, 2, 126, 127, 128, 129, 130, 255, 256, 257, L // 2, L - 129, L - 2, L - 1):
            if 0 <= p < L:
                rows.add(s + p)
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, w.total_tokens, n_random).tolist())
    return np.array(sorted(rows), dtype=np.int64)
