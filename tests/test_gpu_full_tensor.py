"""Whole-tensor parity at the full workload sizes: every element of ``out`` and
``lse`` from the CUDA path (default kernel choice, as the benchmark launches
it) against the FP64 oracle on the same seeded inputs.

The oracle runs over all rows in chunks, so that its FP64 output never has to
be held whole (the 131072-token layer's would be 8.6 GB); the squared norms
behind the relative L2 error are summed over the chunks, so the metric is the
one taken over the whole ``out`` tensor.

Layers: the sliding-window layer with sink at 4096 tokens, its varlen form
(16 packed sequences), the global causal layer (2 x 8192 tokens, 4 KV heads)
and the 131072-token sliding-window layer -- the configurations of the model's
two layer kinds (miles docs "MiMo-V2.6-Flash", section 1 Model Introduction:
window 128 with sink on the sliding layers, 4 KV heads and RoPE base 1e7 on
the global ones; section 5.4 Notable quirks: the query plus 128 previous keys).
"""
import numpy as np
import pytest
import torch

import oracle
from global_attention_moe_b200 import workloads as W
from gpu_helpers import TOL_LSE, TOL_MAX_ABS, TOL_REL_L2, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from global_attention_moe_b200 import mimo_attn
    mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)
    assert mimo_attn.check() == mimo_attn.OK


def whole_tensor_errors(w, x, out, lse, rows_per_chunk):
    """max-abs, whole-tensor rel-L2 and LSE max-abs of the GPU result against the
    oracle, the oracle evaluated chunk by chunk over every token row."""
    T = w.total_tokens
    diff2 = ref2 = 0.0
    max_abs = lse_abs = 0.0
    finite = True
    for r0 in range(0, T, rows_per_chunk):
        rows = np.arange(r0, min(T, r0 + rows_per_chunk), dtype=np.int64)
        ref_out, ref_lse = oracle.attn_fwd(x.q, x.k, x.v, x.sink, x.cu_seqlens, w.window, w.rope_base,
                                           w.rope_dims, w.v_scale, rows=rows)
        g = out[r0:r0 + len(rows)].float().cpu().numpy().astype(np.float64)
        gl = lse[:, r0:r0 + len(rows)].cpu().numpy().astype(np.float64)
        finite &= bool(np.all(np.isfinite(g)) and np.all(np.isfinite(gl)))
        d = g - ref_out
        diff2 += float(np.sum(d * d))
        ref2 += float(np.sum(ref_out * ref_out))
        max_abs = max(max_abs, float(np.max(np.abs(d))))
        lse_abs = max(lse_abs, float(np.max(np.abs(gl - ref_lse))))
    return {"rows": T, "max_abs": max_abs, "rel_l2": float(np.sqrt(diff2 / ref2)), "lse_max_abs": lse_abs,
            "finite": finite}


@pytest.mark.parametrize("name,chunk", [("swa4096", 4096), ("swa_varlen", 4096), ("global", 1024),
                                        ("swa_long", 4096)])
def test_full_size_every_element_against_oracle(name, chunk):
    w = W.WORKLOADS[name]()
    x = W.make_inputs(w)
    out, lse = run_gpu(w, x)
    err = whole_tensor_errors(w, x, out, lse, chunk)
    print(f"\n{w.name}: every element of out and lse: max-abs {err['max_abs']:.3e}, "
          f"rel-L2 {err['rel_l2']:.3e}, LSE {err['lse_max_abs']:.3e} over {err['rows']} rows x {w.num_q_heads} heads")
    assert err["finite"], name
    assert err["max_abs"] <= TOL_MAX_ABS, err
    assert err["rel_l2"] <= TOL_REL_L2, err
    assert err["lse_max_abs"] <= TOL_LSE, err
