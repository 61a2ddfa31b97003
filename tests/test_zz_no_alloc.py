"""mimo_attn_fwd_noalloc: the entry point for callers that cannot allocate
device memory during the call (a framework that has reserved the device for
its own caching allocator, a serving loop that forbids allocation on its hot
path).  Its results must match the default entry point's, call after call,
while it keeps its scratch in a fixed array inside the library.

It is collected after the forward and KV-cache suites (tests/conftest.py
orders the GPU modules by when they were established).
"""
import numpy as np
import pytest
import torch

from global_attention_moe_b200 import workloads as W
from gpu_helpers import TOL_LSE, TOL_MAX_ABS, TOL_REL_L2, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from global_attention_moe_b200 import mimo_attn
    mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)
    mimo_attn.check()  # start from a clear error word


CASES = [
    W.custom("noalloc_swa", W.LAYER_SWA, [700, 129, 1], 16, 2, 128, 1e4, True, seed=21),
    W.custom("noalloc_global", W.LAYER_GLOBAL, [900, 300], 8, 2, -1, 1e7, False, seed=22),
    W.custom("noalloc_odd_group", W.LAYER_SWA, [260], 3, 1, 128, 1e4, True, seed=23),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_default_entry_on_two_calls(w):
    from global_attention_moe_b200 import mimo_attn
    x = W.make_inputs(w)
    q, k, v, s, cu = to_device(x)
    ref_out, ref_lse = mimo_attn.fwd(q, k, v, s, cu, w.max_seqlen, w.layer_kind, w.window, w.rope_base)
    assert mimo_attn.check() == mimo_attn.OK
    ref = ref_out.float().cpu().numpy().astype(np.float64)
    ref_l = ref_lse.cpu().numpy().astype(np.float64)
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        mimo_attn.fwd_noalloc(q, k, v, s, cu, w.max_seqlen, w.layer_kind, w.window, w.rope_base, out, lse)
        assert mimo_attn.check() == mimo_attn.OK, f"call {call}"
        got = out.float().cpu().numpy().astype(np.float64)
        got_l = lse.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)) and np.all(np.isfinite(got_l)), f"call {call}"
        d = got - ref
        assert np.abs(d).max() <= TOL_MAX_ABS, f"call {call}"
        assert np.linalg.norm(d) / np.linalg.norm(ref) <= TOL_REL_L2, f"call {call}"
        assert np.abs(got_l - ref_l).max() <= TOL_LSE, f"call {call}"


def test_noalloc_rejects_problems_beyond_its_scratch():
    from global_attention_moe_b200 import mimo_attn
    limit_rows = mimo_attn.noalloc_scratch_bytes() // 128  # T * Hkv rows of 64 FP16 dims
    hkv = 8
    T = limit_rows // hkv + 128
    dims = mimo_attn.make_dims(1, T, T, 16, hkv)
    fake = 1 << 20  # never dereferenced: the size check comes first
    st = mimo_attn.LIB.mimo_attn_fwd_noalloc(fake, fake, fake, None, fake, mimo_attn.ctypes.byref(dims), 0, 128,
                                             1e4, 64, 0.707, fake, fake, None)
    assert st == mimo_attn.ERR_SCRATCH_LIMIT
    assert "scratch" in mimo_attn.status_string(st)
