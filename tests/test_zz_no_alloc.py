"""mimo_attn_fwd_noalloc: the entry point for callers that cannot allocate
device memory during the call (a framework that has reserved the device for
its own caching allocator, a serving loop that forbids allocation on its hot
path).  Its results must match the default entry point's, call after call,
while it keeps its scratch in a fixed array inside the library.

It is collected after every other GPU module (tests/conftest.py puts it last),
so that a failure here cannot stop another suite under -x.
"""
import numpy as np
import pytest
import torch

from global_attention_moe_b200 import workloads as W
from gpu_helpers import to_device

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
    # T * Hkv = 262144 rows of 64 FP16 dims: the scratch array exactly full
    W.custom("noalloc_at_limit", W.LAYER_GLOBAL, [4096] * 8, 16, 8, -1, 1e7, False, seed=24),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_default_entry_on_two_calls(w):
    """Both entry points launch the same kernels on the same inputs, so their
    outputs agree bit for bit, on the first call and on the next one (which
    finds the previous call's contents in the shared scratch array)."""
    from global_attention_moe_b200 import mimo_attn
    x = W.make_inputs(w)
    q, k, v, s, cu = to_device(x)
    ref_out, ref_lse = mimo_attn.fwd(q, k, v, s, cu, w.max_seqlen, w.layer_kind, w.window, w.rope_base)
    assert mimo_attn.check() == mimo_attn.OK
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        mimo_attn.fwd_noalloc(q, k, v, s, cu, w.max_seqlen, w.layer_kind, w.window, w.rope_base, out, lse)
        assert mimo_attn.check() == mimo_attn.OK, f"call {call}"
        assert torch.equal(out, ref_out), f"call {call}: out differs from the default entry point"
        assert torch.equal(lse, ref_lse), f"call {call}: lse differs from the default entry point"
