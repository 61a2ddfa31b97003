"""GPU parity of the KV-cache path above 128 query rows per KV head (chunked prefill) on both kernels:
128-row tiles as one more dimension of the work, each tile's keys clipped to its rows' positions, and
the combine reading the splits that overlap the token's tile."""
import numpy as np
import pytest
import torch

from global_attention_moe_b200 import workloads as W
from decode_helpers import decode_gpu, decode_reference
from gpu_helpers import assert_within, errors, out_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from global_attention_moe_b200 import mimo_attn
    assert mimo_attn.check() == mimo_attn.OK


@pytest.fixture(params=["tensor", "cuda_cores"], autouse=True)
def dkernel(request):
    from global_attention_moe_b200 import mimo_attn
    mimo_attn.set_decode_kernel(mimo_attn.DECODE_TENSOR if request.param == "tensor" else mimo_attn.DECODE_CUDA_CORES)
    yield request.param
    mimo_attn.set_decode_kernel(mimo_attn.DECODE_AUTO)


def parity(x, layer, window, base):
    out, lse = decode_gpu(x, layer, window, base)
    ro, rl = decode_reference(x, window, base)
    assert_within(errors(out_to_f64(out), lse.cpu().numpy().astype(np.float64), ro, rl), "decode")


def test_rows_per_kv_head_above_128(dkernel):
    """9 and 12 new tokens x 16 heads = 144 and 192 rows per KV head: two row tiles."""
    from global_attention_moe_b200 import mimo_attn
    x = W.make_decode_inputs([40, 300], [9, 12], 64, 4, False, seed=37)
    parity(x, W.LAYER_GLOBAL, -1, 1e7)


@pytest.mark.parametrize("kind", ["swa", "global"])
def test_chunked_prefill(kind, dkernel):
    """Chunks of new tokens far above 128 rows per KV head against a cached prefix, and a whole short
    prompt as one chunk: row tiles, each tile's keys clipped to its rows' positions, and the splits
    merged per tile.  The automatic choice runs them (on the CUDA-core kernel)."""
    from global_attention_moe_b200 import mimo_attn
    kv = [1200, 700, 300, 129]
    ql = [300, 200, 300, 64]
    if kind == "swa":
        parity(W.make_decode_inputs(kv, ql, 64, 8, True, seed=38), W.LAYER_SWA, 128, 1e4)
    else:
        parity(W.make_decode_inputs(kv, ql, 64, 4, False, seed=39), W.LAYER_GLOBAL, -1, 1e7)
