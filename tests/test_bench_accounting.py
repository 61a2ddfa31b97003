"""The benchmark's algorithmic bytes and FLOPs against closed forms (every tensor moved once:
46,336 bytes per token for the sliding layer, 43,776 for the global one; 2 x 192 + 2 x 128 = 640
FLOPs per attended pair) and against hand counts for the KV-cache step."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from global_attention_moe_b200 import workloads as W  # noqa: E402


@pytest.mark.parametrize("name,per_token", [("swa4096", 46336), ("global", 43776)])
def test_forward_bytes_per_token(name, per_token):
    w = W.WORKLOADS[name]()
    assert bench.bytes_per_step(w) == per_token * w.total_tokens


def test_forward_flops_swa4096():
    # 4096 queries, each sees min(p + 1, 129) keys: 129 * 4096 - 128 * 129 / 2 = 520,128 pairs per head
    w = W.WORKLOADS["swa4096"]()
    assert bench.flops_per_step(w) == 640 * 520128 * 64


def test_forward_flops_global():
    w = W.WORKLOADS["global"]()
    assert bench.flops_per_step(w) == 640 * 2 * (8192 * 8193 // 2) * 64


def test_decode_bytes_and_flops_by_hand():
    # two requests: 5 keys / 2 new tokens and 300 keys / 3 new tokens; 8 Q heads, 2 KV heads, window 128
    x = W.make_decode_inputs([5, 300], [2, 3], 8, 2, True, seed=1)
    nbytes, flops = bench.decode_bytes_flops(x, 128)
    keys = 5 + 131  # the second request's new tokens see its last 128 + 3 keys
    assert nbytes == keys * (2 * (192 + 128) * 2 + 4) + 5 * 8 * (192 * 2 + 128 * 2 + 4)
    pairs = (4 + 5) + 3 * 129  # positions 3, 4 of the first request; 297..299 of the second
    assert flops == 640 * pairs * 8
    # the global layer reads every key and attends all earlier positions
    nbytes, flops = bench.decode_bytes_flops(x, -1)
    assert nbytes == 305 * (2 * (192 + 128) * 2 + 4) + 5 * 8 * (192 * 2 + 128 * 2 + 4)
    assert flops == 640 * ((4 + 5) + (298 + 299 + 300)) * 8


def test_step_lines_by_hand():
    """The step lines' algorithmic counts against hand counts of their shapes."""
    # backward: 1664 FLOPs per attended pair (S, dQ, dK over 192 dims; dP, dV over 128)
    flops, nbytes, units = bench.step_accounting("bwd")
    assert flops == 1664 * 520128 * 64 and units == 4096
    assert nbytes == 4096 * (64 * (384 + 512 + 4 + 768) + 8 * (384 + 256 + 768 + 512))
    assert bench.step_accounting("bwd_tc") == (flops, nbytes, units)
    # FP8 dequant of a 14848 x 4096 weight: 1 byte in, 2 out per element, 116 x 32 FP32 scales
    assert bench.step_accounting("dequant") == (0, 14848 * 4096 * 3 + 116 * 32 * 4, 14848 * 4096)
    # fused-QKV split: 8 groups x (8 x 192 + 192 + 128) = 14848 BF16 per token, read and written once
    assert bench.step_accounting("split") == (0, 16384 * 14848 * 2 * 2, 16384)
    # output projection 4096 x 8192 by 8192 x 4096
    assert bench.step_accounting("proj") == (2 * 4096 * 8192 * 4096, 2 * (2 * 4096 * 8192 + 4096 * 4096), 4096)
    # router: FP32 logits and bias in, int32 ids and FP32 weights of the top 8 out
    assert bench.step_accounting("route") == (0, 262144 * 256 * 4 + 256 * 4 + 262144 * 8 * 8, 262144)
