"""GPU parity of the KV-cache path (mimo_attn_decode) against the oracle, and
against the forward kernel on the same sequences; edge cases and error
reporting."""
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
    """Every test runs on both decode kernels (tcgen05, and FP32 on the CUDA cores)."""
    from global_attention_moe_b200 import mimo_attn
    mimo_attn.set_decode_kernel(mimo_attn.DECODE_TENSOR if request.param == "tensor" else mimo_attn.DECODE_CUDA_CORES)
    yield request.param
    mimo_attn.set_decode_kernel(mimo_attn.DECODE_AUTO)


def parity(x, layer, window, base):
    out, lse = decode_gpu(x, layer, window, base)
    ro, rl = decode_reference(x, window, base)
    assert_within(errors(out_to_f64(out), lse.cpu().numpy().astype(np.float64), ro, rl), "decode")


@pytest.mark.parametrize("hq,hkv", [(64, 8), (8, 2), (4, 1), (8, 8)])
def test_swa_sink(hq, hkv):
    """Sliding window 128 with a sink: single-token decode, speculative chunks of up to 8, a whole
    short sequence as its own chunk, and keys on both sides of the window edge."""
    kv = [1, 5, 128, 129, 130, 300, 1000, 8]
    ql = [1, 1, 8, 3, 8, 2, 8, 8]
    parity(W.make_decode_inputs(kv, ql, hq, hkv, True, seed=31), W.LAYER_SWA, 128, 1e4)


@pytest.mark.parametrize("window", [0, 1, 31, 127])
def test_swa_windows(window):
    parity(W.make_decode_inputs([40, 300, 7], [8, 4, 7], 8, 2, False, seed=32), W.LAYER_SWA, window, 1e4)


def test_global_long_context_splits():
    """Global layer (16 query heads per KV head, 8 new tokens = 128 rows), contexts long enough that
    the keys are split over many CTAs and merged."""
    kv = [1, 700, 3000]
    ql = [1, 8, 4]
    parity(W.make_decode_inputs(kv, ql, 64, 4, False, seed=33), W.LAYER_GLOBAL, -1, 1e7)


def test_many_sequences_single_token():
    rng = np.random.default_rng(34)
    kv = [int(v) for v in rng.integers(1, 600, size=64)]
    parity(W.make_decode_inputs(kv, [1] * 64, 64, 8, True, seed=34), W.LAYER_SWA, 128, 1e4)


def test_matches_forward_kernel_rows():
    """With the cache holding each sequence's K/V in order, the decode of the last q_len tokens
    equals the forward kernel's rows for them (two independently written kernels)."""
    from global_attention_moe_b200 import mimo_attn
    w = W.custom("dec_fwd", W.LAYER_SWA, [300, 129, 17], 8, 2, 128, 1e4, True, seed=35)
    x = W.make_inputs(w)
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    sink = torch.from_numpy(x.sink).cuda()
    out_f, lse_f = mimo_attn.fwd(dev(x.q), dev(x.k), dev(x.v), sink, torch.from_numpy(x.cu_seqlens).cuda(),
                                 w.max_seqlen, W.LAYER_SWA, 128, 1e4)
    q_lens = [8, 3, 17]
    rows = np.concatenate([np.arange(int(x.cu_seqlens[b + 1]) - q, int(x.cu_seqlens[b + 1]))
                           for b, q in enumerate(q_lens)])
    cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    idx = torch.arange(w.total_tokens, dtype=torch.int32, device="cuda")
    out_d, lse_d = mimo_attn.decode(dev(np.ascontiguousarray(x.q[rows])), dev(x.k), dev(x.v), idx,
                                    torch.from_numpy(x.cu_seqlens).cuda(), torch.from_numpy(cu_q).cuda(), sink,
                                    max(q_lens), w.max_seqlen, W.LAYER_SWA, 128, 1e4)
    assert mimo_attn.check() == mimo_attn.OK
    rt = torch.from_numpy(rows).cuda()
    a, b = out_d.float(), out_f.index_select(0, rt).float()
    assert float((a - b).abs().max()) <= 2e-2
    assert float((a - b).norm() / b.norm()) <= 5e-3
    assert float((lse_d - lse_f.index_select(1, rt)).abs().max()) <= 1e-3


def test_bad_index_and_lengths_reported():
    """Cache rows outside the cache and q_len > kv_len are reported (no row outside the cache is read)."""
    from global_attention_moe_b200 import mimo_attn
    x = W.make_decode_inputs([50, 60], [2, 3], 8, 2, False, seed=36)
    x.kv_indices = x.kv_indices.copy()
    x.kv_indices[7] = x.k_cache.shape[0] + 1000
    with pytest.raises(AssertionError, match="cu_seqlens inconsistent"):
        decode_gpu(x, W.LAYER_SWA, 128, 1e4)
    y = W.make_decode_inputs([50, 60], [2, 3], 8, 2, False, seed=36)
    y.cu_q = np.array([0, 2, 5], dtype=np.int32)
    y.kv_indptr = np.array([0, 50, 52], dtype=np.int32)  # second sequence: 3 new tokens, 2 keys
    y.kv_lens = [50, 2]
    y.kv_indices = y.kv_indices[:52].copy()
    with pytest.raises(AssertionError, match="cu_seqlens inconsistent"):
        decode_gpu(y, W.LAYER_SWA, 128, 1e4)
    assert mimo_attn.check() == mimo_attn.OK


def test_chunk_and_ring_boundaries():
    """Contexts at and around the 64-key step of the tensor-core kernel, and long enough per CTA
    (24 requests x 4 KV heads: few splits) that its 4-stage ring wraps several times."""
    kv = [63, 64, 65, 128, 191, 192, 257, 320, 1500, 2000, 2600, 3100, 4000, 3500, 900, 1200,
          2222, 3333, 1111, 777, 2048, 2049, 3999, 66]
    ql = [1, 8, 2, 8, 3, 8, 4, 8, 5, 6, 7, 8, 1, 2, 3, 4, 5, 6, 7, 8, 8, 8, 8, 2]
    parity(W.make_decode_inputs(kv, ql, 64, 4, False, seed=38), W.LAYER_GLOBAL, -1, 1e7)


@pytest.mark.parametrize("kind", W.DECODE_KINDS)
def test_serving_batch_sampled(kind):
    """The bench's serving batch (64 requests, 8 new tokens, contexts 1024..8192) in its own launch
    configuration: requests 0, 1 and the last against the oracle."""
    x, layer, window, base = W.decode_batch(kind)
    out, lse = decode_gpu(x, layer, window, base)
    seqs = [0, 1, len(x.kv_lens) - 1]
    ro, rl = decode_reference(W.decode_subset(x, seqs), window, base)
    rows = np.concatenate([np.arange(x.cu_q[b], x.cu_q[b + 1]) for b in seqs])
    assert_within(errors(out_to_f64(out)[rows], lse.cpu().numpy().astype(np.float64)[:, rows], ro, rl), kind)


@pytest.mark.parametrize("kind", W.DECODE_KINDS)
def test_kernels_agree_on_serving_batch(kind, dkernel):
    """Every output row of the two decode kernels (written independently) agree on the full batch."""
    from global_attention_moe_b200 import mimo_attn
    if dkernel != "tensor":
        pytest.skip("one comparison per batch")
    x, layer, window, base = W.decode_batch(kind, seed=1)
    out_t, lse_t = decode_gpu(x, layer, window, base)
    mimo_attn.set_decode_kernel(mimo_attn.DECODE_CUDA_CORES)
    out_c, lse_c = decode_gpu(x, layer, window, base)
    a, b = out_t.float(), out_c.float()
    assert bool(torch.isfinite(a).all())
    assert float((a - b).abs().max()) <= 2e-2
    assert float((a - b).norm() / b.norm()) <= 5e-3
    assert float((lse_t - lse_c).abs().max()) <= 1e-3
