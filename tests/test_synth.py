"""The seeded input generator: SplitMix64 against its scalar definition, BF16
rounding against torch, chunking and stream independence."""
import numpy as np
import pytest
import torch

from global_attention_moe_b200 import synth, workloads


def test_splitmix64_matches_scalar_definition():
    cnt = np.array([0, 1, 2, 12345, (3 << 40) + 7, (1 << 63) + 5], dtype=np.uint64)
    for seed in (0, 1, 0xDEADBEEF, (1 << 64) - 1):
        vec = synth.splitmix64(seed, cnt)
        for c, z in zip(cnt.tolist(), vec.tolist()):
            assert z == synth.splitmix64_scalar(seed, c)


def test_splitmix64_published_sequence():
    # First outputs of SplitMix64 seeded with 0 (the state advances by the golden gamma first).
    assert synth.splitmix64_scalar(0, 0) == 0xE220A8397B1DCDAF
    assert synth.splitmix64_scalar(0, 1) == 0x6E789E6AA1B965F4


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.00390625, 1.01171875, -1.00390625, 0.0, -0.0, 3.0e38, 1e-40], dtype=np.float32)])
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(synth.bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_normals_chunking_and_offsets():
    a = synth.normal_bf16(0, synth.STREAM_Q, (3, 5, 7))
    flat = synth._normals_chunk(0, synth.STREAM_Q, 0, 105).astype(np.float32)
    assert np.array_equal(a.reshape(-1), synth.f32_to_bf16_bits(flat))
    # an odd offset regenerates the same elements
    part = synth._normals_chunk(0, synth.STREAM_Q, 33, 40)
    assert np.array_equal(part, synth._normals_chunk(0, synth.STREAM_Q, 0, 73)[33:])
    # multi-chunk generation equals single-shot
    n = synth._CHUNK + 1001
    big = synth.normal_bf16(3, synth.STREAM_K, (n,), threads=4)
    assert np.array_equal(big[-50:], synth.f32_to_bf16_bits(
        synth._normals_chunk(3, synth.STREAM_K, n - 50, 50).astype(np.float32)))


def test_normal_moments_and_streams():
    x = synth.bf16_bits_to_f32(synth.normal_bf16(0, synth.STREAM_Q, (200000,))).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    y = synth.bf16_bits_to_f32(synth.normal_bf16(0, synth.STREAM_K, (200000,))).astype(np.float64)
    assert abs(np.corrcoef(x, y)[0, 1]) < 0.01


def test_varlen_lengths():
    w = workloads.swa_varlen()
    assert len(w.lengths) == 16 and all(256 <= L <= 2048 for L in w.lengths)
    assert w.lengths == workloads.swa_varlen().lengths
    cu = synth.cu_seqlens_from_lengths(w.lengths)
    assert cu[0] == 0 and cu[-1] == w.total_tokens and np.all(np.diff(cu) == np.array(w.lengths))


def test_workload_pair_counts():
    # SWA: sum_p min(p+1, 129) = 129 L - 8256 for L >= 129; causal: L(L+1)/2
    assert workloads.attended_pairs([4096], 128, 1) == 129 * 4096 - 8256
    assert workloads.attended_pairs([8192, 8192], -1, 1) == 8192 * 8193
    assert workloads.attended_pairs([512], 128, 4) == 4 * (129 * 512 - 8256)


@pytest.mark.parametrize("kind", workloads.DECODE_KINDS)
@pytest.mark.parametrize("contiguous", [False, True])
def test_decode_batch_rows(kind, contiguous):
    """Every stored cache row is used by exactly one key; the sliding layer's older positions
    point at row 0 (never read); the contiguous layout keeps each request's rows in order."""
    x, layer, window, base = workloads.decode_batch(kind, seed=3, num_seqs=5, kv_lo=100, kv_hi=400, contiguous=contiguous)
    stored = []
    for b, kv in enumerate(x.kv_lens):
        idx = x.kv_indices[x.kv_indptr[b]:x.kv_indptr[b + 1]]
        assert len(idx) == kv
        keep = min(kv, window + x.q_lens[b]) if window >= 0 else kv
        assert np.all(idx[:kv - keep] == 0)
        live = idx[kv - keep:]
        assert np.all((live >= 1) & (live < x.k_cache.shape[0]))
        if contiguous:
            assert np.all(np.diff(live) == 1)
        stored.append(live)
    allrows = np.concatenate(stored)
    assert len(np.unique(allrows)) == len(allrows) == x.k_cache.shape[0] - 1
