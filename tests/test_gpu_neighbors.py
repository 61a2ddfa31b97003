"""GPU parity of the steps beside the attention kernel (FP8 blockwise dequant, fused-QKV split, output
projection, MoE router) against the numpy oracle: bit-exact for the dequant and the split; the
projection within the BF16 rounding of its outputs; the router's choice equal where the FP32 keys
are not tied, weights to FP32 rounding."""
import numpy as np
import pytest
import torch

from oracle import neighbors as NB

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def f64_to_bf16_bits(x):
    """Round-to-nearest-even of FP64 values to BF16, one rounding: 8 significant bits in the normal
    range, the fixed grid of 2^-133 below 2^-126 (subnormals), infinity past the largest finite value."""
    x = np.asarray(x, dtype=np.float64)
    b = x.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    r = (b + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)  # 8 significant bits left
    with np.errstate(over="ignore"):
        f32 = r.view(np.float64).astype(np.float32)  # exact: at most 8 significant bits
    out = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    sub = np.abs(x) < 2.0 ** -126
    m = np.rint(np.abs(x[sub]) * 2.0 ** 133).astype(np.uint16)  # rint rounds halves to even
    out[sub] = m | (np.signbit(x[sub]).astype(np.uint16) << np.uint16(15))
    return out


@pytest.mark.parametrize("shape,block", [((300, 512), (128, 128)), ((128, 16), (128, 128)), ((77, 96), (32, 48)),
                                         ((45, 160), (16, 40)), ((20, 64), (3, 8)),
                                         ((5, 4352), (2, 128)), ((3, 8224), (1, 48))])
def test_fp8_dequant_bit_exact(shape, block):
    _dequant_case(shape, block, False)


# Scales for the rounding of the dequant products (a product rounded to FP32 first and then to BF16
# differs from the single rounding on the first kind).
TIE_SCALES = np.concatenate([
    # FP32 scales whose products with 32-45 of the E4M3 values lie just beside a BF16 midpoint, closer
    # than half an FP32 ulp (found by comparing both roundings over 2e6 random scales)
    np.array([1070475106, 1071501685, 1070290262, 1072649557, 1068944589, 1068420301], dtype=np.uint32)
    .view(np.float32),
    # 8883769 * 2^-149, near the bottom of FP32's normal range: its product with 1.125 lies 2^-152 above
    # a BF16 midpoint, below FP32's smallest subnormal, so an FP32 error term would lose that sticky bit
    np.array([8883769], dtype=np.uint32).view(np.float32),
    # products exactly on midpoints (ties to even), far below the normal range (the FP64 path), either
    # side of 2^-96, past the largest finite value (infinity), and of both signs
    np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -9, 2.0 ** -110, 3 * 2.0 ** -112, 1.37 * 2.0 ** -100, 1.5 * 2.0 ** 120,
              -1.3], dtype=np.float32)])


@pytest.mark.parametrize("shape,block", [((256, 512), (8, 16)), ((40, 96), (1, 1))])
def test_fp8_dequant_rounding_midpoints(shape, block):
    _dequant_case(shape, block, True)


def _dequant_case(shape, block, ties):
    from global_attention_moe_b200 import mimo_attn as M
    rng = np.random.default_rng(51)
    codes = rng.integers(0, 256, size=shape).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3F  # no NaN codes
    gs = (-(-shape[0] // block[0]), -(-shape[1] // block[1]))
    scale = (np.exp2(rng.integers(-8, 8, size=gs)) * rng.uniform(1, 2, size=gs)).astype(np.float32)
    if ties:
        scale = TIE_SCALES[rng.integers(0, len(TIE_SCALES), size=gs)]
    out = M.fp8_dequant_blockwise(torch.from_numpy(codes).cuda(), torch.from_numpy(scale).cuda(), block)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    want = f64_to_bf16_bits(NB.dequant_fp8_blockwise(codes, scale.astype(np.float64), block))
    assert np.array_equal(got, want)


@pytest.mark.parametrize("hq,hkv,T", [(64, 8, 257), (64, 4, 100), (8, 8, 3), (6, 2, 9)])
def test_qkv_split_bit_exact(hq, hkv, T):
    from global_attention_moe_b200 import mimo_attn as M
    rng = np.random.default_rng(52)
    width = hkv * (hq // hkv * 192 + 192 + 128)
    fused = rng.integers(0, 1 << 16, size=(T, width)).astype(np.uint16)
    q, k, v = M.qkv_split(torch.from_numpy(fused.view(np.int16)).cuda().view(torch.bfloat16), hq, hkv)
    rq, rk, rv = NB.split_qkv(fused, hq, hkv)
    for a, r in ((q, rq), (k, rk), (v, rv)):
        assert np.array_equal(a.view(torch.int16).cpu().numpy().view(np.uint16), r)


@pytest.mark.parametrize("E,k,T,shift", [(256, 8, 4099, 0.0), (64, 8, 33, 0.0), (32, 1, 7, 0.0), (256, 16, 1001, 0.0),
                                         (256, 17, 999, 0.0), (256, 20, 513, 0.0), (256, 8, 777, -2.0),
                                         (64, 20, 301, -2.0)])
def test_route(E, k, T, shift):
    """Ids equal to the oracle's up to FP32 key ties; with the bias shifted by -2 every key is negative."""
    from global_attention_moe_b200 import mimo_attn as M
    rng = np.random.default_rng(53)
    logits = (rng.standard_normal((T, E)) * 2).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.1 + shift).astype(np.float32)
    ids, w = M.moe_route(torch.from_numpy(logits).cuda(), torch.from_numpy(bias).cuda(), k)
    ids, w = ids.cpu().numpy(), w.cpu().numpy().astype(np.float64)
    rid, rw, key = NB.route(logits, bias, k)
    same = np.all(ids == rid, axis=1)
    # rows that differ must be a different order of FP32 keys that tie within one rounding of the sigmoid
    for t in np.nonzero(~same)[0]:
        kk = key[t, ids[t]]
        assert len(set(ids[t].tolist())) == k
        assert np.all(np.abs(np.sort(kk)[::-1] - key[t, rid[t]]) <= 2 * np.spacing(np.abs(key[t, rid[t]])))
    assert same.mean() > 0.999
    assert np.max(np.abs(w[same] - rw[same])) <= 1e-6
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)


@pytest.mark.parametrize("T,hq,N", [(300, 8, 512), (1, 64, 4096), (130, 64, 264)])
def test_linear_proj(T, hq, N):
    """y = x . W^T (cuBLAS, FP32 accumulation, one BF16 rounding per output) against the FP64 oracle.
    Tolerance from the arithmetic: the BF16 rounding of each output is at most 2^-9 relative (RMS
    about 2^-9 / sqrt(3) = 1.1e-3 over many outputs); FP32 accumulation over K <= 8192 terms adds
    about sqrt(K) 2^-24 = 5e-6.  So rel-L2 <= 2e-3, and each output within 2^-8 |y| plus 1e-3 of
    the outputs' RMS."""
    from global_attention_moe_b200 import mimo_attn as M
    rng = np.random.default_rng(54)
    K = hq * 128
    bf16 = lambda a: (a.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    x = bf16(rng.standard_normal((T, hq, 128)))
    w = bf16(rng.standard_normal((N, K)) / np.sqrt(K))
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    y = M.linear_proj(dev(x), dev(w))
    assert M.check() == M.OK
    assert tuple(y.shape) == (T, N)
    got = NB.bf16_bits_to_f64(y.view(torch.int16).cpu().numpy().view(np.uint16))
    ref = NB.linear_proj(x.reshape(T, K), w)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 2e-3
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-3 * np.sqrt(np.mean(ref ** 2)))


def test_route_exact_ties_take_lower_experts():
    """Rows of equal logits with a zero bias tie on every key: the choice is experts 0..k-1, in order,
    and the normalised weights are all 1/k."""
    from global_attention_moe_b200 import mimo_attn as M
    logits = np.full((5, 256), 0.25, dtype=np.float32)
    ids, w = M.moe_route(torch.from_numpy(logits).cuda(), torch.zeros(256).cuda(), 8)
    assert M.check() == M.OK
    assert np.array_equal(ids.cpu().numpy(), np.tile(np.arange(8, dtype=np.int32), (5, 1)))
    assert np.allclose(w.cpu().numpy(), 1.0 / 8, rtol=0, atol=1e-7)


@pytest.mark.parametrize("E,k,adjacent", [(256, 8, False), (64, 32, False), (256, 8, True), (256, 20, True)])
def test_route_tied_pairs(E, k, adjacent):
    """Every key twice (experts e and e + E/2, or 2i and 2i + 1, share logit and bias): the top k are
    pairs of exact ties, each ordered by the lower expert first, and the ids match the oracle row for
    row."""
    from global_attention_moe_b200 import mimo_attn as M
    rng = np.random.default_rng(57)
    logits = (rng.standard_normal((301, E)) * 2).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.1).astype(np.float32)
    if adjacent:
        logits[:, 1::2] = logits[:, 0::2]
        bias[1::2] = bias[0::2]
    else:
        logits[:, E // 2:] = logits[:, :E // 2]
        bias[E // 2:] = bias[:E // 2]
    ids, w = M.moe_route(torch.from_numpy(logits).cuda(), torch.from_numpy(bias).cuda(), k)
    assert M.check() == M.OK
    ids, w = ids.cpu().numpy(), w.cpu().numpy().astype(np.float64)
    rid, rw, key = NB.route(logits, bias, k)
    same = np.all(ids == rid, axis=1)
    assert same.mean() > 0.99
    assert np.max(np.abs(w[same] - rw[same])) <= 1e-6
    for t in range(len(ids)):  # within every pair of equal keys the lower expert comes first
        kk = key[t, ids[t]]
        for a in range(k - 1):
            if kk[a] == kk[a + 1]:
                assert ids[t, a] < ids[t, a + 1]


def test_empty_inputs():
    """Zero tokens / rows: nothing to launch, empty results."""
    from global_attention_moe_b200 import mimo_attn as M
    ids, w = M.moe_route(torch.zeros((0, 256)).cuda(), torch.zeros(256).cuda(), 8)
    assert tuple(ids.shape) == (0, 8) and tuple(w.shape) == (0, 8)
    q, k, v = M.qkv_split(torch.zeros((0, 8 * (8 * 192 + 320)), dtype=torch.bfloat16).cuda(), 64, 8)
    assert tuple(q.shape) == (0, 64, 192) and tuple(k.shape) == (0, 8, 192) and tuple(v.shape) == (0, 8, 128)
    out = M.fp8_dequant_blockwise(torch.zeros((0, 512), dtype=torch.uint8).cuda(), torch.ones((0, 4)).cuda())
    assert tuple(out.shape) == (0, 512)
    y = M.linear_proj(torch.zeros((0, 8, 128), dtype=torch.bfloat16).cuda(), torch.zeros((64, 1024), dtype=torch.bfloat16).cuda())
    assert tuple(y.shape) == (0, 64)
    assert M.check() == M.OK
