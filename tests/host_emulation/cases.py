"""Cases for the host-compiled CUDA-core kernels, checked against the oracle.  Run as a child process
(an out-of-range access is a segfault there, not in the test runner):

    python cases.py <libhost_kernels.so> <mode> <case> [<case> ...]

mode 0: every buffer ends at a guard page; mode 1: every buffer starts right after one.

Backward: the kernel forms D = dO . out from the stored BF16 out.  The gradients are linear in dLSE and
D enters only as (dLSE - D), so the kernel's result is the method's exact gradient with dLSE replaced
by dLSE - dO . (out_stored - out); the oracle is given that shifted dLSE.  What is left is FP32
arithmetic (dot products of 192 / 128 terms, sums over the keys): rel-L2 <= 1e-4 per gradient.
"""
import ctypes as C
import os
import sys

import numpy as np

TESTS = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(TESTS))
sys.path.insert(0, TESTS)
import oracle  # noqa: E402
from oracle import neighbors as NB  # noqa: E402
from global_attention_moe_b200 import synth, workloads as W  # noqa: E402
from decode_helpers import decode_reference  # noqa: E402

# forward tolerances (BF16 out): max-abs, rel-L2, LSE max-abs
TOL_MAX_ABS, TOL_REL_L2, TOL_LSE = 2e-2, 5e-3, 1e-3
DECODE_AUTO, DECODE_CUDA_CORES, DECODE_TENSOR = 0, 1, 2
ERR_UNSUPPORTED = 2

TOL_BWD = 1e-4
LAYER_SWA, LAYER_GLOBAL = 0, 1
vp = C.c_void_p


class Dims(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("num_seqs", "total_tokens", "max_seqlen", "num_q_heads", "num_kv_heads",
                                         "head_dim_qk", "head_dim_v")]


class DecodeDims(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("num_seqs", "total_q", "total_kv", "cache_rows", "max_q_len", "max_kv_len",
                                         "num_q_heads", "num_kv_heads", "head_dim_qk", "head_dim_v")]


class Host:
    def __init__(self, path):
        L = self.L = C.CDLL(path)
        L.hemu_alloc.restype = vp
        L.hemu_alloc.argtypes = [C.c_size_t]
        L.hemu_free.argtypes = [vp]
        L.hemu_error_word.restype = C.c_uint
        L.mimo_attn_bwd.argtypes = [vp, vp, vp, vp, vp, C.POINTER(Dims), C.c_int, C.c_int, C.c_double, C.c_int,
                                    C.c_float, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.mimo_fp8_dequant_blockwise.argtypes = [vp, vp, C.c_int64, C.c_int64, C.c_int, C.c_int, vp, vp]
        L.mimo_qkv_split.argtypes = [vp, C.c_int64, C.c_int, C.c_int, vp, vp, vp, vp]
        L.mimo_moe_route.argtypes = [vp, vp, C.c_int64, C.c_int, C.c_int, C.c_int, vp, vp, vp]
        L.mimo_attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, C.POINTER(DecodeDims), C.c_int, C.c_int,
                                       C.c_double, C.c_int, C.c_float, vp, vp, vp]
        L.mimo_attn_set_decode_kernel.argtypes = [C.c_int]
        L.mimo_attn_set_bwd_kernel.argtypes = [C.c_int]
        assert L.mimo_attn_set_bwd_kernel(1) == 0  # the CUDA-core backward: the one this library holds
        self.live = []

    def put(self, a):
        if a is None:
            return None
        a = np.ascontiguousarray(a)
        p = self.L.hemu_alloc(max(a.nbytes, 1))
        C.memmove(p, a.ctypes.data, a.nbytes)
        self.live.append(p)
        return p

    def empty(self, shape, dtype):
        p = self.L.hemu_alloc(max(int(np.prod(shape)) * np.dtype(dtype).itemsize, 1))
        self.live.append(p)
        return p

    def get(self, p, shape, dtype):
        a = np.empty(shape, dtype=dtype)
        C.memmove(a.ctypes.data, p, a.nbytes)
        return a

    def done(self, status):
        while self.live:
            self.L.hemu_free(self.live.pop())
        assert status == 0, f"status {status}"
        assert self.L.hemu_errors() == 0, "barrier deadlock or warp-collective with exited lanes"
        w = self.L.hemu_error_word()
        assert w == 0, f"kernel error word {w}"


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


def bwd(H, lens, hq, hkv, layer, window, base, has_sink, seed, dlse=True):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = synth.f32_to_bf16_bits(rng.standard_normal((T, hq, 192)).astype(np.float32))
    k = synth.f32_to_bf16_bits(rng.standard_normal((T, hkv, 192)).astype(np.float32))
    v = synth.f32_to_bf16_bits(rng.standard_normal((T, hkv, 128)).astype(np.float32))
    sink = rng.standard_normal(hq).astype(np.float32) if has_sink else None
    go = synth.f32_to_bf16_bits(rng.standard_normal((T, hq, 128)).astype(np.float32))
    gl = (rng.standard_normal((hq, T)) * 0.3).astype(np.float32) if dlse else None
    w = window if layer == LAYER_SWA else -1
    out, lse = oracle.attn_fwd(q, k, v, sink, cu, w, base)
    out_b = f64_to_bf16_bits(out)
    d = Dims(len(lens), T, max(lens), hq, hkv, 192, 128)
    shapes = ((T, hq, 192), (T, hkv, 192), (T, hkv, 128), (hq,))
    ptrs = [H.empty(s, np.float32) for s in shapes[:3]] + [H.empty(shapes[3], np.float32) if has_sink else None]
    st = H.L.mimo_attn_bwd(H.put(q), H.put(k), H.put(v), H.put(sink), H.put(cu), C.byref(d), layer, window, base, 64,
                           0.707, H.put(out_b), H.put(lse.astype(np.float32)), H.put(go), H.put(gl), *ptrs, None)
    got = [None if p is None else H.get(p, s, np.float32) for p, s in zip(ptrs, shapes)]
    H.done(st)
    go64 = synth.bf16_bits_to_f32(go).astype(np.float64)
    shift = np.einsum("thd,thd->ht", go64, synth.bf16_bits_to_f32(out_b).astype(np.float64) - out)
    gl_eff = (0.0 if gl is None else gl.astype(np.float64)) - shift
    ref = oracle.attn_bwd(q, k, v, sink, cu, w, base, 64, 0.707, go64, gl_eff)
    for name, a, r in zip(("dq", "dk", "dv", "dsink"), got, ref):
        if r is None:
            assert a is None
            continue
        rel = np.linalg.norm(a.astype(np.float64) - r) / np.linalg.norm(r)
        assert rel <= TOL_BWD, f"{name}: rel-L2 {rel:.2e}"


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


def dequant(H, shape, block, seed=51, ties=False):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=shape).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3F  # no NaN codes
    gs = (-(-shape[0] // block[0]), -(-shape[1] // block[1]))
    scale = (np.exp2(rng.integers(-8, 8, size=gs)) * rng.uniform(1, 2, size=gs)).astype(np.float32)
    if ties:
        scale = TIE_SCALES[rng.integers(0, len(TIE_SCALES), size=gs)]
    po = H.empty(shape, np.uint16)
    st = H.L.mimo_fp8_dequant_blockwise(H.put(codes), H.put(scale), shape[0], shape[1], block[0], block[1], po, None)
    got = H.get(po, shape, np.uint16)
    H.done(st)
    assert np.array_equal(got, f64_to_bf16_bits(NB.dequant_fp8_blockwise(codes, scale.astype(np.float64), block)))


def split(H, hq, hkv, T, seed=52):
    rng = np.random.default_rng(seed)
    fused = rng.integers(0, 1 << 16, size=(T, hkv * (hq // hkv * 192 + 320))).astype(np.uint16)
    shapes = ((T, hq, 192), (T, hkv, 192), (T, hkv, 128))
    ptrs = [H.empty(s, np.uint16) for s in shapes]
    st = H.L.mimo_qkv_split(H.put(fused), T, hq, hkv, *ptrs, None)
    got = [H.get(p, s, np.uint16) for p, s in zip(ptrs, shapes)]
    H.done(st)
    for a, r in zip(got, NB.split_qkv(fused, hq, hkv)):
        assert np.array_equal(a, r.reshape(a.shape))


def route(H, E, k, T, normalize=True, ties=False, pairs=False, adjacent=False, shift=0.0, seed=53):
    rng = np.random.default_rng(seed)
    logits = (rng.standard_normal((T, E)) * 2).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.1 + shift).astype(np.float32)  # shift -2: every key negative
    if ties:  # rows of equal logits with a zero bias: the choice is the k lowest expert indices
        logits[::3] = 0.5
        bias[:] = 0
    if pairs:  # every key twice (experts e and e + E/2): the top k are pairs of exact ties
        logits[:, E // 2:] = logits[:, :E // 2]
        bias[E // 2:] = bias[:E // 2]
    if adjacent:  # every key twice (experts 2i and 2i + 1, held by different lanes): pairs of exact ties
        logits[:, 1::2] = logits[:, 0::2]
        bias[1::2] = bias[0::2]
    pi, pw = H.empty((T, k), np.int32), H.empty((T, k), np.float32)
    st = H.L.mimo_moe_route(H.put(logits), H.put(bias), T, E, k, int(normalize), pi, pw, None)
    ids, w = H.get(pi, (T, k), np.int32), H.get(pw, (T, k), np.float32).astype(np.float64)
    H.done(st)
    rid, rw, _ = NB.route(logits, bias, k, normalize)
    assert np.array_equal(ids, rid)
    assert np.max(np.abs(w - rw)) <= 1e-6 * max(1.0, np.max(np.abs(rw)))


def decode(H, kv, ql, hq, hkv, layer, window, base, has_sink, seed, choice=DECODE_AUTO, expect=0, bad_index=False):
    """The KV-cache path through mimo_attn_decode on the CUDA-core kernel (the tensor-core kernel is a
    stub here that flags an error if launched)."""
    x = W.make_decode_inputs(kv, ql, hq, hkv, has_sink, seed)
    if bad_index:  # cache rows past the end of the cache, and a negative one
        x.kv_indices = x.kv_indices.copy()
        x.kv_indices[[3, len(x.kv_indices) - 1]] = [x.k_cache.shape[0] + 1000, -7]
    Tq = int(sum(ql))
    d = DecodeDims(len(kv), Tq, int(sum(kv)), x.k_cache.shape[0], max(ql), max(kv), hq, hkv, 192, 128)
    po, pl = H.empty((Tq, hq, 128), np.uint16), H.empty((hq, Tq), np.float32)
    assert H.L.mimo_attn_set_decode_kernel(choice) == 0
    st = H.L.mimo_attn_decode(H.put(x.q), H.put(x.k_cache), H.put(x.v_cache), H.put(x.kv_indices),
                              H.put(x.kv_indptr), H.put(x.cu_q), H.put(x.sink), C.byref(d), layer, window, base, 64,
                              0.707, po, pl, None)
    H.L.mimo_attn_set_decode_kernel(DECODE_AUTO)
    if expect:
        H.done(0)
        assert st == expect, f"status {st}, expected {expect}"
        return
    if bad_index:  # reported for mimo_attn_check; the guard pages show no row outside the cache was read
        assert st == 0 and H.L.hemu_error_word() == 4, "bad index not reported as BAD_SEQLENS"
        H.done(0)
        return
    out = synth.bf16_bits_to_f32(H.get(po, (Tq, hq, 128), np.uint16)).astype(np.float64)
    lse = H.get(pl, (hq, Tq), np.float32).astype(np.float64)
    H.done(st)
    ro, rl = decode_reference(x, window if layer == LAYER_SWA else -1, base)
    diff = out - ro
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    assert np.max(np.abs(diff)) <= TOL_MAX_ABS, np.max(np.abs(diff))
    assert np.linalg.norm(diff) / np.linalg.norm(ro) <= TOL_REL_L2
    assert np.max(np.abs(lse - rl)) <= TOL_LSE, np.max(np.abs(lse - rl))


CASES = {
    "bwd_swa_sink": lambda H: bwd(H, [300, 129, 17, 1], 8, 2, LAYER_SWA, 128, 1e4, True, 41),
    "bwd_window0": lambda H: bwd(H, [200, 70], 4, 2, LAYER_SWA, 0, 1e4, False, 42),
    "bwd_window31_mqa": lambda H: bwd(H, [90, 33], 4, 1, LAYER_SWA, 31, 1e4, True, 46),
    "bwd_global": lambda H: bwd(H, [333, 64, 5], 8, 2, LAYER_GLOBAL, -1, 1e7, False, 43),
    "bwd_no_dlse": lambda H: bwd(H, [150], 4, 4, LAYER_SWA, 128, 1e4, True, 44, dlse=False),
    # 16-code chunks inside one scale block, across two (40-column blocks), and across several (8)
    "dequant": lambda H: (dequant(H, (300, 512), (128, 128)), dequant(H, (77, 96), (32, 48)),
                          dequant(H, (45, 160), (16, 40)), dequant(H, (20, 64), (3, 8)),
                          dequant(H, (64, 256), (4, 16), ties=True), dequant(H, (40, 96), (1, 1), ties=True),
                          dequant(H, (5, 4352), (2, 128)), dequant(H, (3, 8224), (1, 48), ties=True)),
    "split": lambda H: (split(H, 64, 8, 33), split(H, 6, 2, 9), split(H, 8, 8, 3), split(H, 64, 4, 17)),
    "route": lambda H: (route(H, 256, 8, 200), route(H, 64, 8, 33), route(H, 32, 1, 7),
                        route(H, 256, 8, 64, normalize=False), route(H, 96, 32, 40, ties=True),
                        route(H, 32, 8, 12, ties=True), route(H, 256, 8, 50, pairs=True),
                        route(H, 64, 32, 20, pairs=True), route(H, 256, 17, 40), route(H, 256, 20, 40, adjacent=True),
                        route(H, 256, 8, 40, adjacent=True), route(H, 256, 8, 40, shift=-2.0),
                        route(H, 64, 20, 30, shift=-2.0)),
    # 40 new tokens x 4 heads = 160 rows (two tiles) beside one-tile sequences; keys clipped per tile
    "decode_tiles_swa": lambda H: decode(H, [300, 90, 20], [40, 20, 20], 8, 2, LAYER_SWA, 128, 1e4, True, 61,
                                         choice=DECODE_CUDA_CORES),
    # a 300-token chunk (ten tiles) after a 300-token prefix: later tiles start several splits in
    "decode_tiles_swa_long": lambda H: decode(H, [600, 64], [300, 64], 8, 2, LAYER_SWA, 128, 1e4, True, 65,
                                              choice=DECODE_CUDA_CORES),
    # three and seven tiles, the second sequence a whole prompt as one chunk
    "decode_tiles_global": lambda H: decode(H, [200, 50], [36, 50], 8, 1, LAYER_GLOBAL, -1, 1e7, False, 62,
                                            choice=DECODE_CUDA_CORES),
    # the CUDA-core kernel forced on one-tile sequences (decode and speculative chunks)
    "decode_one_tile": lambda H: decode(H, [5, 129, 300], [1, 8, 3], 8, 2, LAYER_SWA, 128, 1e4, True, 63,
                                        choice=DECODE_CUDA_CORES),
    # cache indices outside the cache: reported, never dereferenced
    "decode_bad_index": lambda H: decode(H, [50, 300], [2, 40], 8, 2, LAYER_SWA, 128, 1e4, True, 66,
                                         choice=DECODE_CUDA_CORES, bad_index=True),
}

if __name__ == "__main__":
    lib, mode = sys.argv[1], int(sys.argv[2])
    H = Host(lib)
    H.L.hemu_set_mode(mode)
    for name in sys.argv[3:]:
        CASES[name](H)
        print("ok", name, flush=True)
