"""Cases for the host build of the whole library (tensor-core kernels through the device model),
checked against the oracle with the forward tolerances.  Run as a child process:

    python library_cases.py <libmimo_attn_host.so> <case> [<case> ...]
"""
import ctypes as C
import os
import sys

import numpy as np

TESTS = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(TESTS))
sys.path.insert(0, TESTS)
import oracle  # noqa: E402
from global_attention_moe_b200 import synth, workloads as W  # noqa: E402
from decode_helpers import decode_reference  # noqa: E402

TOL_MAX_ABS, TOL_REL_L2, TOL_LSE = 2e-2, 5e-3, 1e-3
KERNEL = {"auto": 0, "simple": 1, "pipelined": 2, "window": 3, "packed": 4}
DECODE = {"auto": 0, "cuda_cores": 1, "tensor": 2}
vp = C.c_void_p


class Dims(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("num_seqs", "total_tokens", "max_seqlen", "num_q_heads", "num_kv_heads",
                                         "head_dim_qk", "head_dim_v")]


class DecodeDims(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("num_seqs", "total_q", "total_kv", "cache_rows", "max_q_len", "max_kv_len",
                                         "num_q_heads", "num_kv_heads", "head_dim_qk", "head_dim_v")]


class Lib:
    def __init__(self, path):
        L = self.L = C.CDLL(path)
        L.hemu_alloc.restype = vp
        L.hemu_alloc.argtypes = [C.c_size_t]
        L.hemu_free.argtypes = [vp]
        L.mimo_attn_fwd.argtypes = [vp, vp, vp, vp, vp, C.POINTER(Dims), C.c_int, C.c_int, C.c_double, C.c_int,
                                    C.c_float, vp, vp, vp]
        L.mimo_attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, C.POINTER(DecodeDims), C.c_int, C.c_int,
                                       C.c_double, C.c_int, C.c_float, vp, vp, vp]
        L.mimo_attn_check.argtypes = [vp]
        L.mimo_attn_bwd.argtypes = [vp, vp, vp, vp, vp, C.POINTER(Dims), C.c_int, C.c_int, C.c_double, C.c_int,
                                    C.c_float, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        self.live = []

    def put(self, a):
        if a is None:
            return None
        a = np.ascontiguousarray(a)
        p = self.L.hemu_alloc(max(a.nbytes, 1))
        C.memmove(p, a.ctypes.data, a.nbytes)
        self.live.append(p)
        return p

    def empty(self, nbytes):
        p = self.L.hemu_alloc(max(nbytes, 1))
        self.live.append(p)
        return p

    def get(self, p, shape, dtype):
        a = np.empty(shape, dtype=dtype)
        C.memmove(a.ctypes.data, p, a.nbytes)
        return a

    def finish(self, status):
        while self.live:
            self.L.hemu_free(self.live.pop())
        assert status == 0, f"status {status}"
        assert self.L.hemu_errors() == 0, "device-model or barrier error"
        st = self.L.mimo_attn_check(None)
        assert st == 0, f"kernel error status {st}"


def check(out_bits, lse, ro, rl):
    out = synth.bf16_bits_to_f32(out_bits).astype(np.float64)
    d = out - ro
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    assert np.max(np.abs(d)) <= TOL_MAX_ABS, np.max(np.abs(d))
    assert np.linalg.norm(d) / np.linalg.norm(ro) <= TOL_REL_L2
    assert np.max(np.abs(lse - rl)) <= TOL_LSE, np.max(np.abs(lse - rl))


def fwd(H, w, kernel):
    x = W.make_inputs(w)
    T, hq = w.total_tokens, w.num_q_heads
    d = Dims(w.num_seqs, T, w.max_seqlen, hq, w.num_kv_heads, 192, 128)
    assert H.L.mimo_attn_set_kernel(KERNEL[kernel]) == 0
    po, pl = H.empty(T * hq * 128 * 2), H.empty(hq * T * 4)
    st = H.L.mimo_attn_fwd(H.put(x.q), H.put(x.k), H.put(x.v), H.put(x.sink), H.put(x.cu_seqlens), C.byref(d),
                           w.layer_kind, w.window, w.rope_base, 64, 0.707, po, pl, None)
    out, lse = H.get(po, (T, hq, 128), np.uint16), H.get(pl, (hq, T), np.float32).astype(np.float64)
    H.L.mimo_attn_set_kernel(0)
    H.finish(st)
    check(out, lse, *oracle.attn_fwd(x.q, x.k, x.v, x.sink, x.cu_seqlens, w.window, w.rope_base))


def decode(H, kv, ql, hq, hkv, layer, window, base, has_sink, seed, kernel="tensor"):
    x = W.make_decode_inputs(kv, ql, hq, hkv, has_sink, seed)
    Tq = int(sum(ql))
    d = DecodeDims(len(kv), Tq, int(sum(kv)), x.k_cache.shape[0], max(ql), max(kv), hq, hkv, 192, 128)
    assert H.L.mimo_attn_set_decode_kernel(DECODE[kernel]) == 0
    po, pl = H.empty(Tq * hq * 128 * 2), H.empty(hq * Tq * 4)
    st = H.L.mimo_attn_decode(H.put(x.q), H.put(x.k_cache), H.put(x.v_cache), H.put(x.kv_indices),
                              H.put(x.kv_indptr), H.put(x.cu_q), H.put(x.sink), C.byref(d), layer, window, base, 64,
                              0.707, po, pl, None)
    out, lse = H.get(po, (Tq, hq, 128), np.uint16), H.get(pl, (hq, Tq), np.float32).astype(np.float64)
    H.L.mimo_attn_set_decode_kernel(0)
    H.finish(st)
    check(out, lse, *decode_reference(x, window if layer == W.LAYER_SWA else -1, base))


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


def bwd(H, lens, hq, hkv, layer, window, base, has_sink, seed, kernel, tol):
    """The backward against the oracle's, with dLSE shifted by -dO . (out_stored - out) (the kernels form
    D from the stored BF16 out; the gradients are linear in dLSE)."""
    rng = np.random.default_rng(seed)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = synth.f32_to_bf16_bits(rng.standard_normal((T, hq, 192)).astype(np.float32))
    k = synth.f32_to_bf16_bits(rng.standard_normal((T, hkv, 192)).astype(np.float32))
    v = synth.f32_to_bf16_bits(rng.standard_normal((T, hkv, 128)).astype(np.float32))
    sink = rng.standard_normal(hq).astype(np.float32) if has_sink else None
    go = synth.f32_to_bf16_bits(rng.standard_normal((T, hq, 128)).astype(np.float32))
    gl = (rng.standard_normal((hq, T)) * 0.3).astype(np.float32)
    w = window if layer == W.LAYER_SWA else -1
    out, lse = oracle.attn_fwd(q, k, v, sink, cu, w, base)
    out_b = f64_to_bf16_bits(out)
    d = Dims(len(lens), T, max(lens), hq, hkv, 192, 128)
    shapes = ((T, hq, 192), (T, hkv, 192), (T, hkv, 128), (hq,))
    ptrs = [H.empty(int(np.prod(s)) * 4) for s in shapes[:3]] + [H.empty(hq * 4) if has_sink else None]
    assert H.L.mimo_attn_set_bwd_kernel({"cuda_cores": 1, "tensor": 2}[kernel]) == 0
    st = H.L.mimo_attn_bwd(H.put(q), H.put(k), H.put(v), H.put(sink), H.put(cu), C.byref(d), layer, window, base, 64,
                           0.707, H.put(out_b), H.put(lse.astype(np.float32)), H.put(go), H.put(gl), *ptrs, None)
    got = [None if p is None else H.get(p, s, np.float32) for p, s in zip(ptrs, shapes)]
    H.L.mimo_attn_set_bwd_kernel(0)
    H.finish(st)
    go64 = synth.bf16_bits_to_f32(go).astype(np.float64)
    shift = np.einsum("thd,thd->ht", go64, synth.bf16_bits_to_f32(out_b).astype(np.float64) - out)
    ref = oracle.attn_bwd(q, k, v, sink, cu, w, base, 64, 0.707, go64, gl.astype(np.float64) - shift)
    for name, a, r in zip(("dq", "dk", "dv", "dsink"), got, ref):
        if r is not None:
            rel = np.linalg.norm(a.astype(np.float64) - r) / np.linalg.norm(r)
            assert rel <= tol, f"{kernel} {name}: rel-L2 {rel:.2e}"


def fwd_timeout(H, kernel):
    """With a wait limit of zero the waits on other roles give up: the kernel must record a timeout and
    leave without a deadlock or a warp-collective instruction with exited lanes."""
    w = W.tiny_swa()
    x = W.make_inputs(w)
    T, hq = w.total_tokens, w.num_q_heads
    d = Dims(w.num_seqs, T, w.max_seqlen, hq, w.num_kv_heads, 192, 128)
    assert H.L.mimo_attn_set_kernel(KERNEL[kernel]) == 0
    po, pl = H.empty(T * hq * 128 * 2), H.empty(hq * T * 4)
    st = H.L.mimo_attn_fwd(H.put(x.q), H.put(x.k), H.put(x.v), H.put(x.sink), H.put(x.cu_seqlens), C.byref(d),
                           w.layer_kind, w.window, w.rope_base, 64, 0.707, po, pl, None)
    H.L.mimo_attn_set_kernel(0)
    while H.live:
        H.L.hemu_free(H.live.pop())
    assert st == 0 and H.L.hemu_errors() == 0, "deadlock or warp-collective with exited lanes"
    assert H.L.mimo_attn_check(None) == 4, "timeout not reported"  # MIMO_ERR_TIMEOUT


CASES = {
    # the three forward kernels on the small sliding-window config (T = 512, 4 query heads, 1 KV head)
    "fwd_tiny_simple": lambda H: fwd(H, W.tiny_swa(), "simple"),
    "fwd_tiny_pipelined": lambda H: fwd(H, W.tiny_swa(), "pipelined"),
    "fwd_tiny_window": lambda H: fwd(H, W.tiny_swa(), "window"),
    # ragged sequences across the 128-row tile and window edges; the global layer
    "fwd_ragged_swa": lambda H: fwd(H, W.custom("ragged", W.LAYER_SWA, [1, 129, 257, 0, 5], 4, 2, 128, 1e4, True), "auto"),
    "fwd_global": lambda H: fwd(H, W.custom("glob", W.LAYER_GLOBAL, [300, 77], 4, 2, -1, 1e7, False), "auto"),
    # the tensor-core KV-cache kernel: decode and speculative chunks, then 128-row tiles
    "decode_tensor": lambda H: decode(H, [5, 129, 300, 64], [1, 8, 3, 8], 8, 2, W.LAYER_SWA, 128, 1e4, True, 71),
    "decode_tensor_tiles_swa": lambda H: decode(H, [600, 90], [300, 20], 8, 2, W.LAYER_SWA, 128, 1e4, True, 72),
    "decode_tensor_tiles_global": lambda H: decode(H, [200, 50], [36, 50], 8, 1, W.LAYER_GLOBAL, -1, 1e7, False, 73),
    # tile edges on both kernels: exactly 128 rows; 129 rows (a one-row tile); 6 query heads per KV head
    # (a token's heads straddle two tiles); window 0 over a whole prompt
    "decode_tile_edges": lambda H: [decode(H, kv, ql, hq, hkv, layer, win, base, sink, seed, kernel=k)
                                    for k in ("tensor", "cuda_cores")
                                    for kv, ql, hq, hkv, layer, win, base, sink, seed in (
                                        ([300, 40], [16, 16], 8, 1, W.LAYER_SWA, 128, 1e4, True, 81),
                                        ([300, 129], [43, 43], 6, 2, W.LAYER_SWA, 128, 1e4, True, 82),
                                        ([500, 200], [30, 25], 6, 1, W.LAYER_GLOBAL, -1, 1e7, False, 83),
                                        ([260, 700], [260, 100], 12, 2, W.LAYER_SWA, 0, 1e4, False, 84))],
    # the backward on the tensor cores (BF16 operands: 1e-2) and on the CUDA cores (FP32: 1e-4)
    "bwd_tensor": lambda H: [bwd(H, *c, "tensor", 1e-2) for c in (
        ([300, 129, 17, 1], 8, 2, W.LAYER_SWA, 128, 1e4, True, 41), ([200, 70], 4, 2, W.LAYER_SWA, 0, 1e4, False, 42),
        ([333, 64, 5], 8, 2, W.LAYER_GLOBAL, -1, 1e7, False, 43), ([150, 40], 6, 2, W.LAYER_SWA, 128, 1e4, True, 44),
        ([90, 30], 2, 2, W.LAYER_GLOBAL, -1, 1e7, False, 45))],
    "bwd_cuda_cores": lambda H: bwd(H, [300, 129, 17, 1], 8, 2, W.LAYER_SWA, 128, 1e4, True, 41, "cuda_cores", 1e-4),
    # the packed window kernel (query heads of a KV group in the tile's rows): 32 tokens x 4 heads on the
    # small config; 16 tokens x 8 heads across ragged and empty sequences, windows 0 .. 128 (run with few
    # SMs so that each CTA walks several tiles, continuing windows and starting new ones)
    "fwd_tiny_packed": lambda H: fwd(H, W.tiny_swa(), "packed"),
    "fwd_packed_g8": lambda H: fwd(H, W.custom("pk8", W.LAYER_SWA, [1, 17, 129, 300, 0, 5, 160], 16, 2, 128, 1e4,
                                               True, seed=91), "packed"),
    "fwd_packed_windows": lambda H: [fwd(H, W.custom("pkw", W.LAYER_SWA, [250, 33], 8, 1, win, 1e4, win % 2 == 0,
                                                     seed=92 + win), "packed") for win in (0, 1, 15, 16, 17, 127)],
    "fwd_packed_g4_ragged": lambda H: fwd(H, W.custom("pk4", W.LAYER_SWA, [31, 32, 33, 200], 8, 2, 128, 1e4, True,
                                                      seed=93), "packed"),
    # only for a build whose wait limit is zero
    "fwd_timeout_pipelined": lambda H: fwd_timeout(H, "pipelined"),
    "fwd_timeout_window": lambda H: fwd_timeout(H, "window"),
    "fwd_timeout_packed": lambda H: fwd_timeout(H, "packed"),
}
TIMEOUT_CASES = ("fwd_timeout_pipelined", "fwd_timeout_window", "fwd_timeout_packed")
PACKED_CASES = ("fwd_tiny_packed", "fwd_packed_g8", "fwd_packed_windows", "fwd_packed_g4_ragged")

if __name__ == "__main__":
    H = Lib(sys.argv[1])
    for name in sys.argv[2:]:
        CASES[name](H)
        print("ok", name, flush=True)
