"""Python binding of the C-ABI library ``libmimo_attn.so`` (include/mimo_attn.h).

Argument marshalling only: torch tensors supply device memory and the current
CUDA stream; every step of the attention forward runs in the library's CUDA
kernels.  There is no CPU or eager fallback -- if the library is missing the
import of this module raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "_build", "libmimo_attn.so")

LAYER_SWA = 0
LAYER_GLOBAL = 1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_RANGE, ERR_BAD_SEQLENS, ERR_SCRATCH_LIMIT = range(8)

# Every symbol include/mimo_attn.h declares.
SYMBOLS = ("mimo_attn_fwd", "mimo_attn_host_workspace_size", "mimo_attn_fwd_host", "mimo_attn_check",
           "mimo_attn_selftest_wait_timeout", "mimo_attn_status_string", "mimo_attn_fwd_noalloc",
           "mimo_attn_noalloc_scratch_bytes", "mimo_attn_set_kernel", "mimo_attn_profile_start",
           "mimo_attn_profile_stop", "mimo_attn_profile_set_stride", "mimo_attn_decode", "mimo_attn_set_decode_kernel", "mimo_attn_version",
           "mimo_attn_bwd", "mimo_fp8_dequant_blockwise", "mimo_qkv_split", "mimo_moe_route",
           "mimo_linear_proj", "mimo_attn_set_bwd_kernel")
KERNEL_AUTO, KERNEL_SIMPLE, KERNEL_PIPELINED, KERNEL_WINDOW, KERNEL_WINDOW_PACKED = 0, 1, 2, 3, 4
DECODE_AUTO, DECODE_CUDA_CORES, DECODE_TENSOR = 0, 1, 2


class Dims(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int32), ("max_seqlen", ctypes.c_int32),
                ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim_qk", ctypes.c_int32), ("head_dim_v", ctypes.c_int32)]


class DecodeDims(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("total_q", ctypes.c_int32), ("total_kv", ctypes.c_int32),
                ("cache_rows", ctypes.c_int32), ("max_q_len", ctypes.c_int32), ("max_kv_len", ctypes.c_int32),
                ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim_qk", ctypes.c_int32), ("head_dim_v", ctypes.c_int32)]


class MimoAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m global_attention_moe_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, D, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_float
    lib.mimo_attn_fwd.restype = I
    lib.mimo_attn_fwd.argtypes = [P, P, P, P, P, ctypes.POINTER(Dims), I, I, D, I, F, P, P, P]
    lib.mimo_attn_host_workspace_size.restype = ctypes.c_size_t
    lib.mimo_attn_host_workspace_size.argtypes = [ctypes.POINTER(Dims), I]
    lib.mimo_attn_fwd_host.restype = I
    lib.mimo_attn_fwd_host.argtypes = [P, P, P, P, P, ctypes.POINTER(Dims), I, I, D, I, F, P, P, P,
                                       ctypes.c_size_t, P]
    lib.mimo_attn_check.restype = I
    lib.mimo_attn_check.argtypes = [P]
    lib.mimo_attn_selftest_wait_timeout.restype = I
    lib.mimo_attn_selftest_wait_timeout.argtypes = [ctypes.c_uint64, P]
    lib.mimo_attn_status_string.restype = ctypes.c_char_p
    lib.mimo_attn_status_string.argtypes = [I]
    lib.mimo_attn_fwd_noalloc.restype = I
    lib.mimo_attn_fwd_noalloc.argtypes = [P, P, P, P, P, ctypes.POINTER(Dims), I, I, D, I, F, P, P, P]
    lib.mimo_attn_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.mimo_attn_noalloc_scratch_bytes.argtypes = []
    lib.mimo_attn_profile_start.restype = I
    lib.mimo_attn_profile_start.argtypes = []
    lib.mimo_attn_profile_set_stride.restype = I
    lib.mimo_attn_profile_set_stride.argtypes = [I]
    lib.mimo_attn_profile_stop.restype = I
    lib.mimo_attn_profile_stop.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]
    lib.mimo_attn_set_kernel.restype = I
    lib.mimo_attn_set_kernel.argtypes = [I]
    lib.mimo_attn_decode.restype = I
    lib.mimo_attn_decode.argtypes = [P, P, P, P, P, P, P, ctypes.POINTER(DecodeDims), I, I, D, I, F, P, P, P]
    lib.mimo_attn_bwd.restype = I
    lib.mimo_attn_bwd.argtypes = [P, P, P, P, P, ctypes.POINTER(Dims), I, I, D, I, F, P, P, P, P, P, P, P, P, P]
    L = ctypes.c_int64
    lib.mimo_fp8_dequant_blockwise.restype = I
    lib.mimo_fp8_dequant_blockwise.argtypes = [P, P, L, L, I, I, P, P]
    lib.mimo_qkv_split.restype = I
    lib.mimo_qkv_split.argtypes = [P, L, I, I, P, P, P, P]
    lib.mimo_attn_set_bwd_kernel.restype = I
    lib.mimo_attn_set_bwd_kernel.argtypes = [I]
    lib.mimo_linear_proj.restype = I
    lib.mimo_linear_proj.argtypes = [P, P, L, L, L, P, P]
    lib.mimo_moe_route.restype = I
    lib.mimo_moe_route.argtypes = [P, P, L, I, I, I, P, P, P]
    lib.mimo_attn_set_decode_kernel.restype = I
    lib.mimo_attn_set_decode_kernel.argtypes = [I]
    lib.mimo_attn_version.restype = I
    lib.mimo_attn_version.argtypes = []
    return lib


LIB = _load()


def status_string(status: int) -> str:
    return LIB.mimo_attn_status_string(int(status)).decode()


def version() -> tuple[int, int]:
    v = LIB.mimo_attn_version()
    return v >> 16, v & 0xFFFF


def set_kernel(choice: int) -> None:
    """Select the kernel mimo_attn_fwd launches (KERNEL_AUTO / _SIMPLE / _PIPELINED / _WINDOW / _WINDOW_PACKED)."""
    st = LIB.mimo_attn_set_kernel(int(choice))
    if st != OK:
        raise MimoAttnError(st, "mimo_attn_set_kernel")


def set_decode_kernel(choice: int) -> None:
    """Select the kernel mimo_attn_decode launches (DECODE_AUTO / _CUDA_CORES / _TENSOR)."""
    st = LIB.mimo_attn_set_decode_kernel(int(choice))
    if st != OK:
        raise MimoAttnError(st, "mimo_attn_set_decode_kernel")


def bwd(q, k, v, sink, cu_seqlens, max_seqlen, layer_kind, window, rope_base, out, lse, dout, dlse=None,
        rope_dims=64, v_scale=0.707, stream=None):
    """Gradients of the forward: q/k/v/out/dout bf16 CUDA tensors, lse / dlse fp32 [Hq, T] (dlse may be
    None).  Returns (dq fp32 [T, Hq, 192], dk fp32 [T, Hkv, 192], dv fp32 [T, Hkv, 128], dsink fp32 [Hq] or
    None)."""
    import torch
    T, hq, dqk = q.shape
    hkv, dv_ = v.shape[1], v.shape[2]
    dq = torch.empty((T, hq, dqk), dtype=torch.float32, device=q.device)
    dk = torch.empty((T, hkv, dqk), dtype=torch.float32, device=q.device)
    dv = torch.empty((T, hkv, dv_), dtype=torch.float32, device=q.device)
    dsink = None if sink is None else torch.empty((hq,), dtype=torch.float32, device=q.device)
    dims = make_dims(cu_seqlens.numel() - 1, T, max_seqlen, hq, hkv)
    ptr = lambda t: None if t is None else t.data_ptr()
    st = LIB.mimo_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), ptr(sink), cu_seqlens.data_ptr(),
                           ctypes.byref(dims), int(layer_kind), int(window), float(rope_base), int(rope_dims),
                           float(v_scale), out.data_ptr(), lse.data_ptr(), dout.data_ptr(), ptr(dlse),
                           dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ptr(dsink), _stream_handle(stream))
    if st != OK:
        raise MimoAttnError(st, "mimo_attn_bwd")
    return dq, dk, dv, dsink


def fp8_dequant_blockwise(codes, scale_inv, block=(128, 128), out=None, stream=None):
    """uint8 E4M3 codes [rows, cols] and fp32 scale_inv [ceil(rows/b0), ceil(cols/b1)] (CUDA) -> bf16."""
    import torch
    rows, cols = codes.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.bfloat16, device=codes.device)
    st = LIB.mimo_fp8_dequant_blockwise(codes.data_ptr(), scale_inv.data_ptr(), rows, cols, int(block[0]),
                                        int(block[1]), out.data_ptr(), _stream_handle(stream))
    if st != OK:
        raise MimoAttnError(st, "mimo_fp8_dequant_blockwise")
    return out


def qkv_split(fused, num_q_heads, num_kv_heads, stream=None):
    """bf16 fused [T, Hkv * (Hq/Hkv*192 + 320)] (CUDA) -> q [T, Hq, 192], k [T, Hkv, 192], v [T, Hkv, 128]."""
    import torch
    T = fused.shape[0]
    q = torch.empty((T, num_q_heads, 192), dtype=torch.bfloat16, device=fused.device)
    k = torch.empty((T, num_kv_heads, 192), dtype=torch.bfloat16, device=fused.device)
    v = torch.empty((T, num_kv_heads, 128), dtype=torch.bfloat16, device=fused.device)
    st = LIB.mimo_qkv_split(fused.data_ptr(), T, int(num_q_heads), int(num_kv_heads), q.data_ptr(), k.data_ptr(),
                            v.data_ptr(), _stream_handle(stream))
    if st != OK:
        raise MimoAttnError(st, "mimo_qkv_split")
    return q, k, v


BWD_AUTO, BWD_CUDA_CORES, BWD_TENSOR = 0, 1, 2


def set_bwd_kernel(choice: int) -> None:
    st = LIB.mimo_attn_set_bwd_kernel(int(choice))
    if st != OK:
        raise MimoAttnError(st, "mimo_attn_set_bwd_kernel")


def linear_proj(x, w, out=None, stream=None):
    """Output projection y = x . w^T: bf16 x [T, K] or the attention output [T, Hq, 128] (CUDA), bf16 w
    [N, K] (a Linear weight) -> bf16 y [T, N] (cuBLAS, FP32 accumulation)."""
    import torch
    T = x.shape[0]
    feats = 1
    for d in x.shape[1:]:
        feats *= int(d)
    x2 = x.reshape(T, feats)  # explicit: reshape(T, -1) is ambiguous for zero tokens
    N, K = w.shape
    if x2.shape[1] != K:
        raise ValueError(f"x has {x2.shape[1]} features per token, w expects {K}")
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=x.device)
    st = LIB.mimo_linear_proj(x2.data_ptr(), w.data_ptr(), T, K, N, out.data_ptr(), _stream_handle(stream))
    if st != OK:
        raise MimoAttnError(st, "mimo_linear_proj")
    return out


def moe_route(logits, bias, top_k=8, normalize=True, stream=None):
    """fp32 logits [T, E] and bias [E] (CUDA) -> ids int32 [T, top_k], weights fp32 [T, top_k]."""
    import torch
    T, E = logits.shape
    ids = torch.empty((T, top_k), dtype=torch.int32, device=logits.device)
    w = torch.empty((T, top_k), dtype=torch.float32, device=logits.device)
    st = LIB.mimo_moe_route(logits.data_ptr(), bias.data_ptr(), T, int(E), int(top_k), int(bool(normalize)),
                            ids.data_ptr(), w.data_ptr(), _stream_handle(stream))
    if st != OK:
        raise MimoAttnError(st, "mimo_moe_route")
    return ids, w


def profile_start() -> None:
    """Record the attention kernel's duration on every following forward (see profile_stop)."""
    LIB.mimo_attn_profile_start()


def profile_set_stride(stride: int) -> None:
    """Record only every stride-th attention-kernel launch while profiling (1: every launch)."""
    st = LIB.mimo_attn_profile_set_stride(stride)
    if st != OK:
        raise MimoAttnError(st, "profile_set_stride")


def profile_stop() -> tuple[int, float]:
    """Stop recording; returns (attention-kernel launches, their summed milliseconds)."""
    n, ms = ctypes.c_int(0), ctypes.c_double(0.0)
    st = LIB.mimo_attn_profile_stop(ctypes.byref(n), ctypes.byref(ms))
    if st != OK:
        raise MimoAttnError(st, "mimo_attn_profile_stop")
    return n.value, ms.value


def make_dims(num_seqs, total_tokens, max_seqlen, hq, hkv, dqk=192, dv=128) -> Dims:
    return Dims(int(num_seqs), int(total_tokens), int(max_seqlen), int(hq), int(hkv), int(dqk), int(dv))


def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def fwd_raw(q_ptr, k_ptr, v_ptr, sink_ptr, cu_ptr, dims: Dims, layer_kind, window, rope_base, rope_dims, v_scale,
            out_ptr, lse_ptr, stream_handle) -> int:
    """Direct C-ABI call with integer device pointers; returns the status code."""
    return LIB.mimo_attn_fwd(q_ptr, k_ptr, v_ptr, sink_ptr, cu_ptr, ctypes.byref(dims), int(layer_kind),
                             int(window), float(rope_base), int(rope_dims), float(v_scale), out_ptr, lse_ptr,
                             stream_handle)


def fwd(q, k, v, sink, cu_seqlens, max_seqlen, layer_kind, window, rope_base, rope_dims=64, v_scale=0.707,
        out=None, lse=None, stream=None):
    """Attention forward on CUDA tensors (bf16 q/k/v in THD layout, int32 cu_seqlens,
    fp32 sink or None).  Returns (out bf16 [T, Hq, 128], lse fp32 [Hq, T])."""
    import torch
    T, hq, dqk = q.shape
    hkv, dv = k.shape[1], v.shape[2]
    for t in (q, k, v):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError("q/k/v must be contiguous bf16 CUDA tensors")
    if out is None:
        out = torch.empty((T, hq, dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((hq, T), dtype=torch.float32, device=q.device)
    dims = make_dims(cu_seqlens.numel() - 1, T, max_seqlen, hq, hkv, dqk, dv)
    st = fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), sink.data_ptr() if sink is not None else None,
                 cu_seqlens.data_ptr(), dims, layer_kind, window, rope_base, rope_dims, v_scale, out.data_ptr(),
                 lse.data_ptr(), _stream_handle(stream))
    if st != OK:
        raise MimoAttnError(st, "mimo_attn_fwd")
    return out, lse


def fwd_noalloc(q, k, v, sink, cu_seqlens, max_seqlen, layer_kind, window, rope_base, out, lse, rope_dims=64,
                v_scale=0.707, stream=None):
    """Same as fwd() through mimo_attn_fwd_noalloc: for callers that cannot allocate
    device memory during the call (the caller passes out and lse; the library's
    scratch is a fixed array of noalloc_scratch_bytes())."""
    dims = make_dims(cu_seqlens.numel() - 1, q.shape[0], max_seqlen, q.shape[1], k.shape[1], q.shape[2], v.shape[2])
    st = LIB.mimo_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                   sink.data_ptr() if sink is not None else None, cu_seqlens.data_ptr(),
                                   ctypes.byref(dims), int(layer_kind), int(window), float(rope_base),
                                   int(rope_dims), float(v_scale), out.data_ptr(), lse.data_ptr(),
                                   _stream_handle(stream))
    if st != OK:
        raise MimoAttnError(st, "mimo_attn_fwd_noalloc")
    return out, lse


def noalloc_scratch_bytes() -> int:
    return LIB.mimo_attn_noalloc_scratch_bytes()


def host_workspace_size(dims: Dims, has_sink: bool) -> int:
    return LIB.mimo_attn_host_workspace_size(ctypes.byref(dims), int(bool(has_sink)))


def fwd_host(q_host, k_host, v_host, sink_host, cu_host, dims: Dims, layer_kind, window, rope_base, rope_dims,
             v_scale, out_host, lse_host, workspace, stream=None):
    """End-to-end call from (pinned) host tensors through a caller-provided device workspace."""
    st = LIB.mimo_attn_fwd_host(q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(),
                                sink_host.data_ptr() if sink_host is not None else None, cu_host.data_ptr(),
                                ctypes.byref(dims), int(layer_kind), int(window), float(rope_base), int(rope_dims),
                                float(v_scale), out_host.data_ptr(), lse_host.data_ptr(), workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if st != OK:
        raise MimoAttnError(st, "mimo_attn_fwd_host")


def check(stream=None) -> int:
    """Sync the stream and return (and clear) the device error status."""
    return LIB.mimo_attn_check(_stream_handle(stream))


def selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    return LIB.mimo_attn_selftest_wait_timeout(int(limit_ns), _stream_handle(stream))


def make_decode_dims(num_seqs, total_q, total_kv, cache_rows, max_q_len, max_kv_len, hq, hkv, dqk=192,
                     dv=128) -> DecodeDims:
    return DecodeDims(int(num_seqs), int(total_q), int(total_kv), int(cache_rows), int(max_q_len),
                      int(max_kv_len), int(hq), int(hkv), int(dqk), int(dv))


def decode_raw(q_ptr, kc_ptr, vc_ptr, idx_ptr, indptr_ptr, cuq_ptr, sink_ptr, dims: DecodeDims, layer_kind, window,
               rope_base, rope_dims, v_scale, out_ptr, lse_ptr, stream_handle) -> int:
    """Direct C-ABI call of mimo_attn_decode with integer device pointers; returns the status code."""
    return LIB.mimo_attn_decode(q_ptr, kc_ptr, vc_ptr, idx_ptr, indptr_ptr, cuq_ptr, sink_ptr, ctypes.byref(dims),
                                int(layer_kind), int(window), float(rope_base), int(rope_dims), float(v_scale),
                                out_ptr, lse_ptr, stream_handle)


def decode(q, k_cache, v_cache, kv_indices, kv_indptr, cu_q, sink, max_q_len, max_kv_len, layer_kind, window,
           rope_base, rope_dims=64, v_scale=0.707, out=None, lse=None, stream=None):
    """New query tokens against a page-size-1 KV cache (CUDA tensors: bf16 q [Tq, Hq, 192], bf16 caches
    [rows, Hkv, 192] / [rows, Hkv, 128], int32 kv_indices / kv_indptr / cu_q, fp32 sink or None).
    Returns (out bf16 [Tq, Hq, 128], lse fp32 [Hq, Tq])."""
    import torch
    Tq, hq, dqk = q.shape
    rows, hkv, dv = v_cache.shape
    for t in (q, k_cache, v_cache):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError("q and the caches must be contiguous bf16 CUDA tensors")
    if out is None:
        out = torch.empty((Tq, hq, dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((hq, Tq), dtype=torch.float32, device=q.device)
    dims = make_decode_dims(cu_q.numel() - 1, Tq, kv_indices.numel(), rows, max_q_len, max_kv_len, hq, hkv, dqk, dv)
    st = decode_raw(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), kv_indices.data_ptr(),
                    kv_indptr.data_ptr(), cu_q.data_ptr(), sink.data_ptr() if sink is not None else None, dims,
                    layer_kind, window, rope_base, rope_dims, v_scale, out.data_ptr(), lse.data_ptr(),
                    _stream_handle(stream))
    if st != OK:
        raise MimoAttnError(st, "mimo_attn_decode")
    return out, lse
