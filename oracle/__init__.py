"""FP64 CPU oracle for the MiMo-V2 attention forward and its gradients -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and it imports nothing
from the product.

The arithmetic lives in ``mimo_attn_oracle.c`` (plain C, FP64, compiled with
gcc, no fast-math); this module only builds it and marshals numpy arrays.

Pins: every function here is pinned by CPU tests against closed forms,
invariants, brute force and library routines (tests/test_oracle_pins.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mimo_attn_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libmimo_attn_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, strict IEEE FP64, no fast-math)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11",
               "-o", tmp, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.oracle_attn_fwd.restype = ctypes.c_int32
    lib.oracle_attn_fwd.argtypes = [P, P, P, P, P, ctypes.c_int32, ctypes.c_int64,
                                    ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                    ctypes.c_int32, ctypes.c_double, ctypes.c_int32, ctypes.c_double,
                                    P, ctypes.c_int64, ctypes.c_int32, P, P]
    lib.oracle_attn_fwd_f64.restype = ctypes.c_int32
    lib.oracle_attn_fwd_f64.argtypes = lib.oracle_attn_fwd.argtypes
    lib.oracle_attn_bwd.restype = ctypes.c_int32
    lib.oracle_attn_bwd.argtypes = [P, P, P, ctypes.c_int32, P, P, ctypes.c_int32, ctypes.c_int64,
                                    ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                    ctypes.c_int32, ctypes.c_double, ctypes.c_int32, ctypes.c_double,
                                    P, P, P, P, P, P]
    lib.oracle_rope.restype = None
    lib.oracle_rope.argtypes = [P, ctypes.c_int64, ctypes.c_double, ctypes.c_int32, ctypes.c_int32, P]
    lib.oracle_rope_transpose.restype = None
    lib.oracle_rope_transpose.argtypes = lib.oracle_rope.argtypes
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1))


def attn_fwd(q, k, v, sink, cu_seqlens, window, rope_base, rope_dims=64, v_scale=0.707, rows=None,
             threads=None, lib=None):
    """Run the oracle.

    q/k/v: uint16 BF16 bit arrays [T, Hq, Dqk] / [T, Hkv, Dqk] / [T, Hkv, Dv].
    sink: float32 [Hq] or None.  cu_seqlens: int32 [B+1].  window < 0: global layer.
    rows: optional int64 token indices; default all tokens.
    Returns (out float64 [n_rows, Hq, Dv], lse float64 [Hq, n_rows]).
    """
    lib = lib or _load()
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T, hq, dqk = q.shape
    hkv, dv = k.shape[1], v.shape[2]
    assert k.shape == (T, hkv, dqk) and v.shape == (T, hkv, dv)
    sk = None if sink is None else np.ascontiguousarray(sink, dtype=np.float32)
    if rows is None:
        rr, n = None, T
    else:
        rr = np.ascontiguousarray(rows, dtype=np.int64)
        n = len(rr)
    out = np.zeros((n, hq, dv), dtype=np.float64)
    lse = np.zeros((hq, n), dtype=np.float64)
    st = lib.oracle_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(sk), _ptr(cu), len(cu) - 1, T, hq, hkv, dqk, dv, int(window),
        float(rope_base), int(rope_dims), float(v_scale), _ptr(rr), n, int(threads or default_threads()),
        _ptr(out), _ptr(lse))
    if st != 0:
        raise ValueError(f"oracle_attn_fwd failed with status {st}")
    return out, lse


def _inputs(q, k, v, sink, cu_seqlens):
    """Marshal q/k/v as BF16 bit arrays (uint16) or FP64 arrays; returns (..., f64 flag)."""
    f64 = np.asarray(q).dtype == np.float64
    dt = np.float64 if f64 else np.uint16
    q = np.ascontiguousarray(q, dtype=dt)
    k = np.ascontiguousarray(k, dtype=dt)
    v = np.ascontiguousarray(v, dtype=dt)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T, hq, dqk = q.shape
    hkv, dv = k.shape[1], v.shape[2]
    assert k.shape == (T, hkv, dqk) and v.shape == (T, hkv, dv)
    sk = None if sink is None else np.ascontiguousarray(sink, dtype=np.float32)
    return q, k, v, sk, cu, f64


def attn_fwd_f64(q, k, v, sink, cu_seqlens, window, rope_base, rope_dims=64, v_scale=0.707, threads=None, lib=None):
    """The forward oracle on FP64 q/k/v (same layouts); returns (out, lse) for every token."""
    lib = lib or _load()
    q, k, v, sk, cu, _ = _inputs(np.asarray(q, dtype=np.float64), k, v, sink, cu_seqlens)
    T, hq, dqk = q.shape
    hkv, dv = k.shape[1], v.shape[2]
    out = np.zeros((T, hq, dv), dtype=np.float64)
    lse = np.zeros((hq, T), dtype=np.float64)
    st = lib.oracle_attn_fwd_f64(
        _ptr(q), _ptr(k), _ptr(v), _ptr(sk), _ptr(cu), len(cu) - 1, T, hq, hkv, dqk, dv, int(window),
        float(rope_base), int(rope_dims), float(v_scale), None, T, int(threads or default_threads()),
        _ptr(out), _ptr(lse))
    if st != 0:
        raise ValueError(f"oracle_attn_fwd_f64 failed with status {st}")
    return out, lse


def attn_bwd(q, k, v, sink, cu_seqlens, window, rope_base, rope_dims, v_scale, dout, dlse=None, lib=None):
    """Gradients of L(q, k, v, sink) given dL/dout (FP64 [T, Hq, Dv]) and dL/dlse (FP64 [Hq, T] or None).

    q/k/v are BF16 bit arrays (uint16) or FP64 arrays.  Returns (dq, dk, dv, dsink) in FP64;
    dsink is None without a sink."""
    lib = lib or _load()
    q, k, v, sk, cu, f64 = _inputs(q, k, v, sink, cu_seqlens)
    T, hq, dqk = q.shape
    hkv, dv = k.shape[1], v.shape[2]
    go = np.ascontiguousarray(dout, dtype=np.float64)
    assert go.shape == (T, hq, dv)
    gl = None if dlse is None else np.ascontiguousarray(dlse, dtype=np.float64)
    dq = np.zeros((T, hq, dqk), dtype=np.float64)
    dk = np.zeros((T, hkv, dqk), dtype=np.float64)
    dvv = np.zeros((T, hkv, dv), dtype=np.float64)
    ds = None if sk is None else np.zeros(hq, dtype=np.float64)
    st = lib.oracle_attn_bwd(
        _ptr(q), _ptr(k), _ptr(v), int(f64), _ptr(sk), _ptr(cu), len(cu) - 1, T, hq, hkv, dqk, dv, int(window),
        float(rope_base), int(rope_dims), float(v_scale), _ptr(go), _ptr(gl), _ptr(dq), _ptr(dk), _ptr(dvv), _ptr(ds))
    if st != 0:
        raise ValueError(f"oracle_attn_bwd failed with status {st}")
    return dq, dk, dvv, ds


def rope_transpose(x, pos, base, rope_dims=64, lib=None):
    """Oracle transpose of RoPE (rotation by the negative angle) of one vector."""
    lib = lib or _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    lib.oracle_rope_transpose(_ptr(x), int(pos), float(base), int(rope_dims), x.shape[0], _ptr(y))
    return y


def rope(x, pos, base, rope_dims=64, lib=None):
    """Oracle RoPE of one vector x (float64 [D]) at position pos."""
    lib = lib or _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    lib.oracle_rope(_ptr(x), int(pos), float(base), int(rope_dims), x.shape[0], _ptr(y))
    return y


class Variant:
    """The oracle compiled from another C source (used by the mutation tests to
    confirm that the pins reject a deliberately broken copy)."""

    def __init__(self, c_source: str, workdir: str):
        src = os.path.join(workdir, "variant.c")
        so = os.path.join(workdir, "libvariant.so")
        with open(src, "w") as f:
            f.write(c_source)
        subprocess.run(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11",
                        "-o", so, src, "-lm", "-lpthread"], check=True)
        self.lib = _bind(so)

    def attn_fwd(self, *a, **kw):
        kw["lib"] = self.lib
        return attn_fwd(*a, **kw)

    def rope(self, *a, **kw):
        kw["lib"] = self.lib
        return rope(*a, **kw)

    def attn_fwd_f64(self, *a, **kw):
        kw["lib"] = self.lib
        return attn_fwd_f64(*a, **kw)

    def attn_bwd(self, *a, **kw):
        kw["lib"] = self.lib
        return attn_bwd(*a, **kw)


def source() -> str:
    with open(_SRC) as f:
        return f.read()
