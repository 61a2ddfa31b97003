"""GPU parity of the backward (mimo_attn_bwd) against the FP64 oracle backward.

The kernel forms D = dO . out from the forward's stored BF16 out and P_j = exp(s_j - lse) from its
stored FP32 lse, as any backward that reuses the forward's outputs does.  The gradients are linear in
dLSE, and D enters only as (dLSE - D), so a kernel that uses the stored out computes exactly the
gradient of the method with dLSE replaced by dLSE - dO . (out_stored - out).  The tests hand the
oracle that shifted dLSE (out = the oracle's own FP64 forward), which removes the BF16 rounding of out
from the comparison; without it the cancellation of dO . v_j against D (one key per query at
window 0) leaves only that rounding.

Tolerances, rel-L2 per gradient:
- forward statistics from the oracle (out rounded once to BF16, lse to FP32): 1e-4.  What remains is
  FP32 arithmetic: dot products of 192 / 128 terms and sums over the keys at unit round-off 6e-8,
  times a cancellation factor of at most ~30 where dO . v_j and D nearly cancel.
- forward statistics from the GPU forward (the training chain): 2e-3.  The forward's lse carries the
  FP16 rounding of the rotated Q/K dims (score errors of a few 1e-4), and P inherits that relative
  error.
"""
import numpy as np
import pytest
import torch

import oracle
from global_attention_moe_b200 import synth, workloads as W

pytestmark = pytest.mark.gpu

TOL_ORACLE_STATS = 1e-4
TOL_GPU_STATS = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda_core_kernel():
    """This module checks the FP32 CUDA-core backward (the default is the tensor-core one, checked by
    tests/test_gpu_bwd_tc.py with these cases at its own tolerance)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from global_attention_moe_b200 import mimo_attn as M
    M.set_bwd_kernel(M.BWD_CUDA_CORES)
    yield
    M.set_bwd_kernel(M.BWD_AUTO)


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


def run(lens, hq, hkv, layer, window, base, has_sink, seed, dlse=True, stats="oracle", tol=None):
    """Runs the backward on one case and compares with the oracle (tol: rel-L2 per gradient; by
    default this module's tolerance for the kind of forward statistics)."""
    from global_attention_moe_b200 import mimo_attn as M
    rng = np.random.default_rng(seed)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = synth.f32_to_bf16_bits(rng.standard_normal((T, hq, 192)).astype(np.float32))
    k = synth.f32_to_bf16_bits(rng.standard_normal((T, hkv, 192)).astype(np.float32))
    v = synth.f32_to_bf16_bits(rng.standard_normal((T, hkv, 128)).astype(np.float32))
    sink = rng.standard_normal(hq).astype(np.float32) if has_sink else None
    go = synth.f32_to_bf16_bits(rng.standard_normal((T, hq, 128)).astype(np.float32))
    gl = (rng.standard_normal((hq, T)) * 0.3).astype(np.float32) if dlse else None
    w = window if layer == W.LAYER_SWA else -1
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    sk = None if sink is None else torch.from_numpy(sink).cuda()
    cut = torch.from_numpy(cu).cuda()
    out_x, lse_x = oracle.attn_fwd(q, k, v, sink, cu, w, base)
    if stats == "oracle":
        out_b = f64_to_bf16_bits(out_x)
        out, lse = dev(out_b), torch.from_numpy(lse_x.astype(np.float32)).cuda()
        tol = TOL_ORACLE_STATS if tol is None else tol
    else:
        out, lse = M.fwd(dev(q), dev(k), dev(v), sk, cut, max(lens), layer, window, base)
        out_b = out.view(torch.int16).cpu().numpy().view(np.uint16)
        tol = TOL_GPU_STATS if tol is None else tol
    dq, dk, dv, ds = M.bwd(dev(q), dev(k), dev(v), sk, cut, max(lens), layer, window, base, out, lse, dev(go),
                           None if gl is None else torch.from_numpy(gl).cuda())
    assert M.check() == M.OK
    go64 = synth.bf16_bits_to_f32(go).astype(np.float64)
    shift = np.einsum("thd,thd->ht", go64, synth.bf16_bits_to_f32(out_b).astype(np.float64) - out_x)
    gl_eff = (0.0 if gl is None else gl.astype(np.float64)) - shift
    ref = oracle.attn_bwd(q, k, v, sink, cu, w, base, 64, 0.707, go64, gl_eff)
    for name, a, r in zip(("dq", "dk", "dv", "dsink"), (dq, dk, dv, ds), ref):
        if r is None:
            assert a is None
            continue
        a = a.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(a)), name
        rel = np.linalg.norm(a - r) / np.linalg.norm(r)
        assert rel <= tol, f"{name}: rel-L2 {rel:.2e}"


@pytest.mark.parametrize("hq,hkv", [(8, 2), (4, 1), (4, 4)])
def test_swa_sink(hq, hkv):
    run([300, 129, 17, 1], hq, hkv, W.LAYER_SWA, 128, 1e4, True, seed=41)


@pytest.mark.parametrize("window", [0, 1, 31, 127])
def test_swa_windows(window):
    run([200, 70], 4, 2, W.LAYER_SWA, window, 1e4, False, seed=42)


def test_global_causal():
    run([333, 64, 5], 8, 2, W.LAYER_GLOBAL, -1, 1e7, False, seed=43)


def test_without_dlse():
    run([150], 4, 1, W.LAYER_SWA, 128, 1e4, True, seed=44, dlse=False)


@pytest.mark.parametrize("layer,window,base,sink", [(W.LAYER_SWA, 128, 1e4, True), (W.LAYER_GLOBAL, -1, 1e7, False)])
def test_training_chain(layer, window, base, sink):
    """The GPU forward's own out and lse feed the backward, as training does."""
    run([260, 77], 8, 2, layer, window, base, sink, seed=45, stats="gpu")


def test_empty_batch():
    from global_attention_moe_b200 import mimo_attn as M
    z = lambda *s: torch.zeros(s, dtype=torch.bfloat16).cuda()
    cut = torch.zeros(2, dtype=torch.int32).cuda()
    sk = torch.ones(4).cuda()
    lse = torch.zeros((4, 0)).cuda()
    dq, dk, dv, ds = M.bwd(z(0, 4, 192), z(0, 2, 192), z(0, 2, 128), sk, cut, 0, W.LAYER_SWA, 128, 1e4,
                           z(0, 4, 128), lse, z(0, 4, 128))
    assert dq.shape == (0, 4, 192) and dk.shape == (0, 2, 192) and dv.shape == (0, 2, 128)
    assert torch.all(ds.cpu() == 0)


def test_full_size_swa_layer():
    """The sliding-window layer at its full size (4096 tokens, 64 query / 8 KV heads, window 128, sink)
    against the oracle backward on every element of dq, dk, dv and dsink (the oracle's FP64 backward
    runs single-threaded here, about a minute)."""
    run([4096], 64, 8, W.LAYER_SWA, 128, 1e4, True, seed=47)
