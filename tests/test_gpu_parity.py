"""GPU parity: the CUDA path through the C-ABI against the FP64 oracle on the
same seeded inputs, at sizes the oracle finishes in seconds (element by
element) and at the full workload sizes (sampled rows), plus edge cases."""
import numpy as np
import pytest
import torch

from global_attention_moe_b200 import workloads as W
from gpu_helpers import (assert_within, errors, out_to_f64, run_gpu, run_oracle, sample_rows, to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from global_attention_moe_b200 import mimo_attn
    assert mimo_attn.check() == mimo_attn.OK


KERNELS = {"auto": 0, "simple": 1, "pipelined": 2, "window": 3, "packed": 4}
_current = {"kernel": "auto"}


@pytest.fixture(params=["auto", "simple", "pipelined", "window"])
def kernel(request):
    """Run a test with the default kernel choice (the packed window kernel for
    short sliding windows at 4 or 8 query heads per KV head, the pipelined one
    for the global layer), with the serialised cross-check kernel, and with the
    pipelined and the two-head window kernels forced."""
    from global_attention_moe_b200 import mimo_attn
    mimo_attn.set_kernel(KERNELS[request.param])
    _current["kernel"] = request.param
    yield request.param
    mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)
    _current["kernel"] = "auto"


def kernel_supports(name: str, w) -> bool:
    """Shapes a forced kernel choice accepts (the C ABI returns UNSUPPORTED otherwise)."""
    even = (w.num_q_heads // w.num_kv_heads) % 2 == 0
    if name == "pipelined":
        return even
    if name == "window":
        return even and w.layer_kind == W.LAYER_SWA and 0 <= w.window <= 128
    if name == "packed":
        return w.num_q_heads // w.num_kv_heads in (4, 8) and w.layer_kind == W.LAYER_SWA and 0 <= w.window <= 128
    return True


def full_parity(w):
    if not kernel_supports(_current["kernel"], w):
        pytest.skip(f"{_current['kernel']} kernel does not take this shape")
    x = W.make_inputs(w)
    out, lse = run_gpu(w, x)
    ref_out, ref_lse = run_oracle(w, x)
    err = errors(out_to_f64(out), lse.cpu().numpy().astype(np.float64), ref_out, ref_lse)
    assert_within(err, w.name)
    return err


def test_tiny_swa_sink_full(kernel):
    full_parity(W.tiny_swa())


@pytest.mark.parametrize("lengths", [[1], [127], [128], [129], [130], [255], [256], [257],
                                     [1, 127, 128, 129, 130, 255, 256, 257], [0, 300, 0, 5]])
def test_ragged_lengths_swa(lengths, kernel):
    full_parity(W.custom("ragged", W.LAYER_SWA, lengths, 4, 1, 128, 1e4, True, seed=1))


@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 1), (16, 1), (64, 8)])
def test_gqa_ratios(hq, hkv, kernel):
    full_parity(W.custom("gqa", W.LAYER_SWA, [200, 333], hq, hkv, 128, 1e4, True, seed=2))


@pytest.mark.parametrize("window", [0, 1, 5, 127, 128, 129, 200, 300])
def test_windows(window, kernel):
    full_parity(W.custom("win", W.LAYER_SWA, [700, 61], 4, 2, window, 1e4, False, seed=3))


def test_sink_extremes(kernel):
    w = W.custom("sink", W.LAYER_SWA, [400], 8, 2, 128, 1e4, True, seed=4)
    x = W.make_inputs(w)
    x.sink = np.array([8, -8, 8, -8, 0, 3, -3, 20], dtype=np.float32)
    out, lse = run_gpu(w, x)
    ro, rl = run_oracle(w, x)
    assert_within(errors(out_to_f64(out), lse.cpu().numpy().astype(np.float64), ro, rl), "sink extremes")


@pytest.mark.parametrize("lengths", [[300], [1, 129, 640], [1024]])
def test_global_small(lengths, kernel):
    full_parity(W.custom("global", W.LAYER_GLOBAL, lengths, 8, 2, -1, 1e7, False, seed=5))


@pytest.mark.parametrize("name", ["swa4096", "swa_varlen", "global", "swa_long"])
def test_full_size_sampled(name):
    w = W.WORKLOADS[name]()
    x = W.make_inputs(w)
    out, lse = run_gpu(w, x)
    rows = sample_rows(w)
    ref_out, ref_lse = run_oracle(w, x, rows=rows)
    rows_t = torch.from_numpy(rows).to(out.device)
    g_out = out_to_f64(out.index_select(0, rows_t))
    g_lse = lse.index_select(1, rows_t).cpu().numpy().astype(np.float64)
    assert_within(errors(g_out, g_lse, ref_out, ref_lse), name)
    # properties that hold at any size: finite everywhere, lse >= sink, |out| bounded by v_scale*max|v|
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    if x.sink is not None:
        assert (lse >= torch.from_numpy(x.sink).to(lse.device)[:, None] - 1e-4).all()
    vmax = float(np.abs(W.synth.bf16_bits_to_f32(x.v)).max())
    assert float(out.float().abs().max()) <= w.v_scale * vmax * 1.01


def test_packed_equals_separate(kernel):
    w = W.custom("pack", W.LAYER_SWA, [130, 1, 257, 64], 8, 2, 128, 1e4, True, seed=6)
    x = W.make_inputs(w)
    out, lse = run_gpu(w, x)
    for b, L in enumerate(w.lengths):
        s = int(x.cu_seqlens[b])
        wb = W.custom("one", W.LAYER_SWA, [L], 8, 2, 128, 1e4, True, seed=6)
        xb = W.Inputs(x.q[s:s + L], x.k[s:s + L], x.v[s:s + L], x.sink, np.array([0, L], dtype=np.int32))
        ob, lb = run_gpu(wb, xb)
        assert torch.equal(ob, out[s:s + L]) and torch.equal(lb, lse[:, s:s + L])


def test_every_row_written_and_no_overrun(kernel):
    """Outputs live inside larger buffers pre-filled with NaN: every in-range
    element must be overwritten and every guard element left untouched."""
    w = W.custom("guard", W.LAYER_SWA, [1, 200, 129], 4, 1, 128, 1e4, True, seed=7)
    x = W.make_inputs(w)
    T, G = w.total_tokens, 4096
    dev = to_device(x)
    ob = torch.full((T * 4 * 128 + 2 * G,), float("nan"), dtype=torch.bfloat16, device="cuda")
    lb = torch.full((4 * T + 2 * G,), float("nan"), dtype=torch.float32, device="cuda")
    out = ob[G:G + T * 4 * 128].view(T, 4, 128)
    lse = lb[G:G + 4 * T].view(4, T)
    run_gpu(w, x, dev_inputs=dev, out=out, lse=lse)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    assert torch.isnan(ob[:G].float()).all() and torch.isnan(ob[-G:].float()).all()
    assert torch.isnan(lb[:G]).all() and torch.isnan(lb[-G:]).all()


def test_host_entry_matches_device_entry():
    from global_attention_moe_b200 import mimo_attn
    w = W.custom("host", W.LAYER_SWA, [300, 77], 8, 2, 128, 1e4, True, seed=8)
    x = W.make_inputs(w)
    out, lse = run_gpu(w, x)
    dims = mimo_attn.make_dims(w.num_seqs, w.total_tokens, w.max_seqlen, 8, 2)
    pin = lambda a: torch.from_numpy(a).pin_memory()
    qh, kh, vh = (pin(a.view(np.int16)) for a in (x.q, x.k, x.v))
    sh, ch = pin(x.sink), pin(x.cu_seqlens)
    oh = torch.empty(w.total_tokens, 8, 128, dtype=torch.int16).pin_memory()
    lh = torch.empty(8, w.total_tokens, dtype=torch.float32).pin_memory()
    ws = torch.empty(mimo_attn.host_workspace_size(dims, True), dtype=torch.uint8, device="cuda")
    mimo_attn.fwd_host(qh, kh, vh, sh, ch, dims, w.layer_kind, w.window, w.rope_base, 64, w.v_scale, oh, lh, ws)
    assert torch.equal(oh.view(torch.bfloat16), out.cpu()) and torch.equal(lh, lse.cpu())


def test_bounded_wait_reports_timeout_and_context_survives():
    from global_attention_moe_b200 import mimo_attn
    assert mimo_attn.selftest_wait_timeout(2_000_000) == mimo_attn.ERR_TIMEOUT
    assert mimo_attn.check() == mimo_attn.OK
    full_parity(W.tiny_swa())


def test_range_error_recorded():
    from global_attention_moe_b200 import mimo_attn
    w = W.custom("range", W.LAYER_SWA, [64], 4, 1, 128, 1e4, False, seed=9)
    x = W.make_inputs(w)
    q = x.q.copy()
    q[5, 0, 3] = W.synth.f32_to_bf16_bits(np.array([60000.0], dtype=np.float32))[0]
    q[5, 0, 35] = W.synth.f32_to_bf16_bits(np.array([60000.0], dtype=np.float32))[0]
    x.q = q
    dq, dk, dv, ds, dcu = to_device(x)
    mimo_attn.fwd(dq, dk, dv, ds, dcu, 64, 0, 128, 1e4)
    assert mimo_attn.check() == mimo_attn.ERR_RANGE


def test_bad_cu_seqlens_detected_without_overrun():
    from global_attention_moe_b200 import mimo_attn
    w = W.custom("badcu", W.LAYER_SWA, [100, 100], 4, 1, 128, 1e4, False, seed=10)
    x = W.make_inputs(w)
    dq, dk, dv, ds, _ = to_device(x)
    cu = torch.tensor([0, 150, 260], dtype=torch.int32, device="cuda")  # ends past T = 200
    G = 4096
    ob = torch.full((200 * 4 * 128 + 2 * G,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = ob[G:G + 200 * 4 * 128].view(200, 4, 128)
    mimo_attn.fwd(dq, dk, dv, ds, cu, 200, 0, 128, 1e4, out=out)
    assert mimo_attn.check() == mimo_attn.ERR_BAD_SEQLENS
    assert torch.isnan(ob[:G].float()).all() and torch.isnan(ob[-G:].float()).all()


def test_kernels_agree_closely():
    """The pipelined and the serialised kernel take the same rounding steps; on the
    same inputs their outputs agree to a few BF16 ulps (summation order differs)."""
    from global_attention_moe_b200 import mimo_attn
    w = W.custom("agree", W.LAYER_GLOBAL, [700, 129], 8, 2, -1, 1e7, False, seed=11)
    x = W.make_inputs(w)
    dev = to_device(x)
    mimo_attn.set_kernel(mimo_attn.KERNEL_SIMPLE)
    try:
        o1, l1 = run_gpu(w, x, dev_inputs=dev)
    finally:
        mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)
    o2, l2 = run_gpu(w, x, dev_inputs=dev)
    assert float((o1.float() - o2.float()).abs().max()) < 1e-2
    assert float((l1 - l2).abs().max()) < 2e-4


def test_window_and_pipelined_kernels_agree():
    """The window kernel (both key tiles scored, one softmax pass) and the
    pipelined kernel (online softmax over key tiles) both meet the oracle
    tolerances on the same inputs, and their mutual difference stays within
    the same bounds.  (P is rounded to BF16 at different scales -- the row max
    versus a lazily updated running max -- so they are not bit-identical.)"""
    from global_attention_moe_b200 import mimo_attn
    w = W.custom("agree_swa", W.LAYER_SWA, [700, 129, 1, 300], 8, 2, 128, 1e4, True, seed=12)
    x = W.make_inputs(w)
    dev = to_device(x)
    ref_out, ref_lse = run_oracle(w, x)
    res = {}
    for name in ("pipelined", "window"):
        mimo_attn.set_kernel(KERNELS[name])
        try:
            o, l = run_gpu(w, x, dev_inputs=dev)
        finally:
            mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)
        res[name] = (out_to_f64(o), l.cpu().numpy().astype(np.float64))
        assert_within(errors(*res[name], ref_out, ref_lse), name)
    mutual = errors(*res["window"], *res["pipelined"])
    print("window vs pipelined:", mutual)
    assert_within(mutual, "window vs pipelined")


@pytest.mark.parametrize("layer,window,hq,hkv", [(W.LAYER_GLOBAL, -1, 8, 2), (W.LAYER_SWA, 129, 8, 2),
                                                 (W.LAYER_SWA, 128, 8, 8)])
def test_forced_window_kernel_rejects_other_shapes(layer, window, hq, hkv):
    """Forcing the window kernel on a shape it does not take returns UNSUPPORTED
    before anything is launched."""
    from global_attention_moe_b200 import mimo_attn
    w = W.custom("reject", layer, [300], hq, hkv, window, 1e4 if layer == W.LAYER_SWA else 1e7,
                 layer == W.LAYER_SWA, seed=13)
    x = W.make_inputs(w)
    dev = to_device(x)
    mimo_attn.set_kernel(mimo_attn.KERNEL_WINDOW)
    try:
        with pytest.raises(mimo_attn.MimoAttnError) as e:
            run_gpu(w, x, dev_inputs=dev)
        assert e.value.status == mimo_attn.ERR_UNSUPPORTED
    finally:
        mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)
    assert mimo_attn.check() == mimo_attn.OK


@pytest.mark.parametrize("window", [0, 1, 31, 32, 33, 64, 96, 127, 128])
@pytest.mark.parametrize("lengths", [[1000], [1, 128, 129, 383, 5]])
def test_window_kernel_windows(window, lengths):
    """The window kernel across windows that move the run's chunk boundaries."""
    from global_attention_moe_b200 import mimo_attn
    mimo_attn.set_kernel(mimo_attn.KERNEL_WINDOW)
    try:
        _current["kernel"] = "window"
        full_parity(W.custom("wwin", W.LAYER_SWA, lengths, 4, 2, window, 1e4, window % 2 == 0, seed=14))
    finally:
        _current["kernel"] = "auto"
        mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)


@pytest.mark.parametrize("pair", [("window", "pipelined"), ("packed", "pipelined")], ids=lambda p: "-".join(p))
@pytest.mark.parametrize("name", ["swa4096", "swa_varlen", "swa_long"])
def test_full_size_window_and_pipelined_agree_on_every_row(name, pair):
    """At the full workload sizes, every row of a window kernel's output
    against the pipelined kernel's (independently written paths with
    different schedules, tile shapes, K/V reuse and softmax passes)."""
    from global_attention_moe_b200 import mimo_attn
    w = W.WORKLOADS[name]()
    x = W.make_inputs(w)
    dev = to_device(x)
    res = {}
    for kname in pair:
        mimo_attn.set_kernel(KERNELS[kname])
        try:
            res[kname] = run_gpu(w, x, dev_inputs=dev)
        finally:
            mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)
    (o1, l1), (o2, l2) = res[pair[0]], res[pair[1]]
    a, b = o1.float(), o2.float()
    assert bool(torch.isfinite(a).all()) and bool(torch.isfinite(b).all())
    assert float((a - b).abs().max()) <= 2e-2
    assert float((a - b).norm() / b.norm()) <= 5e-3
    assert float((l1 - l2).abs().max()) <= 1e-3


def test_many_short_sequences_cross_pair_and_sequence_boundaries():
    """Forty sequences of 1..300 tokens with 16 query heads: CTAs get several
    units each, and their blocks cross sequence starts and head-pair changes
    (where a unit may or may not reuse the previous unit's key tile)."""
    rng = np.random.default_rng(15)
    lengths = [int(v) for v in rng.integers(1, 301, size=40)]
    full_parity(W.custom("many", W.LAYER_SWA, lengths, 16, 2, 128, 1e4, True, seed=15))


@pytest.mark.parametrize("which", ["q", "k"])
@pytest.mark.parametrize("value,overflows", [(46080.0, False), (48128.0, True)])
def test_fp16_range_limit_of_rotated_dims(which, value, overflows):
    """A rope pair (x_0, x_32) = (a, -a) at position 1 rotates to a (cos 1 + sin 1) = 1.3818 a on
    dim 0: a = 46080 gives 63673, inside FP16's largest finite value 65504, and a = 48128 gives
    66503, past it.  The first call runs clean, the second records MIMO_ERR_RANGE."""
    from global_attention_moe_b200 import mimo_attn
    w = W.custom("range_limit", W.LAYER_SWA, [64], 4, 1, 128, 1e4, True, seed=17)
    x = W.make_inputs(w)
    a = W.synth.f32_to_bf16_bits(np.array([value, -value], dtype=np.float32))
    t = getattr(x, which).copy()
    t[1, 0, 0], t[1, 0, 32] = a[0], a[1]
    setattr(x, which, t)
    dq, dk, dv, ds, dcu = to_device(x)
    out, lse = mimo_attn.fwd(dq, dk, dv, ds, dcu, 64, 0, 128, 1e4)
    st = mimo_attn.check()
    if overflows:
        assert st == mimo_attn.ERR_RANGE
    else:
        assert st == mimo_attn.OK
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_pool_scratch_returned_after_synchronize():
    """Scratch a call takes from the library's stream-ordered pool (here the pre-rotated K rope
    dims of the global layer's kernel, T * Hkv * 128 bytes = 32 MiB) goes back to the device at
    the next synchronization: free device memory after a synchronized call is what it was before."""
    w = W.custom("pool", W.LAYER_GLOBAL, [8192] * 4, 16, 8, -1, 1e7, False, seed=18)
    x = W.make_inputs(w)
    dev = to_device(x)
    out = torch.empty(w.total_tokens, 16, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(16, w.total_tokens, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        run_gpu(w, x, dev_inputs=dev, out=out, lse=lse)  # synchronizes (mimo_attn_check)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert free0 - free1 < 4 * 2 ** 20, (free0, free1)


@pytest.mark.parametrize("layer,window,hq,hkv", [(W.LAYER_GLOBAL, -1, 8, 2), (W.LAYER_SWA, 129, 8, 2),
                                                 (W.LAYER_SWA, 128, 8, 4), (W.LAYER_SWA, 128, 16, 1),
                                                 (W.LAYER_SWA, 128, 6, 1)])
def test_forced_packed_kernel_rejects_other_shapes(layer, window, hq, hkv):
    """The packed window kernel takes sliding windows of at most 128 keys at 4 or 8 query heads per
    KV head; forced on anything else the call returns UNSUPPORTED before anything is launched."""
    from global_attention_moe_b200 import mimo_attn
    w = W.custom("reject_packed", layer, [300], hq, hkv, window, 1e4 if layer == W.LAYER_SWA else 1e7,
                 layer == W.LAYER_SWA, seed=19)
    x = W.make_inputs(w)
    dev = to_device(x)
    mimo_attn.set_kernel(mimo_attn.KERNEL_WINDOW_PACKED)
    try:
        with pytest.raises(mimo_attn.MimoAttnError) as e:
            run_gpu(w, x, dev_inputs=dev)
        assert e.value.status == mimo_attn.ERR_UNSUPPORTED
    finally:
        mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)
    assert mimo_attn.check() == mimo_attn.OK


@pytest.mark.parametrize("window", [0, 1, 15, 16, 17, 31, 64, 127, 128])
@pytest.mark.parametrize("lengths,hq,hkv", [([1000], 8, 1), ([1, 16, 17, 128, 129, 383, 5], 16, 2),
                                           ([31, 32, 33, 300], 8, 2)])
def test_packed_kernel_windows(window, lengths, hq, hkv):
    """The packed window kernel across windows that move the run across its 16-key ring slots, sequences
    that end inside a tile and on slot edges, at 8 (16 x 8 tiles) and 4 (32 x 4) query heads per KV head."""
    from global_attention_moe_b200 import mimo_attn
    mimo_attn.set_kernel(mimo_attn.KERNEL_WINDOW_PACKED)
    try:
        _current["kernel"] = "packed"
        full_parity(W.custom("pwin", W.LAYER_SWA, lengths, hq, hkv, window, 1e4, window % 2 == 0, seed=20))
    finally:
        _current["kernel"] = "auto"
        mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)


def test_packed_kernel_many_tiles_per_cta():
    """Forty sequences over two KV groups with 16 query heads: every CTA walks many tiles, whose
    windows continue the previous tile's ring or start afresh at sequence and group changes."""
    from global_attention_moe_b200 import mimo_attn
    rng = np.random.default_rng(21)
    lengths = [int(v) for v in rng.integers(1, 700, size=40)]
    mimo_attn.set_kernel(mimo_attn.KERNEL_WINDOW_PACKED)
    try:
        _current["kernel"] = "packed"
        full_parity(W.custom("pmany", W.LAYER_SWA, lengths, 16, 2, 128, 1e4, True, seed=21))
    finally:
        _current["kernel"] = "auto"
        mimo_attn.set_kernel(mimo_attn.KERNEL_AUTO)
