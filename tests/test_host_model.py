"""The whole library built for the CPU, tensor-core kernels included: their unchanged source runs on
the fiber runtime with a device model of the tcgen05 / TMA / mbarrier wrappers
(tests/host_emulation/device_model), and the results are compared with the oracle at the forward's
tolerances.  The model reproduces the errors measured on a B200 for the tensor-core forward kernels
on the small sliding-window config (max-abs 4.4e-3 simple, 7.3e-3 pipelined), i.e. the same
rounding points.  Planted mistakes in the kernels' operand addressing, row tiling and MMA completion
waits are caught (the device model runs an MMA only when its commit's barrier is first waited on)."""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
EMU = os.path.join(HERE, "host_emulation")
sys.path.insert(0, EMU)
import build_library  # noqa: E402
from library_cases import CASES, PACKED_CASES, TIMEOUT_CASES  # noqa: E402


def run_cases(lib, names, sms=None):
    env = dict(os.environ, HEMU_SMS=str(sms)) if sms else None
    r = subprocess.run([sys.executable, os.path.join(EMU, "library_cases.py"), lib, *names], capture_output=True,
                       text=True, timeout=900, env=env)
    return r.returncode, (r.stdout + r.stderr)[-2000:]


@pytest.fixture(scope="module")
def host_library(tmp_path_factory):
    return build_library.build(str(tmp_path_factory.mktemp("library_host")))


def test_library_matches_oracle(host_library):
    rc, log = run_cases(host_library, [c for c in CASES if c not in TIMEOUT_CASES + PACKED_CASES])
    assert rc == 0, log


def test_decode_kernel_with_one_and_two_sms(host_library):
    """The persistent KV-cache kernel on 1 and 2 SMs: every CTA then takes many items in turn, so the
    item boundaries (the previous item's last PV before the next item's first score, Q reloaded once
    the last score has read it) and the lander's per-chunk angle tables turn over many times."""
    for sms in (1, 2):
        rc, log = run_cases(host_library, ["decode_tensor", "decode_tensor_tiles_swa", "decode_tensor_tiles_global"],
                            sms=sms)
        assert rc == 0, log


def test_backward_with_two_sms(host_library):
    """The tensor-core backward on a 2-SM grid: the prep kernel's warps then walk many tokens of a head
    each, and each SM runs many key tiles in turn."""
    rc, log = run_cases(host_library, ["bwd_tensor"], sms=2)
    assert rc == 0, log


def test_packed_window_kernel_matches_oracle(host_library):
    """The packed window kernel with 5 SMs, so that each CTA walks several tiles: windows that continue
    the previous tile's ring and windows that start afresh at sequence and KV-group changes."""
    rc, log = run_cases(host_library, list(PACKED_CASES), sms=5)
    assert rc == 0, log


def test_packed_window_kernel_rescale_path(tmp_path):
    """The packed kernel's softmax keeps a lazily updated running max and rescales the P it has
    already written when a later score chunk passes it by more than the threshold -- rare with these
    inputs.  A build with threshold 0 rescales at every increase of the running max: the results
    must still match the oracle."""
    lib = build_library.build(str(tmp_path), mutations=[(
        "attn_fwd_swa_packed.cuh", "constexpr float kRescaleThreshold = 8.0f;",
        "constexpr float kRescaleThreshold = 0.0f;")])
    rc, log = run_cases(lib, list(PACKED_CASES), sms=5)
    assert rc == 0, log


def test_packed_window_kernel_rescale_mistake_is_caught(tmp_path):
    """The same threshold-0 build with the rescale of written P left out must fail."""
    lib = build_library.build(str(tmp_path), mutations=[
        ("attn_fwd_swa_packed.cuh", "constexpr float kRescaleThreshold = 8.0f;",
         "constexpr float kRescaleThreshold = 0.0f;"),
        ("attn_fwd_swa_packed.cuh", "pk[e] = pack_bf16x2(f.x * corr, f.y * corr);", "pk[e] = pack_bf16x2(f.x, f.y);")])
    rc, _ = run_cases(lib, ["fwd_packed_windows"], sms=5)
    assert rc != 0, "not caught: written P not rescaled when the running max grows"


def test_pipelined_kernel_rescale_path(tmp_path):
    """The pipelined kernel's softmax raises its running max lazily (when a tile's max passes it by
    more than the threshold) and then rescales O.  Under threshold 0 it rescales at every increase:
    the results must still match the oracle, and leaving the O rescale out must not."""
    thr = ("attn_fwd_pipelined.cuh", "constexpr float kRescaleThreshold = 8.0f;", "constexpr float kRescaleThreshold = 0.0f;")
    cases = ["fwd_global", "fwd_tiny_pipelined"]
    lib = build_library.build(str(tmp_path / "ok"), mutations=[thr])
    rc, log = run_cases(lib, cases)
    assert rc == 0, log
    lib = build_library.build(str(tmp_path / "no_o"), mutations=[thr, (
        "attn_fwd_pipelined.cuh", "o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);", "o[i] = o[i];")])
    rc, _ = run_cases(lib, cases)
    assert rc != 0, "not caught: O not rescaled"


def test_timed_out_waits_end_cleanly(tmp_path):
    """A build whose bounded waits have a zero limit: the forward kernels' roles give up on each other,
    record a timeout and leave without a deadlock or a warp-collective instruction with exited lanes."""
    lib = build_library.build(str(tmp_path), mutations=[(
        "mimo_attn_api.cu", "constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;",
        "constexpr uint64_t kDefaultWaitLimitNs = 0ull;")])
    rc, log = run_cases(lib, list(TIMEOUT_CASES))
    assert rc == 0, log


PLANTED = [
    ("rotated-dims K operand not advanced per K-step", "attn_fwd_pipelined.cuh",
     "mma_ss_lo(d_tmem, q0 + 2 * sub, k0 + 2 * sub, pipe::kIdescSF16",
     "mma_ss_lo(d_tmem, q0 + 2 * sub, k0, pipe::kIdescSF16", "fwd_tiny_pipelined"),
    ("V operand stepped by 8 keys instead of 16", "attn_fwd_pipelined.cuh",
     "v_lo + kk * (2048 >> 4)", "v_lo + kk * (1024 >> 4)", "fwd_tiny_pipelined"),
    ("KV-cache row tiles all start at row 0", "attn_decode_tc.cuh", "w.row0 = 128 * qt;", "w.row0 = 0;",
     "decode_tensor_tiles_swa"),
    ("KV-cache lander reads the previous chunk's angle table", "attn_decode_tc.cuh",
     "rope_rotate_chunk_pair_add(kr, r, c0 + h, base, off[h])",
     "rope_rotate_chunk_pair_add(kr, r, c0 + h, C->k_base[(landed + 1) & 1], off[h])",
     "decode_tensor_tiles_global"),
    ("KV-cache lander offsets each key row by one position too many", "attn_decode_tc.cuh",
     "rope_sincos(qt & 63, C->theta", "rope_sincos((qt & 63) + 1, C->theta", "decode_tensor"),
    ("backward dQ reads dS without its MN-major flag", "attn_bwd_tc.cuh",
     "kIdescDQ = make_idesc_f32acc(1, 1, 128, 192) | (1u << 15);", "kIdescDQ = make_idesc_f32acc(1, 1, 128, 192);",
     "bwd_tensor"),
    ("backward: dK / dV restarted for every head a CTA takes", "attn_bwd_tc.cuh", "first = h == h0;", "first = 1;",
     "bwd_tensor"),
    ("packed kernel: score columns mapped to keys one ring slot off", "attn_fwd_swa_packed.cuh",
     "const int c0 = (base + klo) % S::kN;", "const int c0 = (base + klo + kBlk) % S::kN;", "fwd_packed_g8"),
    ("packed kernel: K rotated at the next key's position", "attn_fwd_swa_packed.cuh",
     "* kBlk + r / 4;", "* kBlk + r / 4 + 1;", "fwd_packed_g8"),
    ("packed kernel: PV reads the V of the slot after each P", "attn_fwd_swa_packed.cuh",
     "v_lo + s * (kSlot >> 4)", "v_lo + ((s + 1) % S::kR) * (kSlot >> 4)", "fwd_packed_g8"),
    ("packed kernel: a continuing window re-uses one load too few", "attn_fwd_swa_packed.cuh",
     "new_from = max(p_blk_hi, blk_lo);", "new_from = max(p_blk_hi - 1, blk_lo);", "fwd_packed_g8"),
    ("scores read from TMEM without waiting for their MMAs", "attn_fwd_simple.cuh",
     "      fail = !mbar_wait(&bars[2], mma_phase, P.wait_limit_ns);\n      mma_phase ^= 1;\n"
     "      if (__syncthreads_or(fail)) { fail = true; break; }\n      tc_fence_after_sync();\n\n      uint32_t s[4][32];",
     "      mma_phase ^= 1;\n      if (__syncthreads_or(fail)) { fail = true; break; }\n      tc_fence_after_sync();\n\n"
     "      uint32_t s[4][32];", "fwd_tiny_simple"),
]


@pytest.mark.parametrize("what,file,old,new,case", PLANTED, ids=[p[0] for p in PLANTED])
def test_planted_kernel_mistake_is_caught(tmp_path, what, file, old, new, case):
    lib = build_library.build(str(tmp_path), mutations=[(file, old, new)])
    rc, _ = run_cases(lib, [case], sms=5 if case in PACKED_CASES else None)
    assert rc != 0, f"not caught: {what}"
