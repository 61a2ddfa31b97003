"""The CUDA-core kernels (backward, FP8 blockwise dequant, fused-QKV split, MoE router, the KV-cache
partial kernel in 128-row tiles and the combine) and their C entry points, compiled unchanged for the
CPU against a fiber runtime (tests/host_emulation), compared with the oracle.  Every buffer and the
shared-memory block sit against guard pages, once at their end and once at their start, so any
out-of-range index faults, and start filled with NaN, so a read of memory nobody wrote shows;
barriers and warp shuffles are checked for deadlock and exited lanes.  This checks the kernels' index
arithmetic, masks and block-level protocol on the CPU; the GPU parity tests check them on the
device."""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
EMU = os.path.join(HERE, "host_emulation")
sys.path.insert(0, EMU)
import build_host  # noqa: E402
from cases import CASES  # noqa: E402


@pytest.fixture(scope="module")
def host_lib(tmp_path_factory):
    return build_host.build(str(tmp_path_factory.mktemp("host_kernels")))


def run_cases(lib, mode, names):
    r = subprocess.run([sys.executable, os.path.join(EMU, "cases.py"), lib, str(mode), *names],
                       capture_output=True, text=True, timeout=600)
    return r.returncode, (r.stdout + r.stderr)[-2000:]


@pytest.mark.parametrize("mode", [0, 1])
def test_kernels_match_oracle(host_lib, mode):
    rc, log = run_cases(host_lib, mode, list(CASES))
    assert rc == 0, log


# Mistakes planted in the host copy of the kernels, each of which the cases above must catch.
PLANTED = [
    ("dequant reads and writes one row past the end", "has1 = i1 < M;", "has1 = i1 <= M;", "dequant"),
    ("dequant rounds the FP32 product to BF16 without the midpoint check",
     "      mid |= (__float_as_uint(b) & 0xFFFFu) == 0x8000u;\n", "", "dequant"),
    ("dequant takes the first block's scale one column past its edge", "(j < c.edge ? s0 : s1)",
     "(j <= c.edge ? s0 : s1)", "dequant"),
    ("dequant's exact path rounds the product to FP32 first",
     "static_cast<double>(dequant_code(lut, cw[jj >> 2], jj & 3)) *\n                                                  static_cast<double>(sc)",
     "static_cast<float>(dequant_code(lut, cw[jj >> 2], jj & 3)) *\n                                                  static_cast<float>(sc)",
     "dequant"),
    ("shared-memory block one row-vector short", "kRows * kPS + 2 * kRows) * 4;", "kRows * kPS + kRows) * 4;",
     "bwd_window0"),
    ("barrier between the K/V load and its rotation dropped",
     "    __syncthreads();\n    for (int e = tid; e < kChunk * (kRopeDims / 2); e += kThreads) {",
     "    for (int e = tid; e < kChunk * (kRopeDims / 2); e += kThreads) {", "bwd_window0"),
    ("window mask one key short", "pos - kpos <= P.window", "pos - kpos < P.window", "bwd_window31_mqa"),
    ("router ties to the higher expert", "(ok == bk && oe < be)", "(ok == bk && oe > be)", "route"),
    ("QKV split writes V eight elements off", "dst = v + (t * hkv + g) * 128 + (o - group * 192 - 192);",
     "dst = v + (t * hkv + g) * 128 + (o - group * 192 - 184);", "split"),
    ("two-token router: the halves' candidate buffers overlap", "(threadIdx.x >> 5) * 96 + 3 * hbase;",
     "(threadIdx.x >> 5) * 96 + hbase;", "route"),
    ("two-token router: slot scan skips one lane's count", "if (hl >= o) scan += y;", "if (hl > o) scan += y;",
     "route"),
    ("two-token router: the exact loop runs for the first token of the pair", "const int64_t ts = 2 * pr + hh;",
     "const int64_t ts = 2 * pr;", "route"),
    ("router ranks tied candidates by the higher expert", "\n            rank += (kj > key || (kj == key && c_id[j] < id))",
     "\n            rank += (kj > key || (kj == key && c_id[j] > id))", "route"),
    ("two-token router ranks tied candidates by the higher expert",
     "| static_cast<uint32_t>(~id);", "| static_cast<uint32_t>(id);", "route"),
    ("two-token router orders negative keys as unsigned bits", "(kb & 0x80000000u) ? ~kb : (kb | 0x80000000u)",
     "kb", "route"),
    ("router candidates all written to the first slot", "const int pos = at + __popc(cand[m] & ((1u << lane) - 1u));",
     "const int pos = at;", "route"),
    ("decode row tiles all start at row 0", "const int row0 = kMaxRows * qt;", "const int row0 = 0;",
     "decode_tiles_swa"),
    ("decode combine reads splits before the tile's keys", "const int s_lo = (lo_t - lo) / P.split_keys,",
     "const int s_lo = 0,", "decode_tiles_swa_long"),
    ("decode dereferences a cache index outside the cache",
     "bad_index = true;\n        row = 0;", "bad_index = true;", "decode_bad_index"),
]


@pytest.mark.parametrize("what,old,new,case", PLANTED, ids=[p[0] for p in PLANTED])
def test_planted_mistake_is_caught(tmp_path, what, old, new, case):
    src = build_host.generate()
    assert src.count(old) == 1, what
    lib = build_host.build(str(tmp_path), src.replace(old, new))
    rc = max(run_cases(lib, m, [case])[0] != 0 for m in (0, 1))
    assert rc, f"not caught: {what}"
