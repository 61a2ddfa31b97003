"""The C-ABI library: it loads, exports every symbol include/mimo_attn.h
declares, and rejects bad arguments before touching CUDA (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

from global_attention_moe_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def M():
    build.build()
    from global_attention_moe_b200 import mimo_attn
    return mimo_attn


def header_functions():
    src = open(os.path.join(ROOT, "include", "mimo_attn.h")).read()
    return sorted(set(re.findall(r"MIMO_API\s+[\w\s\*]*?\b(mimo_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(M):
    declared = header_functions()
    assert declared and sorted(M.SYMBOLS) == declared
    nm = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (mimo_\w+)", nm))
    assert set(declared) <= exported
    for name in declared:
        assert getattr(M.LIB, name) is not None


def test_status_strings_and_version(M):
    for s in range(8):
        assert M.status_string(s) and M.status_string(s) != "unknown status"
    assert M.status_string(99) == "unknown status"
    assert M.version()[0] == 1


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def call(M, dims, layer=0, window=128, base=1e4, rope_dims=64, sink=None, q=FAKE, out=FAKE, lse=FAKE):
    return M.fwd_raw(q, FAKE, FAKE, sink, FAKE, dims, layer, window, base, rope_dims, 0.707, out, lse, None)


@pytest.mark.parametrize("case,expect", [
    (dict(dims=dict(hq=6, hkv=4)), 1),             # Hq % Hkv != 0
    (dict(dims=dict(dqk=128)), 2),                  # head dims other than 192/128
    (dict(dims=dict(dv=192)), 2),
    (dict(rope_dims=32), 2),                        # only 64 rotary dims are built
    (dict(rope_dims=63), 1),                        # odd
    (dict(rope_dims=256), 1),                       # > head dim
    (dict(window=-1), 1),                           # SWA needs window >= 0
    (dict(layer=1, sink=FAKE), 1),                  # global layers have no sink
    (dict(layer=7), 1),                             # unknown layer kind
    (dict(base=0.0), 1),
    (dict(base=float("nan")), 1),
    (dict(q=FAKE + 8), 1),                          # misaligned
    (dict(out=0), 1),                               # null output
    (dict(out=FAKE + 16), 1),                       # output rows are written with 32-byte stores
    (dict(dims=dict(num_seqs=0)), 1),
    (dict(dims=dict(max_seqlen=10 ** 6)), 1),       # max_seqlen > total tokens
])
def test_validation_rejects(M, case, expect):
    d = dict(num_seqs=1, total_tokens=512, max_seqlen=512, hq=4, hkv=1, dqk=192, dv=128)
    d.update(case.pop("dims", {}))
    dims = M.make_dims(d["num_seqs"], d["total_tokens"], d["max_seqlen"], d["hq"], d["hkv"], d["dqk"], d["dv"])
    assert call(M, dims, **case) == expect


def test_null_dims_rejected(M):
    st = M.LIB.mimo_attn_fwd(FAKE, FAKE, FAKE, None, FAKE, None, 0, 128, 1e4, 64, 0.707, FAKE, FAKE, None)
    assert st == M.ERR_INVALID_ARG


def test_host_entry_checks_cu_seqlens_on_host(M):
    import torch
    dims = M.make_dims(2, 300, 200, 4, 1)
    ws_bytes = M.host_workspace_size(dims, True)
    assert ws_bytes > 300 * 4 * 192 * 2
    q = torch.zeros(300, 4, 192, dtype=torch.bfloat16)
    k = torch.zeros(300, 1, 192, dtype=torch.bfloat16)
    v = torch.zeros(300, 1, 128, dtype=torch.bfloat16)
    o = torch.zeros(300, 4, 128, dtype=torch.bfloat16)
    l = torch.zeros(4, 300)
    s = torch.zeros(4)

    class FakeWs:  # only size and address are read before the cu_seqlens check fails
        def data_ptr(self):
            return 1 << 20

        def numel(self):
            return ws_bytes

        def element_size(self):
            return 1

    for bad in ([0, 250, 300], [1, 100, 300], [0, 100, 299], [0, 150, 100]):
        cu = torch.tensor(bad, dtype=torch.int32)
        with pytest.raises(M.MimoAttnError) as e:
            M.LIB.mimo_attn_fwd_host  # noqa: B018
            st = M.LIB.mimo_attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), s.data_ptr(), cu.data_ptr(),
                                          ctypes.byref(dims), 0, 128, 1e4, 64, 0.707, o.data_ptr(), l.data_ptr(),
                                          FakeWs().data_ptr(), ws_bytes, None)
            if st != 0:
                raise M.MimoAttnError(st, "fwd_host")
        assert e.value.status == M.ERR_INVALID_ARG


def test_kernel_choice_values(M):
    for choice in (M.KERNEL_SIMPLE, M.KERNEL_PIPELINED, M.KERNEL_WINDOW, M.KERNEL_WINDOW_PACKED, M.KERNEL_AUTO):
        M.set_kernel(choice)
    for bad in (-1, 5, 99):
        with pytest.raises(M.MimoAttnError) as e:
            M.set_kernel(bad)
        assert e.value.status == M.ERR_INVALID_ARG
    M.set_kernel(M.KERNEL_AUTO)


def test_decode_kernel_choice_values(M):
    for choice in (M.DECODE_CUDA_CORES, M.DECODE_TENSOR, M.DECODE_AUTO):
        M.set_decode_kernel(choice)
    for bad in (-1, 3, 99):
        with pytest.raises(M.MimoAttnError) as e:
            M.set_decode_kernel(bad)
        assert e.value.status == M.ERR_INVALID_ARG
    M.set_decode_kernel(M.DECODE_AUTO)


@pytest.mark.parametrize("case,expect", [
    (dict(hq=6, hkv=4), 1),                 # Hq % Hkv != 0
    (dict(max_q_len=70000, total_q=70000, max_kv_len=70000, total_kv=70000, cache_rows=70000, hq=64, hkv=4), 2),
    # 70000 x 16 rows per KV head > 2^20
    (dict(max_q_len=20, max_kv_len=10), 1), # max_q_len > max_kv_len
    (dict(cache_rows=0), 1),                # keys but no cache
    (dict(dqk=128), 2),
    (dict(rope_dims=32), 2),
    (dict(window=-1), 1),
    (dict(layer=1, sink=FAKE), 1),
    (dict(q=FAKE + 8), 1),
    (dict(out=FAKE + 16), 1),               # output rows are written with 32-byte stores
])
def test_decode_validation_rejects(M, case, expect):
    d = dict(num_seqs=2, total_q=4, total_kv=100, cache_rows=128, max_q_len=2, max_kv_len=60, hq=8, hkv=2,
             dqk=192, dv=128)
    args = dict(layer=0, window=128, rope_dims=64, sink=None, q=FAKE, out=FAKE)
    for key in list(case):
        (d if key in d else args)[key] = case[key]
    dims = M.make_decode_dims(d["num_seqs"], d["total_q"], d["total_kv"], d["cache_rows"], d["max_q_len"],
                              d["max_kv_len"], d["hq"], d["hkv"], d["dqk"], d["dv"])
    st = M.decode_raw(args["q"], FAKE, FAKE, FAKE, FAKE, FAKE, args["sink"], dims, args["layer"], args["window"],
                      1e4, args["rope_dims"], 0.707, args["out"], FAKE, None)
    assert st == expect


@pytest.mark.parametrize("args,expect", [
    (dict(tokens=-1), 1),                      # negative token count
    (dict(k=0), 1),                            # no input features
    (dict(n=-8), 1),
    (dict(k=12), 2),                           # rows not a multiple of 16 bytes
    (dict(n=20), 2),
    (dict(k=1 << 31), 2),                      # beyond the GEMM's 32-bit sizes
    (dict(x=FAKE + 8), 1),                     # misaligned
    (dict(y=None), 1),                         # missing output
    (dict(tokens=0, x=None, w=None, y=None), 0),  # nothing to do: no pointer is needed
])
def test_linear_proj_validation(M, args, expect):
    a = dict(x=FAKE, w=FAKE, tokens=4, k=1024, n=512, y=FAKE)
    a.update(args)
    assert M.LIB.mimo_linear_proj(a["x"], a["w"], a["tokens"], a["k"], a["n"], a["y"], None) == expect


def test_noalloc_rejects_problems_beyond_its_scratch(M):
    """The no-alloc entry point checks its fixed scratch size before any CUDA
    call: one row past the limit is refused on a machine without a GPU too."""
    limit_rows = M.noalloc_scratch_bytes() // 128  # T * Hkv rows of 64 FP16 dims
    hkv = 8
    T = limit_rows // hkv + 1
    dims = M.make_dims(1, T, T, 16, hkv)
    st = M.LIB.mimo_attn_fwd_noalloc(FAKE, FAKE, FAKE, None, FAKE, ctypes.byref(dims), 1, -1, 1e7, 64, 0.707,
                                     FAKE, FAKE, None)
    assert st == M.ERR_SCRATCH_LIMIT
    assert "scratch" in M.status_string(st)


def test_profile_stride_values(M):
    for good in (1, 16):
        M.profile_set_stride(good)
    for bad in (0, -3):
        with pytest.raises(M.MimoAttnError) as e:
            M.profile_set_stride(bad)
        assert e.value.status == M.ERR_INVALID_ARG
    M.profile_set_stride(1)


@pytest.mark.parametrize("args,expect", [
    (dict(rows=-1), 1),                        # negative size
    (dict(bm=0), 1),                           # empty scale blocks
    (dict(bn=-4), 1),
    (dict(cols=40), 2),                        # rows not made of 16-byte chunks
    (dict(cols=1 << 31), 2),                   # beyond the kernel's 32-bit column index
    (dict(codes=FAKE + 8), 1),                 # misaligned
    (dict(scale=FAKE + 2), 1),
    (dict(out=None), 1),                       # missing output
    (dict(rows=0, codes=None, scale=None, out=None), 0),  # nothing to do: no pointer is needed
])
def test_fp8_dequant_validation(M, args, expect):
    a = dict(codes=FAKE, scale=FAKE, rows=256, cols=4096, bm=128, bn=128, out=FAKE)
    a.update(args)
    assert M.LIB.mimo_fp8_dequant_blockwise(a["codes"], a["scale"], a["rows"], a["cols"], a["bm"], a["bn"],
                                            a["out"], None) == expect
