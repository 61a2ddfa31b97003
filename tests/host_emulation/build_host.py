"""Compiles the library's CUDA-core kernels (backward, FP8 dequant, fused-QKV split, MoE router) and
their host entry points for the CPU against fiber_runtime.h, into a shared library for the tests.

The kernel files are taken as they are; the only source transforms are: project includes removed
(their few definitions are pulled in by name: params.cuh whole, the error bits of sm100.cuh, the
rope_sincos of rope_smem.cuh), the dynamic shared-memory declaration pointed at the runtime's guarded
block, `kernel<<<grid, block, smem, stream>>>(args)` turned into a runtime launch, and in the host
functions the device query, the pool allocation and cudaGetLastError replaced by host forms.
Test infrastructure only."""
import os
import re
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
CS = os.path.join(ROOT, "global_attention_moe_b200", "csrc")
SMS = 148  # grid sizes of the grid-stride kernels follow the B200's SM count

ENTRY_POINTS = ("mimo_attn_bwd", "mimo_fp8_dequant_blockwise", "mimo_qkv_split", "mimo_moe_route")


def _read(name):
    with open(os.path.join(CS, name)) as f:
        return f.read()


def _function(src, start):
    """Text of the function whose definition starts with `start` (ends at the first column-0 brace)."""
    a = src.index(start)
    b = src.index("\n}\n", a) + 3
    return src[a:b]


def _kernel(name):
    s = re.sub(r'#include "[^"]+"\n', "", _read(name)).replace("#pragma once", "")
    decl = "extern __shared__ __align__(16) float sm[];"
    if decl in s:
        s = s.replace(decl, "float* sm = reinterpret_cast<float*>(hemu::g_smem);")
    return s


def _launches(s):
    def rep(m):
        parts = [p.strip() for p in m.group(2).split(",")]
        smem = parts[2] if len(parts) > 2 else "0"
        return f"g_launch_ok = hemu::launch(dim3({parts[0]}), dim3({parts[1]}), {smem}, [&] {{ {m.group(1)}({m.group(3)}); }});"
    return re.subn(r"([\w:]+(?:<\d+>)?)<<<(.*?)>>>\((.*?)\);", rep, s, flags=re.S)


HOST_FORMS = [
    (r"  int dev = 0;\n  if \(cudaGetDevice\(&dev\) != cudaSuccess\) return MIMO_ERR_CUDA;\n", ""),
    (r"  DeviceInfo\* info = device_info\(dev\);\n", ""),
    (r"  if \(!info \|\| !info->kernels_ready \|\| !info->pool\) return MIMO_ERR_CUDA;\n", ""),
    (r"  if \(!info\) return MIMO_ERR_CUDA;\n", ""),
    (r"info->sms", "kSms"),
    (r"cudaMallocFromPoolAsync\(&scratch, ([^,]+), info->pool, stream\)", r"host_malloc(&scratch, \1)"),
    (r"cudaFreeAsync\(scratch, stream\)", "(hemu::guarded_free(scratch), cudaSuccess)"),
    (r"cudaGetLastError\(\)", "(g_launch_ok ? cudaSuccess : cudaErrorUnknown)"),
    (r"cudaMemsetAsync\(dsink, 0, ([^,]+), [^;]+\);", r"std::memset(dsink, 0, \1);"),
]


def generate() -> str:
    api = _read("mimo_attn_api.cu")
    host = _function(api, "int launch_bwd(") + "\n".join(_function(api, f"int {e}(") for e in ENTRY_POINTS)
    for pat, new in HOST_FORMS:
        host, n = re.subn(pat, new, host)
        assert n >= 1, f"host form not found: {pat}"
    host, n = _launches(host)
    assert n == 6, f"expected 6 launches, found {n}"
    rope = _read("rope_smem.cuh")
    rope = rope[rope.index("constexpr double kTwoPi"):rope.index("// Rotates chunk pair")]
    sm100 = _read("sm100.cuh")
    a = sm100.index("enum : unsigned int {")
    errs = sm100[a:sm100.index("};", a) + 2]
    validate = api[api.index("bool aligned16(const void* p)"):api.index("void fill_params(")]
    wrappers = []
    for e in ENTRY_POINTS:
        sig = _function(api, f"int {e}(")
        sig = sig[:sig.index("{")].strip()
        params = re.findall(r"(\w+)\s*(?:,|\)$)", sig)
        wrappers.append(f"{sig} {{ return mimo::{e}({', '.join(params)}); }}")
    return "\n".join([
        '#include "fiber_runtime.h"',
        f'#include "{os.path.join(ROOT, "include", "mimo_attn.h")}"',
        f'#include "{os.path.join(CS, "params.cuh")}"',
        "namespace mimo {", errs, rope, "}",
        _kernel("attn_bwd_simple.cuh"), _kernel("neighbors.cuh"),
        "namespace mimo {", "namespace {", f"constexpr int kSms = {SMS};", "bool g_launch_ok = true;", validate,
        "cudaError_t host_malloc(void** p, size_t n) { *p = hemu::guarded_alloc(n); return cudaSuccess; }",
        host, "}  // namespace", "}  // namespace mimo",
        'extern "C" {', *wrappers,
        "void* hemu_alloc(size_t n) { return hemu::guarded_alloc(n); }",
        "void hemu_free(void* p) { hemu::guarded_free(p); }",
        "void hemu_set_mode(int m) { hemu::g_mode = m; }",
        "int hemu_errors(void) { return hemu::g_errors; }",
        "unsigned hemu_error_word(void) { unsigned w = mimo::g_mimo_error; mimo::g_mimo_error = 0; return w; }",
        "}",
    ])


def build(out_dir: str, source: str | None = None) -> str:
    """Writes the generated source (or `source`) to out_dir and compiles it; returns the .so path."""
    os.makedirs(out_dir, exist_ok=True)
    src = os.path.join(out_dir, "host_kernels.cpp")
    with open(src, "w") as f:
        f.write(source if source is not None else generate())
    so = os.path.join(out_dir, "libhost_kernels.so")
    cmd = ["g++", "-std=c++20", "-O1", "-fPIC", "-shared", "-w", "-I/usr/local/cuda/include", "-I" + HERE, src,
           "-o", so]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode:
        raise RuntimeError("host build failed:\n" + r.stderr[-4000:])
    return so
