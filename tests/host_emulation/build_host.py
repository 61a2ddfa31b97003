"""Compiles the library's CUDA-core kernels (backward, FP8 dequant, fused-QKV split, MoE router, the
KV-cache partial and combine kernels) and their host entry points for the CPU against
fiber_runtime.h, into a shared library for the tests.

The kernel files are taken as they are; the only source transforms are: project includes removed
(their few definitions are pulled in by name: params.cuh whole, the error bits of sm100.cuh, the
rope_sincos of rope_smem.cuh, ex2_approx as the host exp2f), the dynamic shared-memory declaration
pointed at the runtime's guarded block, the tensor-core KV-cache kernel replaced by a stub that
records an error if it is ever launched, `kernel<<<grid, block, smem, stream>>>(args)` turned into a
runtime launch, and in the host functions the device query, the pool allocation, the stream-ordered
memset and cudaGetLastError replaced by host forms.
Test infrastructure only."""
import os
import re
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
CS = os.path.join(ROOT, "global_attention_moe_b200", "csrc")
SMS = 148  # grid sizes of the grid-stride kernels follow the B200's SM count

ENTRY_POINTS = ("mimo_attn_bwd", "mimo_fp8_dequant_blockwise", "mimo_qkv_split", "mimo_moe_route",
                "mimo_attn_decode", "mimo_attn_set_decode_kernel", "mimo_attn_set_bwd_kernel")


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


def _split_top(cfg):
    """Splits a launch configuration at the commas outside parentheses."""
    parts, depth, cur = [], 0, ""
    for ch in cfg:
        if ch == "," and depth == 0:
            parts.append(cur.strip())
            cur = ""
            continue
        depth += ch == "("
        depth -= ch == ")"
        cur += ch
    return parts + [cur.strip()]


def _launches(s):
    def rep(m):
        parts = _split_top(m.group(2))
        smem = parts[2] if len(parts) > 2 else "0"
        return f"g_launch_ok = hemu::launch(dim3({parts[0]}), dim3({parts[1]}), {smem}, [&] {{ {m.group(1)}({m.group(3)}); }});"
    return re.subn(r"([\w:]+(?:<[\w, ]+>)?)<<<(.*?)>>>\((.*?)\);", rep, s, flags=re.S)


HOST_FORMS = [
    (r"  int dev = 0;\n  if \(cudaGetDevice\(&dev\) != cudaSuccess\) return MIMO_ERR_CUDA;\n", ""),
    (r"  DeviceInfo\* info = device_info\(dev\);\n", ""),
    (r"  if \(!info \|\| !info->kernels_ready \|\| !info->pool\) return MIMO_ERR_CUDA;\n", ""),
    (r"  if \(!info\) return MIMO_ERR_CUDA;\n", ""),
    (r"info->sms", "kSms"),
    (r"cudaMallocFromPoolAsync\(&(\w+), ([^,]+), info->pool, stream\)", r"host_malloc(&\1, \2)"),
    (r"cudaFreeAsync\((\w+), stream\)", r"(hemu::guarded_free(\1), cudaSuccess)"),
    (r"cudaMemsetAsync\(P\.item_counter, 0, sizeof\(unsigned long long\), stream\)",
     "(std::memset(P.item_counter, 0, sizeof(unsigned long long)), cudaSuccess)"),
    (r"cudaGetLastError\(\)", "(g_launch_ok ? cudaSuccess : cudaErrorUnknown)"),
    (r"cudaMemsetAsync\(dsink, 0, ([^,]+), [^;]+\);", r"std::memset(dsink, 0, \1);"),
]


# forms that only some versions of the host code contain
OPTIONAL_HOST_FORMS = [
    (r"cudaMemsetAsync\((\w+), 0, ([^,]+), stream\)", r"(std::memset(\1, 0, \2), cudaSuccess)"),
    (r"  if \(!bwd_attributes_ready\(dev\)\) return MIMO_ERR_CUDA;\n", ""),
]


def generate() -> str:
    api = _read("mimo_attn_api.cu")
    host = "\n".join([_function(api, "int launch_bwd("), _function(api, "int launch_decode(")] +
                     [_function(api, f"int {e}(") for e in ENTRY_POINTS])
    for pat, new in HOST_FORMS:
        host, n = re.subn(pat, new, host)
        assert n >= 1, f"host form not found: {pat}"
    for pat, new in OPTIONAL_HOST_FORMS:
        host = re.sub(pat, new, host)
    host, n = _launches(host)
    assert n >= 9, f"expected at least 9 launches, found {n}"
    rope = _read("rope_smem.cuh")
    rope = rope[rope.index("constexpr double kTwoPi"):rope.index("// Rotates chunk pair")]
    sm100 = _read("sm100.cuh")
    a = sm100.index("enum : unsigned int {")
    errs = sm100[a:sm100.index("};", a) + 2]
    validate = api[api.index("bool aligned16(const void* p)"):api.index("void fill_params(")]
    validate += api[api.index("// Query rows per KV head (q_len x Hq/Hkv)"):api.index("int launch_decode(")]
    lines = [ln for ln in api.splitlines() if ln.startswith(("constexpr uint64_t kDefaultWaitLimitNs", "constexpr int kBwdHeadsPerCta",
                                                             "std::atomic<int> g_decode_choice", "size_t align256(",
                                                             "std::atomic<int> g_bwd_choice"))]
    assert len(lines) >= 3, lines
    tc = _read("attn_decode_tc.cuh")
    tc_consts = [re.search(rf"constexpr (\w+) {n} = [^;]+;", tc).group(0) for n in ("kThreads", "kChunk")]
    tc_stub = ("namespace dtc {\n" + "\n".join(tc_consts) + "\nconstexpr uint32_t kSmemBytes = 0;\n}\n"
               "template <class... A> void attn_decode_tc_kernel(const A&...) { ++hemu::g_errors; }\n"
               "template <class... A> bool encode_2d(A...) { return false; }  // tensor maps: device path only\n")
    if "attn_bwd_tc_kernel" in api:  # the tensor-core backward: device path only (the device model runs it)
        tc_stub += ("namespace bwdtc {\nconstexpr int kThreads = 128;\nconstexpr uint32_t kSmemBytes = 0;\n}\n"
                    "template <class... A> void attn_bwd_tc_kernel(const A&...) { ++hemu::g_errors; }\n"
                    "template <class... A> void bwdtc_prep_kernel(const A&...) { ++hemu::g_errors; }\n")
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
        "#include <atomic>",
        "#include <cuda.h>",
        "namespace mimo {", errs, rope, "inline float ex2_approx(float x) { return exp2f(x); }", "}",
        _kernel("attn_bwd_simple.cuh"), _kernel("neighbors.cuh"), _kernel("attn_decode.cuh"),
        "namespace mimo {", tc_stub, "namespace {", f"constexpr int kSms = {SMS};", "bool g_launch_ok = true;",
        *lines, validate,
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
    cmd = ["g++", "-std=c++20", "-O1", "-fno-strict-aliasing", "-fPIC", "-shared", "-w", "-I/usr/local/cuda/include", "-I" + HERE, src,
           "-o", so]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode:
        raise RuntimeError("host build failed:\n" + r.stderr[-4000:])
    return so
