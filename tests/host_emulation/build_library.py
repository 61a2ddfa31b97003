"""Builds the whole library (mimo_attn_api.cu with every kernel, tensor-core ones included) for the
CPU: a copy of csrc in which sm100.cuh and cp_async.cuh are replaced by the device models in
device_model/, the launches turned into fiber-runtime launches (as build_host.py does), the dynamic
shared memory pointed at the runtime's 1024-byte-aligned block, and the CUDA runtime calls defined in
cudart_host.h.  Linked with -Bsymbolic so that a CUDA runtime already in the process (torch's) cannot
take the place of those definitions.  Test infrastructure only."""
import os
import shutil
import subprocess

import build_host

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))

EXPORTS = '''
extern "C" {
__attribute__((visibility("default"))) void* hemu_alloc(size_t n) { return hemu::guarded_alloc(n); }
__attribute__((visibility("default"))) void hemu_free(void* p) { hemu::guarded_free(p); }
__attribute__((visibility("default"))) int hemu_errors(void) { return hemu::g_errors; }
}
'''


def build(out_dir: str, src_root: str = ROOT, mutations=()) -> str:
    """mutations: (file, old text, new text) applied to the copied sources (planted-mistake tests)."""
    csrc = os.path.join(out_dir, "csrc")
    shutil.rmtree(csrc, ignore_errors=True)
    shutil.copytree(os.path.join(src_root, "global_attention_moe_b200", "csrc"), csrc)
    for h in ("sm100.cuh", "cp_async.cuh"):
        shutil.copy(os.path.join(HERE, "device_model", h), os.path.join(csrc, h))
    decls = {"extern __shared__ __align__(1024) uint8_t smem[];": "uint8_t* smem = hemu::g_smem;",
             "extern __shared__ __align__(16) float sm[];": "float* sm = reinterpret_cast<float*>(hemu::g_smem);",
             "extern __shared__ uint8_t smem_raw[];": "uint8_t* smem_raw = hemu::g_smem;"}
    for name in os.listdir(csrc):
        p = os.path.join(csrc, name)
        with open(p) as f:
            s = f.read()
        for a, b in decls.items():
            s = s.replace(a, b)
        for f, old, new in mutations:
            if f == name:
                assert s.count(old) == 1, (f, old)
                s = s.replace(old, new)
        if name == "mimo_attn_api.cu":
            s, n = build_host._launches(s)
            assert n >= 16, n
            s = s.replace("g_launch_ok = hemu::launch(", "hemu::g_launch_failed |= !hemu::launch(")
        with open(p, "w") as f:
            f.write(s)
    tu = os.path.join(out_dir, "library_host.cpp")
    with open(tu, "w") as f:
        f.write('#include "fiber_runtime.h"\n'
                "static bool g_align = (hemu::g_smem_start_aligned = true);  // 1024-byte swizzle atoms\n"
                '#include "cudart_host.h"\n'
                f'#include "{os.path.join(csrc, "mimo_attn_api.cu")}"\n'
                '#include "tensormap_host.h"\n' + EXPORTS)
    so = os.path.join(out_dir, "libmimo_attn_host.so")
    cmd = ["g++", "-std=c++20", "-O2", "-fno-strict-aliasing", "-fPIC", "-shared", "-w", "-Wl,-Bsymbolic",
           "-I/usr/local/cuda/include", "-I" + HERE, "-I" + os.path.join(src_root, "include"), tu, "-o", so]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode:
        raise RuntimeError("host build of the library failed:\n" + r.stderr[-4000:])
    return so
