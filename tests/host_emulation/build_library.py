"""Builds the whole library (mimo_attn_api.cu with every kernel, tensor-core ones included) for the
CPU: a copy of csrc in which sm100.cuh and cp_async.cuh are replaced by the device models in
device_model/, the launches turned into fiber-runtime launches (as build_host.py does), the dynamic
shared memory pointed at the runtime's 1024-byte-aligned block, and the CUDA runtime calls defined in
cudart_host.h.  Linked with -Bsymbolic so that a CUDA runtime already in the process (torch's) cannot
take the place of those definitions.  Test infrastructure only."""
import os
import re
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


def _replace_function(s, signature, body):
    """Replaces the definition that starts with `signature` (up to its column-0 closing brace)."""
    a = s.index(signature)
    b = s.index("\n}\n", a) + 3
    return s[:a] + signature + " {\n" + body + "\n}\n" + s[b:]


# The SM-pair window kernel keeps its cluster and cta_group::2 instructions in helpers of its own; the
# host copy calls the device model instead (same arguments, same meaning).
PAIR_HELPERS = [
    ("__device__ __forceinline__ uint32_t cta_rank()", "  return static_cast<uint32_t>(hemu::g_cur_cta);"),
    ("__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank)",
     "  return cluster_addr(smem_u32(p), rank);"),
    ("__device__ __forceinline__ void arrive_cluster(uint32_t bar)",
     "  mbar_arrive_cta(cluster_cta(bar), cluster_off(bar));"),
    ("__device__ __forceinline__ void cluster_sync()", "  hemu::cluster_barrier();"),
    ("__device__ __forceinline__ bool try_wait_cluster(uint64_t* bar, uint32_t parity)",
     "  return mbar_try_wait(bar, parity);"),
    ("__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t leader_bar, int32_t x,\n"
     "                                                 int32_t y)", "  tma_load_2d_pair_model(dst, map, leader_bar, x, y);"),
    ("__device__ __forceinline__ void mma_ss_pair(uint32_t d, uint32_t a_lo, uint32_t b_lo, uint32_t idesc, uint32_t acc)",
     "  const uint64_t hi = static_cast<uint64_t>(kDescHiSw128Sbo1K) << 32;\n"
     "  mma_ss_pair_model(d, hi | a_lo, hi | b_lo, idesc, acc);"),
    ("__device__ __forceinline__ void mma_ts_pair(uint32_t d, uint32_t a_tmem, uint32_t b_lo, uint32_t idesc, uint32_t acc)",
     "  mma_ts_pair_model(d, a_tmem, (static_cast<uint64_t>(kDescHiSw128Sbo1K) << 32) | b_lo, idesc, acc);"),
    ("__device__ __forceinline__ void commit_pair(uint64_t* bar)", "  tc_commit_multicast(bar, kPair);"),
]
PAIR_STATEMENTS = [
    ('asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&C->tmem_base)),\n'
     '                 "r"(kTmemCols)\n                 : "memory");', "tmem_alloc(&C->tmem_base, kTmemCols);"),
    ('asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");', ""),
    ('asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(peer_skip) : "r"(peer_addr(&C->abort, rank ^ 1u)) : "memory");',
     "{ const uint32_t pa = peer_addr(&C->abort, rank ^ 1u);\n"
     "    std::memcpy(&peer_skip, hemu::g_smem_cta[cluster_cta(pa)] + cluster_off(pa), 4); }"),
    ('asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");', ""),
]


# The KV-cache kernel's gather4 fetcher keeps its TMA gather instruction in a helper of its own.
GATHER4_HELPER = ("__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x, "
                  "int32_t r0,\n                                            int32_t r1, int32_t r2, int32_t r3)",
                  "  tma_gather4_model(dst, map, bar, x, r0, r1, r2, r3);")


def adapt_pair_kernel(s):
    for sig, body in PAIR_HELPERS:
        s = _replace_function(s, sig, body)
    for old, new in PAIR_STATEMENTS:
        assert s.count(old) == 1, old[:60]
        s = s.replace(old, new)
    assert "asm" not in s.replace("asm volatile(\"\")", ""), "pair kernel: inline PTX left"
    return s


def build(out_dir: str, src_root: str = ROOT, mutations=()) -> str:
    """mutations: (file, old text, new text) applied to the copied sources (planted-mistake tests)."""
    # the repository's layout, so that the API file finds its header by its relative path
    csrc = os.path.join(out_dir, "global_attention_moe_b200", "csrc")
    shutil.rmtree(os.path.join(out_dir, "global_attention_moe_b200"), ignore_errors=True)
    shutil.rmtree(os.path.join(out_dir, "include"), ignore_errors=True)
    shutil.copytree(os.path.join(src_root, "global_attention_moe_b200", "csrc"), csrc)
    shutil.copytree(os.path.join(src_root, "include"), os.path.join(out_dir, "include"))
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
        if name == "attn_fwd_swa2.cuh":
            s = adapt_pair_kernel(s)
        if name == "attn_decode_tc.cuh" and "void tma_gather4(" in s:
            s = _replace_function(s, *GATHER4_HELPER)
        if name == "mimo_attn_api.cu":
            s, n = build_host._launches(s)
            assert n >= 16, n
            s = s.replace("g_launch_ok = hemu::launch(", "hemu::g_launch_failed |= !hemu::launch(")
            # the SM-pair kernel runs in two-CTA clusters
            s = re.sub(r"(\[&\] \{ attn_fwd_swa2_kernel\([^;]*\); \})\);", r"\1, 2);", s)
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
           "-I/usr/local/cuda/include", "-I" + HERE, tu, "-o", so]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode:
        raise RuntimeError("host build of the library failed:\n" + r.stderr[-4000:])
    return so
