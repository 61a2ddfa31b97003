// fiber_runtime.h -- host emulation of the CUDA thread model, so that the library's kernels run on
// the CPU in tests from their unchanged source (the CUDA-core kernels directly; the tensor-core kernels
// with the device model of their tcgen05 / TMA / mbarrier wrappers in device_model/):
//   - one fiber (ucontext) per CUDA thread, a cooperative scheduler per block, blocks one after another;
//   - __syncthreads / __syncwarp as barriers over the block's / warp's live fibers (exited threads do
//     not count, as on the GPU); a barrier that can never complete is reported as a deadlock;
//   - warp shuffles and votes through an exchange array, with an error if a lane has exited;
//   - named barriers 1..15 with thread counts (bar.sync, bar.red.and) and __syncthreads_or;
//   - a yield for spin-waits (a waiting fiber lets the others run);
//   - atomics as plain read-modify-write (a single OS thread runs every fiber);
//   - every buffer, and the block's dynamic shared memory, sits between two 16 MB PROT_NONE guard
//     regions, flush against the one at its end in mode 0 and the one at its start in mode 1, so an
//     out-of-range access faults on the host; it starts filled with 0xFF bytes (NaN as FP32 or
//     BF16), so a read of memory nobody wrote shows in the results.
// Device math: __sincosf is taken as the host's sinf/cosf (the GPU's is an approximation with an
// absolute error near 2^-21 on [-pi, pi]); exp2f, fmaf and the BF16/FP8 conversions are the host forms.
// Test infrastructure only: nothing in the library includes or calls it.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <sys/mman.h>
#include <ucontext.h>
#include <unistd.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <vector>

#undef __global__
#define __global__
#undef __device__
#define __device__
#undef __host__
#define __host__
#define __launch_bounds__(...)
#undef __noinline__
#define __noinline__
#define __cluster_dims__(...)
#define __grid_constant__
#undef __shared__
#define __shared__ static

using std::max;
using std::min;

namespace hemu {

inline int g_mode = 0;  // 0: buffers end at a guard page; 1: buffers start right after one
inline long g_page = sysconf(_SC_PAGESIZE);
inline constexpr size_t kGuard = size_t(16) << 20;  // PROT_NONE address space on each side of a buffer

struct Alloc {
  void* map;
  size_t map_bytes;
};
inline std::vector<std::pair<void*, Alloc>> g_allocs;

inline void* guarded_alloc(size_t nbytes) {
  const size_t n16 = (nbytes + 15) & ~size_t(15);
  const size_t body = (n16 + g_page - 1) / g_page * g_page;
  const size_t total = body + 2 * kGuard;
  uint8_t* m = static_cast<uint8_t*>(mmap(nullptr, total, PROT_READ | PROT_WRITE, MAP_PRIVATE | MAP_ANONYMOUS, -1, 0));
  if (m == MAP_FAILED) return nullptr;
  mprotect(m, kGuard, PROT_NONE);
  mprotect(m + kGuard + body, kGuard, PROT_NONE);
  uint8_t* p = g_mode == 0 ? m + kGuard + body - n16 : m + kGuard;
  std::memset(p, 0xFF, n16);  // NaN in every float / BF16 lane: a read of unwritten memory shows
  g_allocs.push_back({p, {m, total}});
  return p;
}

inline void guarded_free(void* p) {
  for (size_t i = 0; i < g_allocs.size(); ++i)
    if (g_allocs[i].first == p) {
      munmap(g_allocs[i].second.map, g_allocs[i].second.map_bytes);
      g_allocs.erase(g_allocs.begin() + i);
      return;
    }
}

struct Fiber {
  ucontext_t ctx;
  bool done;
  int wait;  // 0 runnable, 1 block barrier, 2 warp barrier, 3 named barrier, 4 cluster barrier
  int bar_id;
  int cta;   // CTA of the fiber within its cluster
  uint64_t gen;
  bool result;  // reduction result handed back by a barrier
};

constexpr int kMaxCluster = 8;
// Per-CTA barrier state (the blocks of one cluster run together): block barrier (bar.sync 0, with the
// OR reduction of __syncthreads_or) and named barriers 1..15 (thread counts, AND reduction).
struct CtaState {
  uint64_t block_gen = 0;
  int block_arrived = 0;
  bool block_or = false;
  int nb_count[16] = {}, nb_arrived[16] = {};
  uint64_t nb_gen[16] = {};
  bool nb_and[16] = {};
};
inline CtaState g_cta[kMaxCluster];
inline int g_cluster = 1;    // CTAs per cluster of the current launch
inline int g_cur_cta = 0;    // CTA of the running fiber
inline uint64_t g_cl_gen = 0;
inline int g_cl_arrived = 0;
inline std::vector<std::function<void(int)>> g_block_reset;  // per-CTA state of device models (CTA index)
inline bool g_smem_start_aligned = false;

inline uint3 g_tid_cur, g_bid_cur;
inline dim3 g_grid_dim, g_block_dim;
inline std::vector<Fiber> g_fibers;
inline std::vector<uint8_t*> g_stacks;
inline constexpr size_t kStack = 256 * 1024;
inline ucontext_t g_sched;
inline int g_cur = -1;
inline std::vector<uint64_t> g_warp_gen;
inline std::vector<int> g_warp_arrived;
inline std::function<void()> g_body;
inline uint8_t* g_smem = nullptr;  // the running fiber's CTA's shared memory
inline uint8_t* g_smem_cta[kMaxCluster] = {};
inline uint64_t g_xch[64 * kMaxCluster][32];
inline int g_errors = 0;

inline int lin_tid() { return static_cast<int>(g_tid_cur.x + g_block_dim.x * (g_tid_cur.y + g_block_dim.y * g_tid_cur.z)); }
inline int warp_slot() { return g_cur / 32; }  // warp index over the whole cluster

inline void syncthreads() {
  Fiber& f = g_fibers[g_cur];
  CtaState& c = g_cta[f.cta];
  f.wait = 1;
  f.gen = c.block_gen;
  ++c.block_arrived;
  swapcontext(&f.ctx, &g_sched);
}

inline bool syncthreads_or(bool pred) {
  CtaState& c = g_cta[g_fibers[g_cur].cta];
  c.block_or = c.block_or || pred;
  syncthreads();
  return g_fibers[g_cur].result;
}

// Every thread of every CTA of the cluster (barrier.cluster arrive + wait).
inline void cluster_barrier() {
  Fiber& f = g_fibers[g_cur];
  f.wait = 4;
  f.gen = g_cl_gen;
  ++g_cl_arrived;
  swapcontext(&f.ctx, &g_sched);
}

// Lets the other fibers run (a spin-wait step).
inline void yield() {
  Fiber& f = g_fibers[g_cur];
  f.wait = 0;
  swapcontext(&f.ctx, &g_sched);
}

inline bool named_bar(int id, int nthreads, bool pred) {
  Fiber& f = g_fibers[g_cur];
  CtaState& c = g_cta[f.cta];
  if (c.nb_arrived[id] == 0) {
    c.nb_count[id] = nthreads;
    c.nb_and[id] = true;
  } else if (c.nb_count[id] != nthreads) {
    std::fprintf(stderr, "emu: named barrier %d used with %d and %d threads\n", id, c.nb_count[id], nthreads);
    ++g_errors;
  }
  c.nb_and[id] = c.nb_and[id] && pred;
  ++c.nb_arrived[id];
  f.wait = 3;
  f.bar_id = id;
  f.gen = c.nb_gen[id];
  swapcontext(&f.ctx, &g_sched);
  return g_fibers[g_cur].result;
}

inline void syncwarp() {
  Fiber& f = g_fibers[g_cur];
  const int w = warp_slot();
  f.wait = 2;
  f.gen = g_warp_gen[w];
  ++g_warp_arrived[w];
  swapcontext(&f.ctx, &g_sched);
}

template <class T>
inline T shfl_idx(T v, int src) {
  static_assert(sizeof(T) <= 8, "shuffle width");
  const int w = warp_slot(), l = lin_tid() % 32;
  std::memcpy(&g_xch[w][l], &v, sizeof(T));
  syncwarp();
  T r;
  std::memcpy(&r, &g_xch[w][src & 31], sizeof(T));
  syncwarp();
  return r;
}

inline void trampoline() {
  g_body();
  g_fibers[g_cur].done = true;
}

inline uint8_t* g_smem_map[kMaxCluster] = {};
inline size_t g_smem_map_bytes[kMaxCluster] = {};

inline void set_smem(int cta, size_t bytes) {
  if (g_smem_map[cta]) munmap(g_smem_map[cta], g_smem_map_bytes[cta]);
  const size_t n16 = (bytes + 15) & ~size_t(15);
  const size_t body = (n16 + g_page - 1) / g_page * g_page + g_page;
  g_smem_map_bytes[cta] = body + 2 * kGuard;
  uint8_t* m = static_cast<uint8_t*>(
      mmap(nullptr, g_smem_map_bytes[cta], PROT_READ | PROT_WRITE, MAP_PRIVATE | MAP_ANONYMOUS, -1, 0));
  g_smem_map[cta] = m;
  mprotect(m, kGuard, PROT_NONE);
  mprotect(m + kGuard + body, kGuard, PROT_NONE);
  g_smem_cta[cta] = (g_mode == 0 && !g_smem_start_aligned) ? m + kGuard + body - n16 : m + kGuard;
}

// Runs fn (the kernel call) for every thread of every block; blocks in clusters of `cluster` CTAs
// along x run together.  Returns false on a barrier deadlock or a warp-collective with exited lanes.
inline bool launch(dim3 grid, dim3 block, size_t smem_bytes, const std::function<void()>& fn, int cluster = 1) {
  g_grid_dim = grid;
  g_block_dim = block;
  const int nt = static_cast<int>(block.x * block.y * block.z);
  const int nw = (nt + 31) / 32;
  if (nw > 64 || cluster < 1 || cluster > kMaxCluster || grid.x % cluster != 0 || (cluster > 1 && nt % 32 != 0))
    return false;
  if (smem_bytes > 227 * 1024) {
    std::fprintf(stderr, "emu: dynamic shared memory %zu above the per-block limit\n", smem_bytes);
    return false;
  }
  g_cluster = cluster;
  for (int c = 0; c < cluster; ++c) set_smem(c, smem_bytes > 0 ? smem_bytes : 16);
  const int nf = nt * cluster, nwf = nw * cluster;
  while (static_cast<int>(g_stacks.size()) < nf) g_stacks.push_back(static_cast<uint8_t*>(std::malloc(kStack)));
  g_fibers.assign(nf, Fiber{});
  g_warp_gen.assign(nwf, 0);
  g_warp_arrived.assign(nwf, 0);
  g_body = fn;
  for (unsigned bz = 0; bz < grid.z; ++bz)
    for (unsigned by = 0; by < grid.y; ++by)
      for (unsigned bx0 = 0; bx0 < grid.x; bx0 += cluster) {
        for (int c = 0; c < cluster; ++c) {
          std::memset(g_smem_cta[c], 0xFF, smem_bytes);
          g_cta[c] = CtaState{};
          for (auto& h : g_block_reset) h(c);
        }
        g_cl_gen = 0;
        g_cl_arrived = 0;
        std::fill(g_warp_arrived.begin(), g_warp_arrived.end(), 0);
        for (int i = 0; i < nf; ++i) {
          Fiber& f = g_fibers[i];
          f.done = false;
          f.wait = 0;
          f.gen = 0;
          f.cta = i / nt;
          getcontext(&f.ctx);
          f.ctx.uc_stack.ss_sp = g_stacks[i];
          f.ctx.uc_stack.ss_size = kStack;
          f.ctx.uc_link = &g_sched;
          makecontext(&f.ctx, trampoline, 0);
        }
        for (;;) {
          bool progress = false;
          int alive_all = 0;
          std::vector<int> alive_w(nwf, 0), alive_c(cluster, 0);
          for (int i = 0; i < nf; ++i) {
            Fiber& f = g_fibers[i];
            if (f.done) continue;
            const CtaState& c = g_cta[f.cta];
            if (f.wait == 1 && f.gen == c.block_gen) continue;
            if (f.wait == 2 && f.gen == g_warp_gen[i / 32]) continue;
            if (f.wait == 3 && f.gen == c.nb_gen[f.bar_id]) continue;
            if (f.wait == 4 && f.gen == g_cl_gen) continue;
            f.wait = 0;
            g_cur = i;
            g_cur_cta = f.cta;
            g_smem = g_smem_cta[f.cta];
            const int t = i % nt;
            g_tid_cur = make_uint3(t % block.x, (t / block.x) % block.y, t / (block.x * block.y));
            g_bid_cur = make_uint3(bx0 + f.cta, by, bz);
            swapcontext(&g_sched, &f.ctx);
            progress = true;
          }
          for (int i = 0; i < nf; ++i)
            if (!g_fibers[i].done) {
              ++alive_all;
              ++alive_w[i / 32];
              ++alive_c[i / nt];
            }
          if (alive_all == 0) break;
          for (int cc = 0; cc < cluster; ++cc) {
            CtaState& c = g_cta[cc];
            if (c.block_arrived > 0 && c.block_arrived == alive_c[cc]) {
              for (int i = cc * nt; i < (cc + 1) * nt; ++i)
                if (!g_fibers[i].done && g_fibers[i].wait == 1) g_fibers[i].result = c.block_or;
              ++c.block_gen;
              c.block_arrived = 0;
              c.block_or = false;
              progress = true;
            }
            for (int id = 0; id < 16; ++id)
              if (c.nb_arrived[id] > 0 && c.nb_arrived[id] == c.nb_count[id]) {
                for (int i = cc * nt; i < (cc + 1) * nt; ++i)
                  if (!g_fibers[i].done && g_fibers[i].wait == 3 && g_fibers[i].bar_id == id &&
                      g_fibers[i].gen == c.nb_gen[id])
                    g_fibers[i].result = c.nb_and[id];
                ++c.nb_gen[id];
                c.nb_arrived[id] = 0;
                progress = true;
              }
          }
          if (g_cl_arrived > 0 && g_cl_arrived == alive_all) {
            ++g_cl_gen;
            g_cl_arrived = 0;
            progress = true;
          }
          for (int w = 0; w < nwf; ++w)
            if (g_warp_arrived[w] > 0 && g_warp_arrived[w] == alive_w[w]) {
              if (alive_w[w] != std::min(32, nt - 32 * (w % nw))) {
                std::fprintf(stderr, "emu: warp-collective with exited lanes (block %u,%u,%u warp %d)\n", bx0, by, bz, w);
                ++g_errors;
              }
              ++g_warp_gen[w];
              g_warp_arrived[w] = 0;
              progress = true;
            }
          if (!progress) {
            std::fprintf(stderr, "emu: barrier deadlock in cluster at block %u,%u,%u (alive %d)\n", bx0, by, bz,
                         alive_all);
            ++g_errors;
            return false;
          }
        }
      }
  return g_errors == 0;
}

}  // namespace hemu

// the built-in index variables: references to the running fiber's values (variables, not macros, so
// that members of the same names, such as cudaLaunchConfig_t::gridDim, stay untouched)
inline const uint3& threadIdx = hemu::g_tid_cur;
inline const uint3& blockIdx = hemu::g_bid_cur;
inline const dim3& gridDim = hemu::g_grid_dim;
inline const dim3& blockDim = hemu::g_block_dim;
#define __syncthreads() hemu::syncthreads()
#define __syncwarp(...) hemu::syncwarp()

template <class T>
inline T __ldg(const T* p) { return *p; }
template <class T>
inline T __shfl_xor_sync(unsigned, T v, int o) { return hemu::shfl_idx(v, (hemu::lin_tid() % 32) ^ o); }
template <class T>
inline T __shfl_sync(unsigned, T v, int src) { return hemu::shfl_idx(v, src); }
template <class T>
inline T __shfl_up_sync(unsigned, T v, int d) {  // lanes below d keep their own value
  const int l = hemu::lin_tid() % 32;
  return hemu::shfl_idx(v, l >= d ? l - d : l);
}
template <class T>
inline T atomicAdd(T* p, T v) {
  const T o = *p;
  *p = o + v;
  return o;
}
inline bool __all_sync(unsigned, int pred) {
  const int l = hemu::lin_tid() % 32, w = hemu::warp_slot();
  hemu::g_xch[w][l] = pred != 0;
  hemu::syncwarp();
  bool r = true;
  for (int i = 0; i < 32; ++i) r = r && hemu::g_xch[w][i] != 0;
  hemu::syncwarp();
  return r;
}
inline bool __any_sync(unsigned, int pred) {
  const int l = hemu::lin_tid() % 32, w = hemu::warp_slot();
  hemu::g_xch[w][l] = pred != 0;
  hemu::syncwarp();
  bool r = false;
  for (int i = 0; i < 32; ++i) r = r || hemu::g_xch[w][i] != 0;
  hemu::syncwarp();
  return r;
}
inline unsigned __ballot_sync(unsigned, int pred) {
  const int l = hemu::lin_tid() % 32, w = hemu::warp_slot();
  hemu::g_xch[w][l] = pred != 0;
  hemu::syncwarp();
  unsigned r = 0;
  for (int i = 0; i < 32; ++i) r |= (hemu::g_xch[w][i] != 0 ? 1u : 0u) << i;
  hemu::syncwarp();
  return r;
}
inline int __popc(unsigned v) { return __builtin_popcount(v); }
inline int __ffs(unsigned v) { return __builtin_ffs(static_cast<int>(v)); }
inline float __fdiv_rn(float a, float b) { return a / b; }
inline float __fmul_rn(float a, float b) { return a * b; }  // SSE: one IEEE rounding, subnormals kept

inline float __fdividef(float a, float b) { return a / b; }
inline float __expf(float x) { return std::exp(x); }
inline int __syncthreads_or(int pred) { return hemu::syncthreads_or(pred != 0); }
inline uint32_t __float_as_uint(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}
inline float atomicAdd(float* p, float v) {
  const float o = *p;
  *p = o + v;
  return o;
}
inline unsigned atomicOr(unsigned* p, unsigned v) {
  const unsigned o = *p;
  *p = o | v;
  return o;
}
inline float __uint_as_float(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
inline void __sincosf(float x, float* s, float* c) {
  *s = std::sin(x);
  *c = std::cos(x);
}
