// device_model/sm100.cuh -- host model of the library's sm100.cuh wrappers (mbarriers, TMA, tcgen05,
// TMEM), so that the tensor-core kernels run unchanged on the CPU in tests (see build_library.py);
// the library never includes it.  Modelled from the PTX ISA's description of each instruction:
//   mbarrier: expected arrivals, pending arrivals, signed transaction bytes, phase; a phase completes
//             when both reach zero; try_wait.parity P succeeds once the phase of parity P is over.
//   TMA 2-D tile load/store: {64, box_rows} boxes of 16-bit elements, 128-byte swizzle by address
//             (16-byte chunk c of the 128-byte row at smem address a goes to chunk c ^ ((a >> 7) & 7)),
//             zero fill outside the tensor, completion as transaction bytes.
//   tcgen05:  TMEM 128 lanes x 512 columns of 32 bits per block; MMAs are queued by the issuing thread
//             and run only when a thread first polls a barrier that their commit arrives on (the
//             latest moment the hardware could finish them), so an operand overwritten, or an
//             accumulator read, before that wait shows; SS (A K- or MN-major) and TS forms,
//             kind::f16, M = 128; the
//             16-term dot product of one instruction in FP64, added once to the FP32 accumulator.
//   tcgen05.ld/st 32x32b: warp-collective (a warp barrier); warp w reaches lanes 32 (w % 4) .. +31
//             only (checked).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <chrono>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <unordered_map>
#include <vector>

namespace mimo {

enum : unsigned int {
  kErrTimeout = 1u,
  kErrRange = 2u,
  kErrSeqlens = 4u,
};

inline uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(static_cast<const uint8_t*>(p) - hemu::g_smem);
}
inline uint8_t* smem_at(uint32_t a) { return hemu::g_smem + a; }

inline uint64_t globaltimer_ns() {
  return static_cast<uint64_t>(
      std::chrono::duration_cast<std::chrono::nanoseconds>(std::chrono::steady_clock::now().time_since_epoch())
          .count());
}

// ---------------------------------------------------------------- mbarrier
struct MbarState {
  uint32_t expected = 0, pending = 0;
  int64_t tx = 0;
  uint32_t phase = 0;
  bool init = false;
};
inline std::unordered_map<uint32_t, MbarState> g_mbars[hemu::kMaxCluster];  // per CTA, by smem offset

inline MbarState& mbar_state_at(int cta, uint32_t off) {
  MbarState& m = g_mbars[cta][off];
  if (!m.init) {
    std::fprintf(stderr, "tcsim: mbarrier at smem %u of CTA %d used before init\n", off, cta);
    ++hemu::g_errors;
    m.init = true;
    m.expected = m.pending = 1;
  }
  return m;
}
inline MbarState& mbar_state(const void* bar) { return mbar_state_at(hemu::g_cur_cta, smem_u32(bar)); }

inline void mbar_check_phase(MbarState& m) {
  if (m.pending == 0 && m.tx == 0) {
    ++m.phase;
    m.pending = m.expected;
  }
}

inline void mbar_init(uint64_t* bar, uint32_t count) {
  MbarState& m = g_mbars[hemu::g_cur_cta][smem_u32(bar)];
  m = MbarState{};
  m.init = true;
  m.expected = m.pending = count;
}
inline void fence_barrier_init() {}

inline void mbar_arrive_cta(int cta, uint32_t off) {
  MbarState& m = mbar_state_at(cta, off);
  if (m.pending == 0) {
    std::fprintf(stderr, "tcsim: arrival on a completed phase (smem %u of CTA %d)\n", off, cta);
    ++hemu::g_errors;
    return;
  }
  --m.pending;
  mbar_check_phase(m);
}
inline void mbar_arrive_at(uint64_t* bar) { mbar_arrive_cta(hemu::g_cur_cta, smem_u32(bar)); }
inline void mbar_complete_tx_cta(int cta, uint32_t off, uint32_t bytes) {
  MbarState& m = mbar_state_at(cta, off);
  m.tx -= bytes;
  mbar_check_phase(m);
}
inline void mbar_complete_tx(uint64_t* bar, uint32_t bytes) {
  mbar_complete_tx_cta(hemu::g_cur_cta, smem_u32(bar), bytes);
}

// shared::cluster addresses: mapa results carry the target CTA as (rank + 1) << 24; a plain
// shared::cta offset means the executing CTA.
inline uint32_t cluster_addr(uint32_t off, uint32_t rank) { return ((rank + 1u) << 24) | off; }
inline int cluster_cta(uint32_t a) { return (a >> 24) ? static_cast<int>((a >> 24) - 1u) : hemu::g_cur_cta; }
inline uint32_t cluster_off(uint32_t a) { return a & 0xFFFFFFu; }
inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  MbarState& m = mbar_state(bar);
  m.tx += bytes;
  mbar_arrive_at(bar);
}
inline void mbar_arrive(uint64_t* bar) { mbar_arrive_at(bar); }

inline void mma_flush_for(int cta, uint32_t off);
inline bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  mma_flush_for(hemu::g_cur_cta, smem_u32(bar));
  if ((mbar_state(bar).phase & 1u) != (parity & 1u)) return true;
  hemu::yield();
  return (mbar_state(bar).phase & 1u) != (parity & 1u);
}
inline bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t) { return mbar_try_wait(bar, parity); }

constexpr uint32_t kWaitSliceNs = 1000000;

inline bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, kWaitSliceNs)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// ---------------------------------------------------------------- TMA
struct HostTmap {
  const uint8_t* base;
  uint64_t inner, rows, stride;  // elements, rows, bytes per row
  uint32_t box_inner, box_rows, elem;
  uint64_t depth = 1, stride2 = 0;  // 3-D maps: extent and byte stride of the outer dimension
  uint32_t box_depth = 1;
};
static_assert(sizeof(HostTmap) <= sizeof(CUtensorMap), "tensor map model too large");

inline void prefetch_tensormap(const CUtensorMap*) {}

inline void tma_box_to_smem(void* dst, const CUtensorMap* map, int32_t x, int32_t y, int32_t z = 0);
inline void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x, int32_t y) {
  tma_box_to_smem(dst, map, x, y);
  const HostTmap* t = reinterpret_cast<const HostTmap*>(map);
  mbar_complete_tx(bar, t->box_rows * t->box_inner * t->elem);
}
// 3-D box: box_depth x box_rows rows (y fastest), zero fill outside the tensor in any dimension.
inline void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x, int32_t y, int32_t z) {
  const HostTmap* t = reinterpret_cast<const HostTmap*>(map);
  if (t->stride2 == 0) {
    std::fprintf(stderr, "tcsim: 3-D TMA load through a 2-D tensor map\n");
    ++hemu::g_errors;
  }
  tma_box_to_smem(dst, map, x, y, z);
  mbar_complete_tx(bar, t->box_depth * t->box_rows * t->box_inner * t->elem);
}
// Pair form: the box lands in this CTA's shared memory, its bytes count on the (leader's) barrier.
inline void tma_load_2d_pair_model(void* dst, const CUtensorMap* map, uint32_t bar, int32_t x, int32_t y) {
  tma_box_to_smem(dst, map, x, y);
  const HostTmap* t = reinterpret_cast<const HostTmap*>(map);
  mbar_complete_tx_cta(cluster_cta(bar), cluster_off(bar), t->box_rows * t->box_inner * t->elem);
}
inline void tma_box_to_smem(void* dst, const CUtensorMap* map, int32_t x, int32_t y, int32_t z) {
  const HostTmap* t = reinterpret_cast<const HostTmap*>(map);
  uint8_t* d = static_cast<uint8_t*>(dst);
  const uint32_t rb = t->box_inner * t->elem;
  if (rb != 128 || (x * t->elem) % 16 != 0) {
    std::fprintf(stderr, "tcsim: TMA box of %u bytes per row / x %d not 16-byte aligned\n", rb, x);
    ++hemu::g_errors;
  }
  if ((smem_u32(dst) & 1023u) != 0) {
    std::fprintf(stderr, "tcsim: 128-byte-swizzled TMA destination not 1024-byte aligned\n");
    ++hemu::g_errors;
  }
  for (uint32_t r = 0; r < t->box_rows * t->box_depth; ++r) {
    uint8_t row[128];
    const int64_t gy = static_cast<int64_t>(y) + r % t->box_rows;
    const int64_t gz = static_cast<int64_t>(z) + r / t->box_rows;
    for (uint32_t i = 0; i < t->box_inner; ++i) {
      const int64_t gx = static_cast<int64_t>(x) + i;
      if (gy < 0 || gy >= static_cast<int64_t>(t->rows) || gx < 0 || gx >= static_cast<int64_t>(t->inner) ||
          gz < 0 || gz >= static_cast<int64_t>(t->depth))
        std::memset(row + i * t->elem, 0, t->elem);
      else
        std::memcpy(row + i * t->elem, t->base + gz * t->stride2 + gy * t->stride + gx * t->elem, t->elem);
    }
    const uint32_t a = smem_u32(d + r * rb);
    for (uint32_t c = 0; c < 8; ++c) std::memcpy(d + r * rb + ((c ^ ((a >> 7) & 7u)) << 4), row + c * 16, 16);
  }
}

// tile::gather4: rows r0..r3 of the 64-element box column x land as four consecutive 128-byte rows at
// dst (swizzled by address; rows outside the tensor as zeros); their bytes complete on bar.
inline void tma_gather4_model(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x, int32_t r0, int32_t r1,
                              int32_t r2, int32_t r3) {
  const HostTmap* t = reinterpret_cast<const HostTmap*>(map);
  const int32_t rows[4] = {r0, r1, r2, r3};
  uint8_t* d = static_cast<uint8_t*>(dst);
  if (t->box_rows != 1 || t->box_inner * t->elem != 128 || (x * t->elem) % 16 != 0) {
    std::fprintf(stderr, "tcsim: gather4 needs a {64, 1} box and a 16-byte-aligned x\n");
    ++hemu::g_errors;
  }
  for (int i = 0; i < 4; ++i) {
    uint8_t row[128];
    for (uint32_t e = 0; e < t->box_inner; ++e) {
      const int64_t gx = static_cast<int64_t>(x) + e;
      if (rows[i] < 0 || rows[i] >= static_cast<int64_t>(t->rows) || gx >= static_cast<int64_t>(t->inner))
        std::memset(row + e * t->elem, 0, t->elem);
      else
        std::memcpy(row + e * t->elem, t->base + rows[i] * t->stride + gx * t->elem, t->elem);
    }
    const uint32_t a = smem_u32(d + i * 128);
    for (uint32_t c = 0; c < 8; ++c) std::memcpy(d + i * 128 + ((c ^ ((a >> 7) & 7u)) << 4), row + c * 16, 16);
  }
  mbar_complete_tx(bar, 4 * 128);
}

inline void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x, int32_t y, uint64_t) {
  tma_load_2d(dst, map, bar, x, y);
}
inline uint64_t policy_evict_first() { return 0; }
inline uint64_t policy_evict_last() { return 0; }

inline void tma_store_2d(const CUtensorMap* map, const void* src, int32_t x, int32_t y) {
  const HostTmap* t = reinterpret_cast<const HostTmap*>(map);
  const uint8_t* s = static_cast<const uint8_t*>(src);
  const uint32_t rb = t->box_inner * t->elem;
  for (uint32_t r = 0; r < t->box_rows; ++r) {
    uint8_t row[128];
    const uint32_t a = smem_u32(s + r * rb);
    for (uint32_t c = 0; c < 8; ++c) std::memcpy(row + c * 16, s + r * rb + ((c ^ ((a >> 7) & 7u)) << 4), 16);
    const int64_t gy = static_cast<int64_t>(y) + r;
    if (gy < 0 || gy >= static_cast<int64_t>(t->rows)) continue;
    for (uint32_t i = 0; i < t->box_inner; ++i) {
      const int64_t gx = static_cast<int64_t>(x) + i;
      if (gx >= 0 && gx < static_cast<int64_t>(t->inner))
        std::memcpy(const_cast<uint8_t*>(t->base) + gy * t->stride + gx * t->elem, row + i * t->elem, t->elem);
    }
  }
}
inline void tma_store_commit() {}
template <int N>
inline void tma_store_wait_read() {}
template <int N>
inline void tma_store_wait() {}
inline void fence_proxy_async_smem() {}

// ---------------------------------------------------------------- TMEM and MMA
inline uint32_t g_tmem_all[hemu::kMaxCluster][128][512];  // per CTA
inline uint32_t g_tmem_next[hemu::kMaxCluster] = {};

struct MmaOp {
  bool ts, pair;
  int cta;  // issuing CTA
  uint32_t d, a_tmem;
  uint64_t a, b;
  uint32_t idesc, acc;
};
inline std::vector<MmaOp> g_mma_queue;

inline void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  if (hemu::lin_tid() % 32 != 0) return;  // one allocation per warp
  uint32_t& next = g_tmem_next[hemu::g_cur_cta];
  if (next + ncols > 512) {
    std::fprintf(stderr, "tcsim: TMEM allocation beyond 512 columns\n");
    ++hemu::g_errors;
  }
  *dst_smem = next;
  next += ncols;
}
inline void tmem_relinquish() {}
inline void tmem_dealloc(uint32_t, uint32_t) {}
inline void tc_fence_before_sync() {}
inline void tc_fence_after_sync() {}

inline float f16_bits(uint16_t b, bool bf16) {
  if (bf16) {
    uint32_t u = static_cast<uint32_t>(b) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
  }
  __half_raw r;
  r.x = b;
  return __half2float(__half(r));
}

// Element (mn, k) of a 128-byte-swizzled operand described by desc (K-major: mn rows of 128 bytes in
// 8-row groups SBO apart; MN-major: k rows of 128 bytes holding 64 mn values, 8-row groups SBO apart,
// 64-value column blocks LBO apart).
inline float sdesc_elem(const uint8_t* base, uint64_t desc, bool mn_major, uint32_t mn, uint32_t k, bool bf16) {
  const uint32_t start = static_cast<uint32_t>(desc & 0x3FFFu) << 4;
  const uint32_t lbo = static_cast<uint32_t>((desc >> 16) & 0x3FFFu) << 4;
  const uint32_t sbo = static_cast<uint32_t>((desc >> 32) & 0x3FFFu) << 4;
  if (((desc >> 61) & 7u) != 2u || ((desc >> 46) & 1u) != 1u) {
    std::fprintf(stderr, "tcsim: descriptor without 128-byte swizzle or version bit\n");
    ++hemu::g_errors;
  }
  uint32_t a = mn_major ? start + (mn / 64) * lbo + (k / 8) * sbo + (k % 8) * 128 + (mn % 64) * 2
                        : start + (mn / 8) * sbo + (mn % 8) * 128 + k * 2;
  a ^= ((a >> 7) & 7u) << 4;
  uint16_t b;
  std::memcpy(&b, base + a, 2);
  return f16_bits(b, bf16);
}

inline void mma_execute(const MmaOp& op) {
  const uint32_t id = op.idesc;
  const bool a_bf16 = ((id >> 7) & 7u) == 1u, b_bf16 = ((id >> 10) & 7u) == 1u;
  const bool a_mn = (id >> 15) & 1u, b_mn = (id >> 16) & 1u;
  const uint32_t N = ((id >> 17) & 0x3Fu) << 3, M = ((id >> 24) & 0x1Fu) << 4;
  // single CTA: M = 128 rows in the issuer's TMEM and smem; pair (cta_group::2): M = 256, rows
  // 0..127 in CTA 0 and 128..255 in CTA 1 (A from each CTA's smem or TMEM, D into each CTA's TMEM),
  // B's N rows split in halves, the first from CTA 0's smem and the second from CTA 1's, at the same
  // descriptor address.
  const uint32_t Mc = op.pair ? 256u : 128u;
  if (((id >> 4) & 3u) != 1u || a_bf16 != b_bf16 || M != Mc || (a_mn && op.ts) || (op.pair && N % 16 != 0)) {
    std::fprintf(stderr, "tcsim: unsupported instruction descriptor %08x\n", id);
    ++hemu::g_errors;
    return;
  }
  const int c0 = op.pair ? 0 : op.cta;
  const uint32_t dl = op.d >> 16, dc = op.d & 0xFFFFu;
  const uint32_t al = op.a_tmem >> 16, ac = op.a_tmem & 0xFFFFu;
  static float A[256][16], B[256][16];
  for (uint32_t m = 0; m < M; ++m) {
    const int cta = c0 + static_cast<int>(m / 128);
    for (uint32_t k = 0; k < 16; ++k) {
      if (op.ts) {
        const uint32_t w = g_tmem_all[cta][al + m % 128][ac + k / 2];
        A[m][k] = f16_bits(static_cast<uint16_t>(k % 2 ? w >> 16 : w & 0xFFFFu), a_bf16);
      } else {
        A[m][k] = sdesc_elem(hemu::g_smem_cta[cta], op.a, a_mn, m % 128, k, a_bf16);
      }
    }
  }
  for (uint32_t n = 0; n < N; ++n) {
    const uint32_t half = op.pair ? N / 2 : N;
    const int cta = c0 + static_cast<int>(n / half);
    for (uint32_t k = 0; k < 16; ++k) B[n][k] = sdesc_elem(hemu::g_smem_cta[cta], op.b, b_mn, n % half, k, b_bf16);
  }
  for (uint32_t m = 0; m < M; ++m) {
    uint32_t (&T)[128][512] = g_tmem_all[c0 + static_cast<int>(m / 128)];
    for (uint32_t n = 0; n < N; ++n) {
      double s = 0.0;
      for (uint32_t k = 0; k < 16; ++k) s += static_cast<double>(A[m][k]) * B[n][k];
      float acc = 0.f;
      if (op.acc) std::memcpy(&acc, &T[dl + m % 128][dc + n], 4);
      acc = static_cast<float>(acc + s);
      std::memcpy(&T[dl + m % 128][dc + n], &acc, 4);
    }
  }
}

// A commit does not run its MMAs: they run, in issue order, when a thread first polls a barrier that
// one of the commits arrives on (the latest moment the hardware could finish them), or when the
// cluster's CTAs have all exited.  So an operand overwritten, or an accumulator read, before the
// commit's barrier has been waited on shows in the results.
struct PendingCommit {
  std::vector<MmaOp> ops;
  std::vector<std::pair<int, uint32_t>> targets;  // (CTA, barrier offset) arrivals
};
inline std::vector<PendingCommit> g_pending;

inline void mma_flush_upto(size_t n) {  // runs the first n pending commits
  for (size_t i = 0; i < n; ++i) {
    for (const MmaOp& op : g_pending[i].ops) mma_execute(op);
    for (const auto& t : g_pending[i].targets) mbar_arrive_cta(t.first, t.second);
  }
  g_pending.erase(g_pending.begin(), g_pending.begin() + static_cast<long>(n));
}
inline void mma_flush_for(int cta, uint32_t off) {
  size_t last = 0;
  for (size_t i = 0; i < g_pending.size(); ++i)
    for (const auto& t : g_pending[i].targets)
      if (t.first == cta && t.second == off) last = i + 1;
  if (last) mma_flush_upto(last);
}
inline void tc_commit(uint64_t* bar) {
  g_pending.push_back({std::move(g_mma_queue), {{hemu::g_cur_cta, smem_u32(bar)}}});
  g_mma_queue.clear();
}
// Pair commit with multicast: arrives on the barrier at the same offset in every CTA of the mask.
inline void tc_commit_multicast(uint64_t* bar, uint16_t mask) {
  PendingCommit pc{std::move(g_mma_queue), {}};
  g_mma_queue.clear();
  for (int c = 0; c < hemu::g_cluster; ++c)
    if ((mask >> c) & 1u) pc.targets.push_back({c, smem_u32(bar)});
  g_pending.push_back(std::move(pc));
}

__host__ __device__ constexpr uint32_t make_idesc_f32acc(uint32_t ab_bf16, uint32_t b_mn_major, uint32_t M,
                                                         uint32_t N) {
  return (1u << 4) | (ab_bf16 << 7) | (ab_bf16 << 10) | (b_mn_major << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

inline uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}
constexpr uint32_t kDescHiSw128Sbo1K = (1024u >> 4) | (1u << 14) | (2u << 29);
__host__ __device__ constexpr uint32_t sdesc_lo(uint32_t saddr, uint32_t lbo) {
  return ((saddr & 0x3FFFFu) >> 4) | (((lbo >> 4) & 0x3FFFu) << 16);
}

inline void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  g_mma_queue.push_back({false, false, hemu::g_cur_cta, d_tmem, 0, a_desc, b_desc, idesc, accumulate});
}
inline void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  g_mma_queue.push_back({true, false, hemu::g_cur_cta, d_tmem, a_tmem, 0, b_desc, idesc, accumulate});
}
inline void mma_ss_pair_model(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  if (hemu::g_cur_cta % 2 != 0) {
    std::fprintf(stderr, "tcsim: pair MMA issued by an odd CTA\n");
    ++hemu::g_errors;
  }
  g_mma_queue.push_back({false, true, hemu::g_cur_cta, d, 0, a, b, idesc, acc});
}
inline void mma_ts_pair_model(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  if (hemu::g_cur_cta % 2 != 0) {
    std::fprintf(stderr, "tcsim: pair MMA issued by an odd CTA\n");
    ++hemu::g_errors;
  }
  g_mma_queue.push_back({true, true, hemu::g_cur_cta, d, a_tmem, 0, b, idesc, acc});
}
inline void mma_ss_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc, uint32_t accumulate) {
  const uint64_t hi = static_cast<uint64_t>(kDescHiSw128Sbo1K) << 32;
  mma_ss(d_tmem, hi | a_lo, hi | b_lo, idesc, accumulate);
}
inline void mma_ts_lo(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t idesc, uint32_t accumulate) {
  mma_ts(d_tmem, a_tmem, (static_cast<uint64_t>(kDescHiSw128Sbo1K) << 32) | b_lo, idesc, accumulate);
}

inline uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) { return base + (lane << 16) + col; }

// tcgen05.ld / st are .sync.aligned: all 32 lanes of the warp execute each one together (a warp
// barrier here, which reports lanes that have exited).
inline void tmem_lane_check(uint32_t taddr) {
  hemu::syncwarp();
  const uint32_t w = hemu::lin_tid() / 32;
  if ((taddr >> 16) != 32 * (w % 4)) {
    std::fprintf(stderr, "tcsim: warp %u addresses TMEM lanes from %u\n", w, taddr >> 16);
    ++hemu::g_errors;
  }
}
inline void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_lane_check(taddr);
  const uint32_t lane = (taddr >> 16) + hemu::lin_tid() % 32, col = taddr & 0xFFFFu;
  for (int j = 0; j < 32; ++j) r[j] = g_tmem_all[hemu::g_cur_cta][lane][col + j];
}
inline void tmem_ld_wait(uint32_t (&)[32]) {}
inline void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  tmem_lane_check(taddr);
  const uint32_t lane = (taddr >> 16) + hemu::lin_tid() % 32, col = taddr & 0xFFFFu;
  for (int j = 0; j < 16; ++j) r[j] = g_tmem_all[hemu::g_cur_cta][lane][col + j];
}
inline void tmem_ld16_wait(uint32_t (&)[16]) {}
inline void reg_fence(uint32_t (&)[32]) {}
inline void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  tmem_lane_check(taddr);
  const uint32_t lane = (taddr >> 16) + hemu::lin_tid() % 32, col = taddr & 0xFFFFu;
  for (int j = 0; j < 32; ++j) g_tmem_all[hemu::g_cur_cta][lane][col + j] = r[j];
}
inline void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  tmem_lane_check(taddr);
  const uint32_t lane = (taddr >> 16) + hemu::lin_tid() % 32, col = taddr & 0xFFFFu;
  for (int j = 0; j < 16; ++j) g_tmem_all[hemu::g_cur_cta][lane][col + j] = r[j];
}
inline void tmem_st_wait() {}

// ---------------------------------------------------------------- warp-group helpers
inline void named_bar_sync(uint32_t id, uint32_t nthreads) { hemu::named_bar(static_cast<int>(id), nthreads, true); }
inline bool named_bar_and(uint32_t id, uint32_t nthreads, bool pred) {
  return hemu::named_bar(static_cast<int>(id), nthreads, pred);
}
template <uint32_t N>
inline void setmaxnreg_inc() {}
template <uint32_t N>
inline void setmaxnreg_dec() {}

inline void st_global_v8(void* dst, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4, uint32_t a5,
                         uint32_t a6, uint32_t a7) {
  const uint32_t v[8] = {a0, a1, a2, a3, a4, a5, a6, a7};
  std::memcpy(dst, v, 32);
}

inline void red_add_f32x4(float* p, float a, float b, float c, float d) {
  if (reinterpret_cast<uintptr_t>(p) & 15u) {
    std::fprintf(stderr, "emu: vector reduction at a misaligned address\n");
    std::abort();
  }
  p[0] += a;
  p[1] += b;
  p[2] += c;
  p[3] += d;
}

// ---------------------------------------------------------------- math helpers
inline float2 ffma2(float2 a, float2 b, float2 c) { return make_float2(std::fma(a.x, b.x, c.x), std::fma(a.y, b.y, c.y)); }
inline float2 fadd2(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
inline float fmax3(float a, float b, float c) { return std::fmax(a, std::fmax(b, c)); }
inline float ex2_approx(float x) { return exp2f(x); }
inline float2 unpack_bf16x2(uint32_t w) {
  const uint32_t lo = w << 16, hi = w & 0xffff0000u;
  float a, b;
  std::memcpy(&a, &lo, 4);
  std::memcpy(&b, &hi, 4);
  return make_float2(a, b);
}
inline uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  uint32_t u;
  std::memcpy(&u, &v, 4);
  return u;
}

// per-block state
inline bool g_tc_reset_registered = [] {
  hemu::g_block_reset.push_back([](int c) {
    g_mbars[c].clear();
    g_tmem_next[c] = 0;
    g_mma_queue.clear();
    g_pending.clear();
    std::memset(g_tmem_all[c], 0xFF, sizeof(g_tmem_all[c]));
  });
  return true;
}();

}  // namespace mimo
