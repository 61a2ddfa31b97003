// attn_fwd_pipelined.cuh -- warp-specialised, persistent tcgen05 attention
// forward for the MiMo-V2 sliding-window (sink) and global causal layers.
//
// Work unit: (sequence, 128-query tile, two query heads of one KV group).
// The two heads share every K/V tile and ping-pong on the tensor core: while
// one head's softmax runs on the CUDA cores, the other head's QK^T or PV runs
// on tcgen05.  CTAs are persistent (one per SM) and walk the units with a
// static stride; within a sequence, causal tiles go longest first.
//
// Shared memory, in 16 KB units (each unit is what one descriptor walk of an
// MMA operand covers; all are 128-byte swizzled):
//   Q region : 6 units = 2 heads x {dims 0..63 (rotated, FP16), 64..127, 128..191}
//              each unit = 128 query rows x 64 dims
//   K/V ring : 8 unit slots; every KV tile is 5 units, in this order:
//              K dims 0..63 (already rotated, FP16, from the RoPE pre-pass),
//              K dims 64..127, K dims 128..191 (128 keys x 64 dims each), then
//              V keys 0..63 and V keys 64..127 (64 keys x 128 dims each, stored
//              as two 8 KB halves: dims 0..63 then 64..127).
//   The ring is consumed and released in load order, so with 8 slots every
//   unit is requested about one KV-tile iteration before its first use.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each.  P_h (bf16)
// overwrites the first 64 columns of S_h and is the A operand of PV.
//
// Warp roles (16 warps, 512 threads):
//   warp 0      Q loader (TMA), per head as soon as that head's Q region frees
//   warp 1      MMA issuer (one thread) and TMEM owner
//   warp 2      K/V loader (TMA); runs ahead across units, bounded by the ring
//   warp 3      idle
//   warps 4-7   softmax + epilogue for the unit's first head (thread = query row = TMEM lane)
//   warps 8-11  softmax + epilogue for the second head
//   warps 12-15 RoPE for Q: rotates each head's rope unit in place, BF16 in,
//               FP16 out.  Each thread owns one row; its per-row angle offsets
//               r*theta_i live in registers, the tile-start angle is evaluated
//               once per frequency per unit.
//
// MMA issue order: one stream over all tiles of all units of the CTA,
//   S0(0) S1(0) | PV0(t) S0(t+1) PV1(t) S1(t+1) | ...
// where tile t+1 may be the first tile of the next unit; a head's Q region is
// released after its last S of a unit, so the next unit's Q loads and rotates
// while the current unit's softmax and PV finish.
#pragma once

#include "params.cuh"
#include "rope_smem.cuh"
#include "sm100.cuh"

namespace mimo {

namespace pipe {
constexpr int kThreads = 512;
constexpr uint32_t kUnit = 16384;
constexpr int kSlots = 8;
constexpr int kUnitsPerTile = 5;
constexpr uint32_t kQOff = 0;
constexpr uint32_t kRingOff = 6 * kUnit;
constexpr uint32_t kCtrlOff = kRingOff + kSlots * kUnit;  // 229376
constexpr uint32_t kCtrlBytes = 2048;
constexpr uint32_t kSmemBytes = kCtrlOff + kCtrlBytes;  // 231424 <= 232448
constexpr uint32_t kTmemCols = 512;
__host__ __device__ constexpr uint32_t col_s(int h) { return 128u * h; }        // S_h: columns [128h, 128h+128)
__host__ __device__ constexpr uint32_t col_o(int h) { return 256u + 128u * h; }  // O_h: columns [256+128h, ...)
constexpr uint32_t kIdescSF16 = make_idesc_f32acc(0, 0, 128, 128);
constexpr uint32_t kIdescSBF16 = make_idesc_f32acc(1, 0, 128, 128);
constexpr uint32_t kIdescPV = make_idesc_f32acc(1, 1, 128, 128);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 2^8 between rescales
constexpr uint32_t kRopeBarId = 1;
// Register split after setmaxnreg (per thread): 128 x ctl + 256 x softmax + 128 x rope <= 65536.
#ifndef MIMO_REGS_CTL
#define MIMO_REGS_CTL 96
#endif
#ifndef MIMO_REGS_SOFTMAX
#define MIMO_REGS_SOFTMAX 152
#endif
#ifndef MIMO_REGS_ROPE
#define MIMO_REGS_ROPE 112
#endif
constexpr uint32_t kRegsCtl = MIMO_REGS_CTL, kRegsSoftmax = MIMO_REGS_SOFTMAX, kRegsRope = MIMO_REGS_ROPE;
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax + 128 * kRegsRope <= 65536, "register split exceeds the launch");

constexpr int kMaxStagedSinks = 256;
struct Ctrl {
  uint64_t q_full[2], q_roped[2], q_empty[2];
  uint64_t slot_full[kSlots], slot_empty[kSlots];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint32_t tmem_base;
  int abort;
  long long total_tiles;  // query tiles over all sequences (filled by kernels that schedule by tile)
  double theta[kRopeDims / 2];
  float2 base_q[kRopeDims / 2];
  float sink[kMaxStagedSinks];  // sink logits staged once per CTA (when hq <= kMaxStagedSinks)
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block too large");
}  // namespace pipe

// Walks the static unit sequence of one CTA: unit u -> (sequence, query tile,
// head pair).  Tiles are numbered sequence by sequence; within a sequence they
// run in ascending order for the sliding window and descending order (longest
// first) for the causal layer.  Every role walks the same sequence.
struct UnitWalker {
  const int32_t* cu;
  int num_seqs, total_tokens, pairs;
  bool causal;
  int b = 0;
  int tile_base = 0;
  int ntiles = -1;
  int s_b = 0, L = 0;
  bool bad = false;

  __device__ __forceinline__ explicit UnitWalker(const FwdParams& P)
      : cu(P.cu_seqlens), num_seqs(P.num_seqs), total_tokens(P.total_tokens), pairs(P.hq / 2), causal(P.window < 0) {}

  __device__ __forceinline__ void reset() {
    b = 0;
    tile_base = 0;
    ntiles = -1;
  }

  __device__ __forceinline__ bool seek(long long ti) {
    while (b < num_seqs) {
      if (ntiles < 0) {
        const int s = __ldg(cu + b), e = __ldg(cu + b + 1);
        if (s < 0 || e < s || e > total_tokens) {  // inconsistent: skip the sequence
          bad = true;
          s_b = 0;
          L = 0;
        } else {
          s_b = s;
          L = e - s;
        }
        ntiles = (L + kBlockM - 1) / kBlockM;
      }
      if (ti < tile_base + ntiles) return true;
      tile_base += ntiles;
      ++b;
      ntiles = -1;
    }
    return false;
  }

  __device__ __forceinline__ bool unit(long long u, int& q0, int& h0) {
    // u < pairs x (query tiles + sequences) < 2^31 (the host bounds Hq x T); 32-bit division
    const uint32_t uu = static_cast<uint32_t>(u), np = static_cast<uint32_t>(pairs);
    const uint32_t ti = uu / np;
    if (!seek(ti)) return false;
    const int local = static_cast<int>(ti) - tile_base;
    const int qt = causal ? (ntiles - 1 - local) : local;
    q0 = qt * kBlockM;
    h0 = 2 * static_cast<int>(uu - ti * np);
    return true;
  }
};

// The units of one CTA as the pipelined kernel schedules them: unit blockIdx.x,
// then every gridDim.x-th unit after it.  Every role builds the same iterator.
struct StridedUnits {
  UnitWalker W;
  long long u;
  __device__ __forceinline__ StridedUnits(const FwdParams& P, const void*) : W(P), u(blockIdx.x) {}
  __device__ __forceinline__ bool next(int& q0, int& h0) {
    if (!W.unit(u, q0, h0)) return false;
    u += gridDim.x;
    return true;
  }
};

__device__ __forceinline__ void kv_range(const FwdParams& P, int q0, int& kt_lo, int& kt_hi) {
  kt_hi = q0 / kBlockN;
  kt_lo = 0;
  if (P.window >= 0) {
    const int lo_key = q0 - P.window;
    kt_lo = lo_key > 0 ? lo_key / kBlockN : 0;
  }
}

// Bounded wait that also gives up once another role has aborted.  (Kept
// inline: a called function would be shared by regions with different
// setmaxnreg budgets, which the register allocator cannot satisfy.)
__device__ __forceinline__ bool pwait_slow(pipe::Ctrl* C, uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, kWaitSliceNs)) return true;
    if (*reinterpret_cast<volatile int*>(&C->abort)) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *reinterpret_cast<volatile int*>(&C->abort) = 1;
      atomicOr(&g_mimo_error, kErrTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ bool pwait(pipe::Ctrl* C, uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  return pwait_slow(C, bar, parity, limit_ns);
}

// ---------------------------------------------------------------- MMA helpers
// S = Q K^T: 4 FP16 K-steps on the rotated unit, 8 BF16 K-steps on the two pass units.
// Descriptor low words address in 16-byte units: +2 per 32-byte K-step.
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint32_t q0, uint32_t q1, uint32_t q2, uint32_t k0,
                                        uint32_t k1, uint32_t k2) {
#pragma unroll
  for (int sub = 0; sub < 4; ++sub) mma_ss_lo(d_tmem, q0 + 2 * sub, k0 + 2 * sub, pipe::kIdescSF16, sub > 0 ? 1u : 0u);
#pragma unroll
  for (int sub = 0; sub < 4; ++sub) mma_ss_lo(d_tmem, q1 + 2 * sub, k1 + 2 * sub, pipe::kIdescSBF16, 1u);
#pragma unroll
  for (int sub = 0; sub < 4; ++sub) mma_ss_lo(d_tmem, q2 + 2 * sub, k2 + 2 * sub, pipe::kIdescSBF16, 1u);
}

// O (+)= P[:, 64 v .. 64 v + 63] V_v for one V unit (64 keys x 128 dims, MN-major):
// 4 K-steps of 16 keys (2 KB apart), dims 64..127 at LBO = 8 KB, 8-key groups at SBO = 1 KB.
__device__ __forceinline__ void issue_pv_half(uint32_t d_tmem, uint32_t p_tmem_half, uint32_t v_lo, bool first) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_ts_lo(d_tmem, p_tmem_half + kk * 8, v_lo + kk * (2048 >> 4), pipe::kIdescPV, (kk > 0 || !first) ? 1u : 0u);
}

// ---------------------------------------------------------------- RoPE helper
// Rotates one row's rope unit in place (BF16 -> FP16) with cos/sin of
// (tile start + r) * theta_i formed as base (tile start) x offset (r).
__device__ __forceinline__ float rope_row_rotate(uint8_t* unit_base, int r, const float2* __restrict__ base,
                                                 const float (&oc)[32], const float (&os)[32]) {
  uint8_t* row = unit_base + r * 128;
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4* plo = reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4));
    uint4* phi = reinterpret_cast<uint4*>(row + (((c + 4) ^ (r & 7)) << 4));
    const uint4 lo = *plo;
    const uint4 hi = *phi;
    const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lo);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hi);
    uint4 olo, ohi;
    __half2* ol = reinterpret_cast<__half2*>(&olo);
    __half2* oh = reinterpret_cast<__half2*>(&ohi);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(l2[e]);
      const float2 y = __bfloat1622float2(h2[e]);
      const int i0 = 8 * c + 2 * e;
      const float2 b0 = base[i0], b1 = base[i0 + 1];
      // cos/sin of (P0 + r) theta = (cb + i sb)(co + i so)
      const float c0 = b0.x * oc[i0] - b0.y * os[i0];
      const float s0 = b0.y * oc[i0] + b0.x * os[i0];
      const float c1 = b1.x * oc[i0 + 1] - b1.y * os[i0 + 1];
      const float s1 = b1.y * oc[i0 + 1] + b1.x * os[i0 + 1];
      const float a0 = x.x * c0 - y.x * s0;
      const float d0 = y.x * c0 + x.x * s0;
      const float a1 = x.y * c1 - y.y * s1;
      const float d1 = y.y * c1 + x.y * s1;
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a0), fabsf(d0)), fmaxf(fabsf(a1), fabsf(d1))));
      ol[e] = __floats2half2_rn(a0, a1);
      oh[e] = __floats2half2_rn(d0, d1);
    }
    *plo = olo;
    *phi = ohi;
  }
  return amax;
}

// ---------------------------------------------------------------- roles
namespace pipe {

__device__ __forceinline__ uint32_t kslot(uint32_t t, int i) { return (t * kUnitsPerTile + i) % kSlots; }
__device__ __forceinline__ uint32_t kphase(uint32_t t, int i) { return ((t * kUnitsPerTile + i) / kSlots) & 1; }

// Waits until tile t's three K units have landed.
__device__ __forceinline__ bool wait_k(Ctrl* C, uint32_t t, uint64_t lim) {
#pragma unroll
  for (int i = 0; i < 3; ++i)
    if (!pwait(C, &C->slot_full[kslot(t, i)], kphase(t, i), lim)) return false;
  tc_fence_after_sync();
  return true;
}

__device__ __forceinline__ void mma_s(uint32_t tmem, uint32_t qdesc, uint32_t rdesc_k, uint32_t t, int h) {
  constexpr uint32_t kStep = kUnit >> 4;
  const uint32_t qh = qdesc + 3 * h * kStep;
  issue_s(tmem + col_s(h), qh, qh + kStep, qh + 2 * kStep, rdesc_k + kslot(t, 0) * kStep,
          rdesc_k + kslot(t, 1) * kStep, rdesc_k + kslot(t, 2) * kStep);
}

__device__ __forceinline__ void mma_pv(uint32_t tmem, uint32_t rdesc_v, uint32_t t, int h, bool first_tile) {
  constexpr uint32_t kStep = kUnit >> 4;
  issue_pv_half(tmem + col_o(h), tmem + col_s(h), rdesc_v + kslot(t, 3) * kStep, first_tile);
  issue_pv_half(tmem + col_o(h), tmem + col_s(h) + 32, rdesc_v + kslot(t, 4) * kStep, false);
}

__device__ __forceinline__ int unit_tiles(const FwdParams& P, int q0) {
  int kt_lo, kt_hi;
  kv_range(P, q0, kt_lo, kt_hi);
  return kt_hi - kt_lo + 1;
}

template <class Units>
__device__ void role_q_loader(uint8_t* smem, Ctrl* C, const CUtensorMap* tm_q, const FwdParams& P) {
  Units U(P, C);
  const UnitWalker& W = U.W;
  int q0, h0;
  for (uint32_t n_u = 0; U.next(q0, h0); ++n_u) {
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      if (n_u > 0 && !pwait(C, &C->q_empty[h], (n_u - 1) & 1, P.wait_limit_ns)) return;
      mbar_arrive_expect_tx(&C->q_full[h], 3 * kUnit);
#pragma unroll
      for (int c = 0; c < 3; ++c)
        tma_load_2d(smem + kQOff + (3 * h + c) * kUnit, tm_q, &C->q_full[h], (h0 + h) * kHeadDimQK + 64 * c,
                    W.s_b + q0);
    }
  }
  if (W.bad) atomicOr(&g_mimo_error, kErrSeqlens);
}

__device__ void role_kv_loader(uint8_t* smem, Ctrl* C, const CUtensorMap* tm_kr, const CUtensorMap* tm_k,
                               const CUtensorMap* tm_v, const FwdParams& P) {
  UnitWalker W(P);
  int q0, h0;
  uint32_t n = 0;
  for (long long u = blockIdx.x; W.unit(u, q0, h0); u += gridDim.x) {
    const int g = h0 / P.group;
    int kt_lo, kt_hi;
    kv_range(P, q0, kt_lo, kt_hi);
    for (int kt = kt_lo; kt <= kt_hi; ++kt) {
      const int row = W.s_b + kt * kBlockN;
#pragma unroll 1
      for (int i = 0; i < kUnitsPerTile; ++i, ++n) {
        const uint32_t slot = n % kSlots;
        if (n >= kSlots && !pwait(C, &C->slot_empty[slot], ((n / kSlots) - 1) & 1, P.wait_limit_ns)) return;
        uint8_t* dst = smem + kRingOff + slot * kUnit;
        mbar_arrive_expect_tx(&C->slot_full[slot], kUnit);
        if (i == 0) {
          tma_load_2d(dst, tm_kr, &C->slot_full[slot], g * kRopeDims, row);  // rotated FP16 rope dims
        } else if (i < 3) {
          tma_load_2d(dst, tm_k, &C->slot_full[slot], g * kHeadDimQK + 64 * i, row);
        } else {
          const int r0 = row + 64 * (i - 3);
          tma_load_2d(dst, tm_v, &C->slot_full[slot], g * kHeadDimV, r0);
          tma_load_2d(dst + kUnit / 2, tm_v, &C->slot_full[slot], g * kHeadDimV + 64, r0);
        }
      }
    }
  }
}

__device__ void role_mma(uint8_t* smem, Ctrl* C, uint32_t tmem, const FwdParams& P) {
  const uint64_t lim = P.wait_limit_ns;
  const uint32_t qdesc = sdesc_lo(smem_u32(smem + kQOff), 16);
  const uint32_t rdesc_k = sdesc_lo(smem_u32(smem + kRingOff), 16);
  const uint32_t rdesc_v = sdesc_lo(smem_u32(smem + kRingOff), kUnit / 2);
  UnitWalker W(P);
  int q0, h0;
  long long u = blockIdx.x;
  if (!W.unit(u, q0, h0)) return;
  int ntile = unit_tiles(P, q0);
  uint32_t n_u = 0, t = 0;
  int j = 0;
  // S of the very first tile
  if (!pwait(C, &C->q_roped[0], 0, lim) || !wait_k(C, 0, lim)) return;
  mma_s(tmem, qdesc, rdesc_k, 0, 0);
  tc_commit(&C->s_full[0]);
  if (ntile == 1) tc_commit(&C->q_empty[0]);
  if (!pwait(C, &C->q_roped[1], 0, lim)) return;
  tc_fence_after_sync();
  mma_s(tmem, qdesc, rdesc_k, 0, 1);
  tc_commit(&C->s_full[1]);
#pragma unroll
  for (int i = 0; i < 3; ++i) tc_commit(&C->slot_empty[kslot(0, i)]);
  if (ntile == 1) tc_commit(&C->q_empty[1]);
  while (true) {
    // the tile after t: the next one of this unit, or the first one of the next unit
    bool has_next, next_first = false, next_last = false;
    int next_ntile = ntile;
    if (j + 1 < ntile) {
      has_next = true;
      next_last = (j + 1 == ntile - 1);
    } else {
      int nq0, nh0;
      has_next = W.unit(u + gridDim.x, nq0, nh0);
      if (has_next) {
        next_ntile = unit_tiles(P, nq0);
        next_first = true;
        next_last = (next_ntile == 1);
      }
    }
    const uint32_t next_nu = next_first ? n_u + 1 : n_u;
    const bool first = (j == 0), last = (j == ntile - 1);
    if (!pwait(C, &C->slot_full[kslot(t, 3)], kphase(t, 3), lim)) return;
    if (!pwait(C, &C->slot_full[kslot(t, 4)], kphase(t, 4), lim)) return;
    // head 0: PV(t), then S(t+1)
    if (!pwait(C, &C->p_full[0], t & 1, lim)) return;
    if (first && n_u > 0 && !pwait(C, &C->o_empty[0], (n_u - 1) & 1, lim)) return;
    tc_fence_after_sync();
    mma_pv(tmem, rdesc_v, t, 0, first);
    if (last) tc_commit(&C->o_full[0]);
    if (has_next) {
      if (next_first && !pwait(C, &C->q_roped[0], next_nu & 1, lim)) return;
      if (!wait_k(C, t + 1, lim)) return;
      mma_s(tmem, qdesc, rdesc_k, t + 1, 0);
      tc_commit(&C->s_full[0]);
      if (next_last) tc_commit(&C->q_empty[0]);
    }
    // head 1: PV(t), then S(t+1)
    if (!pwait(C, &C->p_full[1], t & 1, lim)) return;
    if (first && n_u > 0 && !pwait(C, &C->o_empty[1], (n_u - 1) & 1, lim)) return;
    tc_fence_after_sync();
    mma_pv(tmem, rdesc_v, t, 1, first);
    tc_commit(&C->slot_empty[kslot(t, 3)]);
    tc_commit(&C->slot_empty[kslot(t, 4)]);
    if (last) tc_commit(&C->o_full[1]);
    if (!has_next) break;
    if (next_first && !pwait(C, &C->q_roped[1], next_nu & 1, lim)) return;
    tc_fence_after_sync();
    mma_s(tmem, qdesc, rdesc_k, t + 1, 1);
    tc_commit(&C->s_full[1]);
#pragma unroll
    for (int i = 0; i < 3; ++i) tc_commit(&C->slot_empty[kslot(t + 1, i)]);
    if (next_last) tc_commit(&C->q_empty[1]);
    ++t;
    if (next_first) {
      u += gridDim.x;
      ++n_u;
      ntile = next_ntile;
      j = 0;
    } else {
      ++j;
    }
  }
}

// Softmax + epilogue for head hw (0/1) of every unit; thread r of the warpgroup owns query row r.
__device__ void role_softmax(Ctrl* C, uint32_t tmem, const FwdParams& P, int hw, int r, int wq) {
  const uint64_t lim = P.wait_limit_ns;
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t tS = tmem + lane_base + col_s(hw);
  const uint32_t tO = tmem + lane_base + col_o(hw);
  const float sl2 = P.scale_log2;
  UnitWalker W(P);
  int q0, h0;
  uint32_t n_u = 0, n_t = 0;
  for (long long u = blockIdx.x; W.unit(u, q0, h0); u += gridDim.x, ++n_u) {
    const int head = h0 + hw;
    int kt_lo, kt_hi;
    kv_range(P, q0, kt_lo, kt_hi);
    float m = -INFINITY, l = 0.f;  // m in log2 units (scores x log2(e)/sqrt(d))
    if (P.sink != nullptr) {
      m = (P.hq <= kMaxStagedSinks ? C->sink[head] : __ldg(P.sink + head)) * kLog2e;
      l = 1.f;
    }
    for (int kt = kt_lo; kt <= kt_hi; ++kt, ++n_t) {
      if (!pwait(C, &C->s_full[hw], n_t & 1, lim)) return;
      tc_fence_after_sync();
      uint32_t s[4][32];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(tS + 32 * q, s[q]);
      tmem_ld_wait(s[0]);
      reg_fence(s[1]);
      reg_fence(s[2]);
      reg_fence(s[3]);
      // key column c is allowed iff d - window <= c <= d (d = query pos - tile's first key pos).
      // The allowed columns form one contiguous run [c_lo, c_hi]; masking uses a 32-bit run mask
      // per chunk, and the row max uses 8 independent accumulators (short dependency chains).
      const int d = q0 - kt * kBlockN + r;
      const int c_hi = min(d, kBlockN - 1);
      const int c_lo = (P.window >= 0) ? max(d - P.window, 0) : 0;
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
      if (c_lo == 0 && c_hi == kBlockN - 1) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            mx[(i >> 1) & 7] = fmax3(mx[(i >> 1) & 7], __uint_as_float(s[q][i]), __uint_as_float(s[q][i + 1]));
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int lo = c_lo - 32 * q, hi = c_hi - 32 * q;  // run relative to this chunk
          uint32_t run = 0u;
          if (hi >= 0 && lo <= 31 && lo <= hi) {
            const uint32_t upto = (hi >= 31) ? 0xffffffffu : ((2u << hi) - 1u);
            const uint32_t below = (lo <= 0) ? 0u : ((1u << lo) - 1u);
            run = upto & ~below;
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float x = ((run >> i) & 1u) ? __uint_as_float(s[q][i]) : -INFINITY;
            s[q][i] = __float_as_uint(x);
            mx[i & 7] = fmaxf(mx[i & 7], x);
          }
        }
      }
      float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      mt *= sl2;
      // lazy rescale: keep the running max unless it grows by more than the threshold
      const bool grow = mt > m + kRescaleThreshold;
      const float m_new = grow ? mt : m;
      const float corr = grow ? ex2_approx(m - m_new) : 1.f;  // m = -inf -> 0
      const float base = (m_new == -INFINITY) ? 0.f : m_new;
      // P = exp2(s * scale - m) as bf16 pairs, stored 32 keys (16 columns) at a time as S registers retire;
      // the scale-and-shift and the row sum run two lanes per instruction
      const float2 sl = make_float2(sl2, sl2), nb = make_float2(-base, -base);
      float2 sm[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) sm[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 x = ffma2(make_float2(__uint_as_float(s[q][i]), __uint_as_float(s[q][i + 1])), sl, nb);
          const float p0 = ex2_approx(x.x);
          const float p1 = ex2_approx(x.y);
          sm[(i >> 1) & 3] = fadd2(sm[(i >> 1) & 3], make_float2(p0, p1));
          pk[i >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + 16 * q, pk);
      }
      l = l * corr + (((sm[0].x + sm[0].y) + (sm[1].x + sm[1].y)) + ((sm[2].x + sm[2].y) + (sm[3].x + sm[3].y)));
      m = m_new;
      if (kt != kt_lo && __any_sync(0xffffffffu, grow)) {
        // rescale O; the previous PV has completed (it was issued before this tile's S)
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * q, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
          tmem_st32(tO + 32 * q, o);
        }
      }
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(&C->p_full[hw]);
    }
    // epilogue
    if (!pwait(C, &C->o_full[hw], n_u & 1, lim)) return;
    tc_fence_after_sync();
    uint32_t o[4][32];
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld32(tO + 32 * q, o[q]);
    tmem_ld_wait(o[0]);
    reg_fence(o[1]);
    reg_fence(o[2]);
    reg_fence(o[3]);
    tc_fence_before_sync();
    mbar_arrive(&C->o_empty[hw]);
    const int p = q0 + r;
    if (p < W.L) {
      const float inv = P.v_scale / l;
      uint16_t* dst = P.out + (static_cast<size_t>(W.s_b + p) * P.hq + head) * kHeadDimV;
#pragma unroll
      for (int qd = 0; qd < 8; ++qd) {  // 16 dims (32 bytes) per store
        const int q = qd >> 1, i = (qd & 1) * 16;
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[q][i + 2 * e]) * inv, __uint_as_float(o[q][i + 2 * e + 1]) * inv);
        st_global_v8(dst + 16 * qd, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
      }
      P.lse[static_cast<size_t>(head) * P.total_tokens + W.s_b + p] = (m + log2f(l)) * kLn2;
    }
  }
}

// RoPE warpgroup: thread r owns row r of each head's Q rope unit.
template <class Units>
__device__ void role_rope(uint8_t* smem, Ctrl* C, const FwdParams& P, int r) {
  const uint64_t lim = P.wait_limit_ns;
  float oc[32], os[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) rope_sincos(r, C->theta[i], os[i], oc[i]);
  float amax = 0.f;
  Units U(P, C);
  int q0, h0;
  bool ok = true;
  for (uint32_t n_u = 0; ok && U.next(q0, h0); ++n_u) {
    if (r < 32) {
      float sn, cs;
      rope_sincos(q0, C->theta[r], sn, cs);
      C->base_q[r] = make_float2(cs, sn);
    }
    named_bar_sync(kRopeBarId, 128);
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      const bool got = pwait(C, &C->q_full[h], n_u & 1, lim);
      if (got) {
        amax = fmaxf(amax, rope_row_rotate(smem + kQOff + 3 * h * kUnit, r, C->base_q, oc, os));
        fence_proxy_async_smem();
      }
      ok = named_bar_and(kRopeBarId, 128, got);  // every thread leaves together once any wait fails
      if (!ok) break;
      if (r == 0) mbar_arrive(&C->q_roped[h]);
    }
  }
  if (amax > 65504.f) atomicOr(&g_mimo_error, kErrRange);
}

}  // namespace pipe

// ---------------------------------------------------------------- kernel
__global__ void __launch_bounds__(pipe::kThreads, 1)
    attn_fwd_pipelined_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kr,
                              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                              const __grid_constant__ FwdParams P) {
  using namespace pipe;
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctrl* C = reinterpret_cast<Ctrl*>(smem + kCtrlOff);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // A recorded timeout makes later launches skip their work until the host clears it.
  int skip = 0;
  if (tid == 0) {
    skip = (*reinterpret_cast<volatile unsigned int*>(&g_mimo_error) & kErrTimeout) != 0;
    if (smem_u32(smem) & 1023u) skip = 1;  // swizzled units need a 1 KB aligned base
  }
  if (__syncthreads_or(skip)) return;

  if (tid == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_kr);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&C->q_full[h], 1);
      mbar_init(&C->q_roped[h], 1);
      mbar_init(&C->q_empty[h], 1);
      mbar_init(&C->s_full[h], 1);
      mbar_init(&C->p_full[h], 128);
      mbar_init(&C->o_full[h], 1);
      mbar_init(&C->o_empty[h], 128);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&C->slot_full[s], 1);
      mbar_init(&C->slot_empty[s], 1);
    }
    C->abort = 0;
#pragma unroll
    for (int i = 0; i < kRopeDims / 2; ++i) C->theta[i] = P.theta[i];
    fence_barrier_init();
  }
  if (P.sink != nullptr && P.hq <= kMaxStagedSinks)
    for (int h = tid; h < P.hq; h += kThreads) C->sink[h] = __ldg(P.sink + h);
  if (warp == 1) {
    tmem_alloc(&C->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = C->tmem_base;

  if (warp < 4) {
    setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      if (warp == 0) role_q_loader<StridedUnits>(smem, C, &tm_q, P);
      else if (warp == 1) role_mma(smem, C, tmem, P);
      else if (warp == 2) role_kv_loader(smem, C, &tm_kr, &tm_k, &tm_v, P);
    }
  } else if (warp < 12) {
    setmaxnreg_inc<kRegsSoftmax>();
    const int hw = (warp - 4) >> 2;
    role_softmax(C, tmem, P, hw, tid - 128 * (1 + hw), warp & 3);
  } else {
    setmaxnreg_dec<kRegsRope>();
    role_rope<StridedUnits>(smem, C, P, tid - 384);
  }
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mimo
