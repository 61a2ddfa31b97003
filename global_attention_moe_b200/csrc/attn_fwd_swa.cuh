// attn_fwd_swa.cuh -- sliding-window kernel for windows of at most 128 keys
// (the MiMo-V2 sliding-window layer: the query plus 128 previous keys).
//
// Query tiles are 128 rows aligned to sequence starts, so with window <= 128 a
// tile's keys lie in at most two 128-key tiles: the "left" tile (keys
// q0-128 .. q0-1) and the "diagonal" tile (keys q0 .. q0+127).  Every query
// row's allowed keys form one contiguous run of those 256 keys.  Each head
// therefore computes both S tiles up front into a 256-column TMEM region and
// runs a single softmax pass over the 256 keys: no online rescale between
// tiles and no second S -> softmax -> PV round trip.  32-key chunks that lie
// outside every row of a warp are skipped (no TMEM load, no exponentials;
// P = 0 where PV reads it).
//
// TMEM, 256 columns per head (two heads ping-pong in 512 columns):
//   while S is live : S_left (fp32) at 0..127, S_diag (fp32) at 128..255
//   after softmax   : P_left (bf16 pairs) at 0..63, O (fp32) at 64..191,
//                     P_diag (bf16 pairs) at 192..255
// The softmax reads all of S into registers before it writes P, and PV
// (which writes O) waits for every row's P, so the overlays never race.
//
// Scheduling: units are ordered head pair by head pair, query tiles in order
// within each pair, and every CTA takes one contiguous block of that order.
// Consecutive units of a CTA are then usually consecutive query tiles of the
// same sequence and head pair, and the diagonal K/V tile of one unit is the
// left tile of the next: it stays in the ring and only one new K/V tile is
// loaded per unit (half the shared-memory fill of loading both).
//
// Shared memory, the K/V ring, the Q loader and the RoPE warpgroup are those
// of the pipelined kernel.  Per unit, the MMA issuer runs
//   S_0(left) S_0(diag) S_1(left) S_1(diag) | PV_0 | PV_1
// and releases each head's Q region right after that head's S, so the next
// unit's Q loads and rotates while this unit's softmax, PV and epilogue run.
// A K/V tile's units go back to the ring after the S (K) or PV (V) of the
// last unit that reads it, which is the order they were loaded in.
#pragma once

#include "attn_fwd_pipelined.cuh"

namespace mimo {
namespace swa {

using namespace pipe;

constexpr uint32_t kRegion = 256;  // TMEM columns per head
__host__ __device__ constexpr uint32_t region(int h) { return kRegion * h; }
constexpr uint32_t kColPLeft = 0, kColO = 64, kColPDiag = 192, kColSDiag = 128;

// Bits lo..hi of a 32-bit chunk (bounds relative to the chunk; empty when lo > hi).
__device__ __forceinline__ uint32_t run_mask(int lo, int hi) {
  if (hi < 0 || lo > 31 || lo > hi) return 0u;
  const uint32_t upto = (hi >= 31) ? 0xffffffffu : ((2u << hi) - 1u);
  const uint32_t below = (lo <= 0) ? 0u : ((1u << lo) - 1u);
  return upto & ~below;
}

// The units of one CTA in the window kernel's order: unit u is query tile
// u % tiles of head pair u / tiles (tiles = query tiles over all sequences),
// and CTA c takes units [c U / G, (c+1) U / G) of the U = pairs x tiles.  The
// position advances incrementally (no division per unit): the single-thread
// roles share issue slots with the softmax warps.
struct BlockUnits {
  UnitWalker W;
  uint32_t left;      // units still to visit
  uint32_t ti, pair;  // position of the next unit
  uint32_t tiles;
  __device__ __forceinline__ BlockUnits(const FwdParams& P, const Ctrl* C)
      : W(P), tiles(static_cast<uint32_t>(C->total_tiles)) {
    const uint64_t units = static_cast<uint64_t>(P.hq / 2) * tiles;
    const uint64_t u0 = units * blockIdx.x / gridDim.x, u1 = units * (blockIdx.x + 1) / gridDim.x;
    left = static_cast<uint32_t>(u1 - u0);
    pair = tiles ? static_cast<uint32_t>(u0 / tiles) : 0u;
    ti = tiles ? static_cast<uint32_t>(u0 % tiles) : 0u;
  }
  // After a call, W describes the returned unit's sequence (b, s_b, L) until the next call.
  __device__ __forceinline__ bool next(int& q0, int& h0) {
    if (left == 0) return false;
    if (ti == tiles) {  // next head pair: walk the sequences again
      ti = 0;
      ++pair;
      W.reset();
    }
    if (!W.seek(ti)) return false;
    q0 = static_cast<int>(ti - W.tile_base) * kBlockM;
    h0 = 2 * static_cast<int>(pair);
    --left;
    ++ti;
    return true;
  }
};

// Where a unit's K/V tiles sit in the CTA's stream of loaded tiles.
struct UnitTiles {
  int b = -1, h0 = -1, q0 = -1;  // the previous unit
  uint32_t n_t = 0;              // tiles loaded so far
  uint32_t t_left = 0, t_diag = 0;
  int ntile = 0;
  bool reuse = false;  // the left tile is the previous unit's diagonal tile, already loaded

  // Advances to unit (b, h0, q0); returns how many tiles it loads.
  __device__ __forceinline__ int advance(const FwdParams& P, int b_, int h0_, int q0_) {
    ntile = unit_tiles(P, q0_);
    reuse = ntile == 2 && b_ == b && h0_ == h0 && q0_ == q0 + kBlockM;
    if (reuse) {
      t_left = t_diag;
      t_diag = n_t;
    } else {
      t_left = n_t;
      t_diag = n_t + ntile - 1;
    }
    const int loads = reuse ? 1 : ntile;
    n_t += loads;
    b = b_;
    h0 = h0_;
    q0 = q0_;
    return loads;
  }
};

// The next unit re-reads this unit's diagonal tile as its left tile.
__device__ __forceinline__ bool next_reuses(const FwdParams& P, int b, int h0, int q0, bool has_next, int nb,
                                            int nh0, int nq0) {
  return has_next && nb == b && nh0 == h0 && nq0 == q0 + kBlockM && unit_tiles(P, nq0) == 2;
}

// Number of query tiles over all sequences (one warp).  Sequences whose bounds
// are inconsistent count as empty, as UnitWalker treats them, and are reported
// in the error word here: the walkers of this kernel may never reach them.
__device__ __forceinline__ long long count_tiles(const FwdParams& P, int lane) {
  long long acc = 0;
  bool bad = false;
  for (int b = lane; b < P.num_seqs; b += 32) {
    const int s = __ldg(P.cu_seqlens + b), e = __ldg(P.cu_seqlens + b + 1);
    const bool ok = s >= 0 && e >= s && e <= P.total_tokens;
    bad |= !ok;
    acc += ok ? (e - s + kBlockM - 1) / kBlockM : 0;
  }
  if (bad) atomicOr(&g_mimo_error, kErrSeqlens);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

__device__ void role_kv_loader(uint8_t* smem, Ctrl* C, const CUtensorMap* tm_kr, const CUtensorMap* tm_k,
                               const CUtensorMap* tm_v, const FwdParams& P) {
  BlockUnits U(P, C);
  UnitTiles T;
  int q0, h0;
  uint32_t n = 0;
  while (U.next(q0, h0)) {
    const int g = h0 / P.group;
    const int loads = T.advance(P, U.W.b, h0, q0);
    const int kt_hi = q0 / kBlockN;
#pragma unroll 1
    for (int kt = kt_hi - loads + 1; kt <= kt_hi; ++kt) {
      const int row = U.W.s_b + kt * kBlockN;
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
  constexpr uint32_t kStep = kUnit >> 4;
  BlockUnits U(P, C), Un(P, C);  // Un runs one unit ahead
  UnitTiles T;
  int q0, h0, nq0 = 0, nh0 = 0;
  bool has_next = Un.next(nq0, nh0);
  for (uint32_t n_u = 0; U.next(q0, h0); ++n_u) {
    const int b = U.W.b;
    T.advance(P, b, h0, q0);
    has_next = has_next && Un.next(nq0, nh0);  // Un now holds the unit after this one
    const bool keep = next_reuses(P, b, h0, q0, has_next, Un.W.b, nh0, nq0);
    const int ntile = T.ntile;  // 1 (first tile of a sequence, or window 0) or 2
    // S for both heads: the left tile (resident when reused) before the diagonal one
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      if (!pwait(C, &C->q_roped[h], n_u & 1, lim)) return;
      if (n_u > 0 && !pwait(C, &C->o_empty[h], (n_u - 1) & 1, lim)) return;  // previous O read out
      tc_fence_after_sync();
      const uint32_t qh = qdesc + 3 * h * kStep;
#pragma unroll 1
      for (int j = 2 - ntile; j < 2; ++j) {  // j = 0: left tile, j = 1: diagonal tile
        const uint32_t t = j ? T.t_diag : T.t_left;
        if (h == 0 && !(j == 0 && T.reuse) && !wait_k(C, t, lim)) return;
        issue_s(tmem + region(h) + (j ? kColSDiag : 0u), qh, qh + kStep, qh + 2 * kStep,
                rdesc_k + kslot(t, 0) * kStep, rdesc_k + kslot(t, 1) * kStep, rdesc_k + kslot(t, 2) * kStep);
      }
      tc_commit(&C->s_full[h]);
      tc_commit(&C->q_empty[h]);
    }
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      if (ntile == 2) tc_commit(&C->slot_empty[kslot(T.t_left, i)]);
      if (!keep) tc_commit(&C->slot_empty[kslot(T.t_diag, i)]);
    }
    // PV for both heads: O (columns 64..191) from P_left (0..63) and P_diag (192..255)
#pragma unroll 1
    for (int j = 2 - ntile; j < 2; ++j) {
      if (j == 0 && T.reuse) continue;  // V of a reused tile was waited for by the previous unit
      const uint32_t t = j ? T.t_diag : T.t_left;
      if (!pwait(C, &C->slot_full[kslot(t, 3)], kphase(t, 3), lim)) return;
      if (!pwait(C, &C->slot_full[kslot(t, 4)], kphase(t, 4), lim)) return;
    }
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      if (!pwait(C, &C->p_full[h], n_u & 1, lim)) return;
      tc_fence_after_sync();
      const uint32_t o = tmem + region(h) + kColO;
#pragma unroll 1
      for (int j = 2 - ntile; j < 2; ++j) {
        const uint32_t t = j ? T.t_diag : T.t_left;
        const uint32_t pc = tmem + region(h) + (j ? kColPDiag : kColPLeft);
        issue_pv_half(o, pc, rdesc_v + kslot(t, 3) * kStep, j == 2 - ntile);
        issue_pv_half(o, pc + 32, rdesc_v + kslot(t, 4) * kStep, false);
      }
      tc_commit(&C->o_full[h]);
    }
#pragma unroll
    for (int i = 3; i < 5; ++i) {
      if (ntile == 2) tc_commit(&C->slot_empty[kslot(T.t_left, i)]);
      if (!keep) tc_commit(&C->slot_empty[kslot(T.t_diag, i)]);
    }
  }
}

// Running max of one 32-key chunk over the keys in `run` (8 independent accumulators).
__device__ __forceinline__ void chunk_max(const uint32_t (&x)[32], uint32_t run, float (&mx)[8]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) mx[i & 7] = fmaxf(mx[i & 7], ((run >> i) & 1u) ? __uint_as_float(x[i]) : -INFINITY);
}

// P = exp2(s * scale_log2 - base) for one chunk, as 16 bf16 pairs; keys outside `run` give 0.
__device__ __forceinline__ void chunk_exp(const uint32_t (&x)[32], uint32_t run, float sl2, float base,
                                         float (&sm)[8], uint32_t (&pk)[16]) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    float p0 = ex2_approx(fmaf(__uint_as_float(x[i]), sl2, -base));
    float p1 = ex2_approx(fmaf(__uint_as_float(x[i + 1]), sl2, -base));
    p0 = ((run >> i) & 1u) ? p0 : 0.f;
    p1 = ((run >> (i + 1)) & 1u) ? p1 : 0.f;
    sm[i & 7] += p0;
    sm[(i + 1) & 7] += p1;
    pk[i >> 1] = pack_bf16x2(p0, p1);
  }
}

// Loads chunks 2*cp and 2*cp+1 (64 columns) of the 256-column span.
__device__ __forceinline__ void ld_pair(uint32_t tR, int cp, uint32_t (&s)[2][32]) {
  tmem_ld32(tR + 64 * cp, s[0]);
  tmem_ld32(tR + 64 * cp + 32, s[1]);
  tmem_ld_wait(s[0]);
  reg_fence(s[1]);
}

// Softmax + epilogue for head hw (0/1) of every unit; thread r of the warpgroup owns query row r.
__device__ void role_softmax(Ctrl* C, uint32_t tmem, const FwdParams& P, int hw, int r, int wq) {
  const uint64_t lim = P.wait_limit_ns;
  const uint32_t tR = tmem + (static_cast<uint32_t>(wq * 32) << 16) + region(hw);
  const float sl2 = P.scale_log2;
  BlockUnits U(P, C);
  const UnitWalker& W = U.W;
  int q0, h0;
  for (uint32_t n_u = 0; U.next(q0, h0); ++n_u) {
    const int head = h0 + hw;
    const int ntile = unit_tiles(P, q0);
    // Column c of the 256-key span holds key q0 - 128 + c; row r (query q0 + r) may see
    // columns lo..hi.  With one tile the left half does not exist.
    const int hi = 128 + r;
    const int lo = max(ntile == 2 ? 0 : 128, hi - P.window);
    uint32_t empty = 0u;  // warp-uniform, bit c set when chunk c (32 keys) is outside every row's run
#pragma unroll
    for (int c = 0; c < 8; ++c) empty |= (__all_sync(0xffffffffu, run_mask(lo - 32 * c, hi - 32 * c) == 0u) ? 1u : 0u) << c;
    float sink2 = -INFINITY;
    if (P.sink != nullptr) sink2 = (P.hq <= kMaxStagedSinks ? C->sink[head] : __ldg(P.sink + head)) * kLog2e;

    if (!pwait(C, &C->s_full[hw], n_u & 1, lim)) return;
    tc_fence_after_sync();
    // The pair loops stay rolled: eight softmax warps, the RoPE warpgroup and the
    // single-thread roles share each SM's instruction cache.
    // Pass 1: row max, 64 columns (a chunk pair) at a time, skipping pairs outside every row.
    uint32_t s[2][32];
    float mx[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll 1
    for (int cp = ntile == 2 ? 0 : 2; cp < 4; ++cp) {
      if (((empty >> (2 * cp)) & 3u) == 3u) continue;
      ld_pair(tR, cp, s);
      chunk_max(s[0], run_mask(lo - 64 * cp, hi - 64 * cp), mx);
      chunk_max(s[1], run_mask(lo - 64 * cp - 32, hi - 64 * cp - 32), mx);
    }
    const float mt =
        fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
    const float m = fmaxf(sink2, mt);  // log2 units
    const float base = (m == -INFINITY) ? 0.f : m;
    // Pass 2: P.  P_diag goes to 192..255, P_left to 0..63, and every chunk PV reads is
    // written (0 outside the run).  Pair order 3, 2, 0, 1: each pair's P lands only on
    // columns whose S has already been read (by this pair or an earlier one).
    float sm[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) sm[k] = 0.f;
    const int npairs = ntile == 2 ? 4 : 2;
#pragma unroll 1
    for (int i = 0; i < npairs; ++i) {
      const int cp = i < 2 ? 3 - i : i - 2;
      const uint32_t pcol = tR + (cp >= 2 ? kColPDiag + 32 * (cp - 2) : kColPLeft + 32 * cp);
      uint32_t pk[2][16];
      if (((empty >> (2 * cp)) & 3u) == 3u) {
#pragma unroll
        for (int k = 0; k < 16; ++k) pk[0][k] = pk[1][k] = 0u;
      } else {
        ld_pair(tR, cp, s);
        chunk_exp(s[0], run_mask(lo - 64 * cp, hi - 64 * cp), sl2, base, sm, pk[0]);
        chunk_exp(s[1], run_mask(lo - 64 * cp - 32, hi - 64 * cp - 32), sl2, base, sm, pk[1]);
      }
      tmem_st16(pcol, pk[0]);
      tmem_st16(pcol + 16, pk[1]);
    }
    float l = ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
    if (P.sink != nullptr) l += ex2_approx(sink2 - base);
    tmem_st_wait();
    tc_fence_before_sync();
    mbar_arrive(&C->p_full[hw]);

    // epilogue: O / l (times the V scale), BF16 rows, and the FP32 LSE
    if (!pwait(C, &C->o_full[hw], n_u & 1, lim)) return;
    tc_fence_after_sync();
    uint32_t o[4][32];
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld32(tR + kColO + 32 * q, o[q]);
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

}  // namespace swa

__global__ void __launch_bounds__(pipe::kThreads, 1)
    attn_fwd_swa_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kr,
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
    if (smem_u32(smem) & 1023u) skip = 1;              // swizzled units need a 1 KB aligned base
    if (P.window < 0 || P.window > kBlockN) skip = 1;  // the host only dispatches 0 <= window <= 128 here
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
  if (warp == 3) {
    const long long tiles = swa::count_tiles(P, lane);
    if (lane == 0) C->total_tiles = tiles;
  }
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
      if (warp == 0) role_q_loader<swa::BlockUnits>(smem, C, &tm_q, P);
      else if (warp == 1) swa::role_mma(smem, C, tmem, P);
      else if (warp == 2) swa::role_kv_loader(smem, C, &tm_kr, &tm_k, &tm_v, P);
    }
  } else if (warp < 12) {
    setmaxnreg_inc<kRegsSoftmax>();
    const int hw = (warp - 4) >> 2;
    swa::role_softmax(C, tmem, P, hw, tid - 128 * (1 + hw), warp & 3);
  } else {
    setmaxnreg_dec<kRegsRope>();
    role_rope<swa::BlockUnits>(smem, C, P, tid - 384);
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
