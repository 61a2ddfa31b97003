// attn_fwd_swa_packed.cuh -- sliding-window kernel (window <= 128 keys) with
// the query heads of one KV group packed into the rows of each tile.
//
// The MiMo-V2 sliding-window layer (miles docs "MiMo-V2.6-Flash", section 1
// Model Introduction: window 128, 8 KV heads; section 5.4 Notable quirks: the
// query plus the 128 previous keys) shares every K/V row among the G = Hq/Hkv
// query heads of its group.  A tile here is 128 MMA rows = QT = 128/G query
// tokens x G heads (row r: token r / G, head r % G of the group), so its keys
// are the QT + 128 keys [q0 - 128, q0 + QT): 144 for G = 8, of which each row
// attends 129.  (A tile of 128 tokens of one head spans 256 keys.)  Fewer
// score columns per row means fewer MMAs and fewer exponentials per output.
//
// K/V live in a ring of R = 8 + 2A slots of 16 keys (A = QT / 16 blocks: how
// far the window moves per tile).  Consecutive tiles of a CTA walk one
// (sequence, KV group) in order, so each new tile loads only A new key blocks;
// the slot of load n is n mod R, and a tile's loads are a run of consecutive
// load numbers.  The score MMA takes the whole ring as its N = 16R rows, so
// the window is one MMA per K-step whatever the ring position; score columns
// are ring slots, the softmax maps them back to keys, and columns of slots
// outside the tile's window (the next tile's blocks, possibly still landing)
// are masked by selection, never read into the output.  PV runs over the
// window's slots only.
//
// RoPE (first 64 of the 192 Q/K dims, rotate-half pairs (i, i+32), theta_i =
// base^(-2i/64), positions restart per sequence) is applied in shared memory
// to both operands as they land, BF16 in and FP16 out (11 significant bits):
// Q's rope chunk per tile by the RoPE warpgroup, each new K block's rope chunk
// by the same warpgroup.  No pre-pass, no scratch.
//
// Shared memory (128-byte swizzle throughout; Q chunks are 128 rows x 64
// dims, ring slots 16 rows x 64 dims):
//   Q   : 2 buffers x {rope dims, dims 64..127, dims 128..191}
//   K   : 3 arrays (rope dims, dims 64..127, dims 128..191) x R slots
//   V   : 2 arrays (dims 0..63, dims 64..127) x R slots
// TMEM (512 columns): two regions of 256 columns, tile t in region t % 2:
//   S (fp32) at 0 .. 16R-1; after the softmax, P of slot s (bf16 pairs) at
//   8s .. 8s+7 and O (fp32) at 8R .. 8R+127.  The softmax reads all of S
//   before writing P (to columns of S it has read), and PV waits for every
//   row's P, so the overlays never race.
//
// Warp roles (16 warps):
//   warp 0      Q loader (TMA, 3-D boxes {64 dims, G heads, QT tokens})
//   warp 1      MMA issuer (one thread) and TMEM owner
//   warp 2      K/V loader (TMA, 16-key boxes), bounded by the ring
//   warp 3      counts the tiles at launch
//   warps 4-7   softmax + epilogue of even tiles; warps 8-11 of odd tiles
//   warps 12-15 RoPE of Q rope chunks and K rope blocks
// MMA order: S(t) then PV(t-1); a region is reused two tiles later, once the
// epilogue has read its O.
#pragma once

#include "params.cuh"
#include "rope_smem.cuh"
#include "sm100.cuh"

namespace mimo {
namespace pk {

constexpr int kThreads = 512;
constexpr uint32_t kChunk = 16384;  // Q chunk: 128 rows x 128 bytes
constexpr uint32_t kSlot = 2048;    // ring slot of one K/V array: 16 rows x 128 bytes
constexpr int kBlk = 16;            // keys per ring slot
constexpr uint32_t kRegion = 256;   // TMEM columns per tile region
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxR = 12;
constexpr int kMaxStagedSinks = 256;
constexpr uint32_t kCtrlBytes = 3072;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kRopeBarId = 1;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays below 2^8 between rescales
constexpr uint32_t kRegsCtl = 64, kRegsSoftmax = 168, kRegsRope = 112;  // no spills in any role
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax + 128 * kRegsRope <= 65536, "register split exceeds the launch");

template <int G>
struct Shape {
  static_assert(G == 4 || G == 8, "tiles of 32 x 4 or 16 x 8 rows");
  static constexpr int kQT = 128 / G;          // query tokens per tile
  static constexpr int kA = kQT / kBlk;        // key blocks the window moves per tile
  static constexpr int kWB = 8 + kA;           // key blocks of a tile's window
  static constexpr int kR = 8 + 2 * kA;        // ring slots
  static constexpr int kN = kR * kBlk;         // score columns
  static constexpr int kChunks = kN / 32;      // 32-column chunks of S
  static constexpr uint32_t kColO = kN / 2;    // O follows the P columns
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = 6 * kChunk;
  static constexpr uint32_t kVOff = kKOff + 3 * kR * kSlot;
  static constexpr uint32_t kCtrlOff = kVOff + 2 * kR * kSlot;
  static constexpr uint32_t kSmemBytes = kCtrlOff + kCtrlBytes;
  static_assert(kR <= kMaxR && kColO + 128 <= kRegion && kSmemBytes <= 232448, "layout");
};

struct Ctrl {
  uint64_t q_full[2], q_ready[2], q_empty[2];
  uint64_t k_full[kMaxR], k_ready[kMaxR], k_empty[kMaxR], v_full[kMaxR], v_empty[kMaxR];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint32_t tmem_base;
  int abort;
  long long total_tiles;
  double theta[kRopeDims / 2];
  float2 base_q[kRopeDims / 2];
  float sink[kMaxStagedSinks];
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block too large");

// Bounded wait that also gives up once another role has aborted.  The slow
// path is out of line, one copy per role (Role is only a tag): the roles run
// under different setmaxnreg budgets, which one shared function could not
// satisfy, and keeping it out of the roles' loops keeps their code small.
template <int Role>
__device__ __noinline__ bool pk_wait_slow(Ctrl* C, uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
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

template <int Role>
__device__ __forceinline__ bool pk_wait(Ctrl* C, uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  return pk_wait_slow<Role>(C, bar, parity, limit_ns);
}

// Bits lo..hi of a 32-bit chunk (bounds relative to the chunk; empty when lo > hi).
__device__ __forceinline__ uint32_t bits(int lo, int hi) {
  if (hi < 0 || lo > 31 || lo > hi) return 0u;
  const uint32_t upto = (hi >= 31) ? 0xffffffffu : ((2u << hi) - 1u);
  const uint32_t below = (lo <= 0) ? 0u : ((1u << lo) - 1u);
  return upto & ~below;
}

// The tiles of one CTA, in order: tile u of the whole launch is token tile i of
// KV group g of sequence b, numbered sequence by sequence, then group by group,
// then tile by tile; CTA c takes tiles [c U / grid, (c+1) U / grid).  Along
// with the position, the walker keeps the ring's load numbering: this tile's
// window is key blocks [blk_lo, blk_hi) of its sequence, held by loads
// [n_lo, n_hi), of which [n_new, n_hi) are loaded for this tile (the rest are
// the previous tile's, when it was the preceding tile of the same sequence
// and group).  Every role builds the same walker.
template <int G>
struct TileWalk {
  using S = Shape<G>;
  const int32_t* cu;
  int num_seqs, total_tokens, hkv;
  int b = 0, s_b = 0, L = 0, nt = 0, g = 0, i = 0;
  uint32_t left = 0;
  bool bad = false, started = false;
  uint32_t n_next = 0, n_lo = 0, n_hi = 0, n_new = 0;
  int blk_lo = 0, blk_hi = 0;
  int pb = -1, pg = -1, pi = -1, p_blk_lo = 0, p_blk_hi = 0;
  uint32_t p_n_lo = 0;

  __device__ __forceinline__ bool load_seq() {  // sequence b's bounds; false past the last sequence
    while (b < num_seqs) {
      const int s = __ldg(cu + b), e = __ldg(cu + b + 1);
      if (s < 0 || e < s || e > total_tokens) {
        bad = true;
        L = 0;
      } else {
        s_b = s;
        L = e - s;
      }
      nt = (L + S::kQT - 1) / S::kQT;
      if (nt > 0) return true;
      ++b;
    }
    return false;
  }

  __device__ __forceinline__ TileWalk(const FwdParams& P, long long total)
      : cu(P.cu_seqlens), num_seqs(P.num_seqs), total_tokens(P.total_tokens), hkv(P.hkv) {
    const long long u0 = total * blockIdx.x / gridDim.x, u1 = total * (blockIdx.x + 1) / gridDim.x;
    left = static_cast<uint32_t>(u1 - u0);
    if (left == 0) return;
    long long acc = 0;
    while (load_seq()) {
      const long long here = static_cast<long long>(hkv) * nt;
      if (u0 < acc + here) {
        const long long r = u0 - acc;
        g = static_cast<int>(r / nt);
        i = static_cast<int>(r - static_cast<long long>(g) * nt);
        return;
      }
      acc += here;
      ++b;
    }
    left = 0;  // fewer tiles than the count (inconsistent cu_seqlens): nothing to do
  }

  // Moves to the CTA's next tile (the first one on the first call).
  __device__ __forceinline__ bool next() {
    if (left == 0) return false;
    if (started) {
      if (++i == nt) {
        i = 0;
        if (++g == hkv) {
          g = 0;
          ++b;
          if (!load_seq()) {
            left = 0;
            return false;
          }
        }
      }
    }
    started = true;
    --left;
    const int nblk = (L + kBlk - 1) / kBlk;
    blk_lo = max(0, i * S::kA - 8);
    blk_hi = min(i * S::kA + S::kA, nblk);
    int new_from = blk_lo;
    if (pb == b && pg == g && pi + 1 == i) {  // the window continues the previous tile's
      n_lo = p_n_lo + static_cast<uint32_t>(blk_lo - p_blk_lo);
      new_from = max(p_blk_hi, blk_lo);
    } else {
      n_lo = n_next;
    }
    n_hi = n_lo + static_cast<uint32_t>(blk_hi - blk_lo);
    n_new = n_hi - static_cast<uint32_t>(blk_hi - new_from);
    n_next = n_hi;
    pb = b;
    pg = g;
    pi = i;
    p_blk_lo = blk_lo;
    p_blk_hi = blk_hi;
    p_n_lo = n_lo;
    return true;
  }
};

// Query tiles over all sequences and KV groups (one warp).  Inconsistent
// sequences count as empty, as the walkers treat them, and are reported here.
template <int G>
__device__ __forceinline__ long long count_tiles(const FwdParams& P, int lane) {
  long long acc = 0;
  bool bad = false;
  for (int b = lane; b < P.num_seqs; b += 32) {
    const int s = __ldg(P.cu_seqlens + b), e = __ldg(P.cu_seqlens + b + 1);
    const bool ok = s >= 0 && e >= s && e <= P.total_tokens;
    bad |= !ok;
    acc += ok ? static_cast<long long>(P.hkv) * ((e - s + Shape<G>::kQT - 1) / Shape<G>::kQT) : 0;
  }
  if (bad) atomicOr(&g_mimo_error, kErrSeqlens);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

template <int G>
__device__ void role_q_loader(uint8_t* smem, Ctrl* C, const CUtensorMap* tm_q, const FwdParams& P) {
  using S = Shape<G>;
  TileWalk<G> W(P, C->total_tiles);
  for (uint32_t t = 0; W.next(); ++t) {
    const uint32_t buf = t & 1u;
    if (t >= 2 && !pk_wait<0>(C, &C->q_empty[buf], ((t >> 1) - 1) & 1u, P.wait_limit_ns)) return;
    mbar_arrive_expect_tx(&C->q_full[buf], 3 * kChunk);
#pragma unroll
    for (int c = 0; c < 3; ++c)
      tma_load_3d(smem + S::kQOff + (3 * buf + c) * kChunk, tm_q, &C->q_full[buf], 64 * c, W.g * G,
                  W.s_b + W.i * S::kQT);
  }
  if (W.bad) atomicOr(&g_mimo_error, kErrSeqlens);
}

template <int G>
__device__ void role_kv_loader(uint8_t* smem, Ctrl* C, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                               const FwdParams& P) {
  using S = Shape<G>;
  const uint64_t lim = P.wait_limit_ns;
  TileWalk<G> W(P, C->total_tiles);
  while (W.next()) {
    // K first (the tile's score needs it before its PV needs V)
#pragma unroll 1
    for (uint32_t n = W.n_new; n < W.n_hi; ++n) {
      const uint32_t s = n % S::kR;
      if (n >= S::kR && !pk_wait<1>(C, &C->k_empty[s], ((n / S::kR) - 1) & 1u, lim)) return;
      const int row = W.s_b + (W.blk_lo + static_cast<int>(n - W.n_lo)) * kBlk;
      mbar_arrive_expect_tx(&C->k_full[s], 3 * kSlot);
#pragma unroll
      for (int c = 0; c < 3; ++c)
        tma_load_2d(smem + S::kKOff + (c * S::kR + s) * kSlot, tm_k, &C->k_full[s], W.g * kHeadDimQK + 64 * c, row);
    }
#pragma unroll 1
    for (uint32_t n = W.n_new; n < W.n_hi; ++n) {
      const uint32_t s = n % S::kR;
      if (n >= S::kR && !pk_wait<1>(C, &C->v_empty[s], ((n / S::kR) - 1) & 1u, lim)) return;
      const int row = W.s_b + (W.blk_lo + static_cast<int>(n - W.n_lo)) * kBlk;
      mbar_arrive_expect_tx(&C->v_full[s], 2 * kSlot);
#pragma unroll
      for (int c = 0; c < 2; ++c)
        tma_load_2d(smem + S::kVOff + (c * S::kR + s) * kSlot, tm_v, &C->v_full[s], W.g * kHeadDimV + 64 * c, row);
    }
  }
}

// S = Q K^T over the whole ring (N = 16R rows): 4 FP16 K-steps on the rope
// dims, then 8 BF16 K-steps on the pass-through dims.  Descriptor low words
// count 16-byte units: +2 per 32-byte K-step.
template <int G>
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint32_t q_lo, uint32_t k_lo) {
  using S = Shape<G>;
  constexpr uint32_t kIdF16 = make_idesc_f32acc(0, 0, 128, S::kN);
  constexpr uint32_t kIdBF16 = make_idesc_f32acc(1, 0, 128, S::kN);
  constexpr uint32_t kQStep = kChunk >> 4, kKStep = (S::kR * kSlot) >> 4;
#pragma unroll
  for (int c = 0; c < 3; ++c)
#pragma unroll
    for (int k = 0; k < 4; ++k)
      mma_ss_lo(d_tmem, q_lo + c * kQStep + 2 * k, k_lo + c * kKStep + 2 * k, c == 0 ? kIdF16 : kIdBF16,
                (c | k) != 0 ? 1u : 0u);
}

// O = P V over the window's loads [n_lo, n_hi): one K-step of 16 keys per
// load, A = P of its slot (8 TMEM columns), B = the slot's V (MN-major, the
// two 64-dim halves an array apart).
template <int G>
__device__ __forceinline__ void issue_pv(uint32_t region, uint32_t v_lo, uint32_t n_lo, uint32_t n_hi) {
  using S = Shape<G>;
  constexpr uint32_t kIdPV = make_idesc_f32acc(1, 1, 128, 128);
  uint32_t s = n_lo % S::kR;
#pragma unroll
  for (int j = 0; j < S::kWB; ++j) {
    if (n_lo + j < n_hi)
      mma_ts_lo(region + S::kColO, region + 8 * s, v_lo + s * (kSlot >> 4), kIdPV, j > 0 ? 1u : 0u);
    s = (s + 1 == S::kR) ? 0u : s + 1;
  }
}

template <int G>
__device__ void role_mma(uint8_t* smem, Ctrl* C, uint32_t tmem, const FwdParams& P) {
  using S = Shape<G>;
  const uint64_t lim = P.wait_limit_ns;
  const uint32_t q_lo = sdesc_lo(smem_u32(smem + S::kQOff), 16);
  const uint32_t k_lo = sdesc_lo(smem_u32(smem + S::kKOff), 16);
  const uint32_t v_lo = sdesc_lo(smem_u32(smem + S::kVOff), S::kR * kSlot);
  TileWalk<G> W(P, C->total_tiles), Wn(P, C->total_tiles);  // Wn runs one tile ahead
  bool has = W.next();
  if (has) Wn.next();
  uint32_t p_lo = 0, p_hi = 0, v_wait = 0;  // previous tile's loads; V waited for below v_wait
  for (uint32_t t = 0; has; ++t) {
    const uint32_t buf = t & 1u;
    const bool has_next = Wn.next();  // Wn: the tile after t
    if (!pk_wait<2>(C, &C->q_ready[buf], (t >> 1) & 1u, lim)) return;
    if (t >= 2 && !pk_wait<2>(C, &C->o_empty[buf], ((t >> 1) - 1) & 1u, lim)) return;
#pragma unroll 1
    for (uint32_t n = W.n_new; n < W.n_hi; ++n)
      if (!pk_wait<2>(C, &C->k_ready[n % S::kR], (n / S::kR) & 1u, lim)) return;
    tc_fence_after_sync();
    issue_s<G>(tmem + buf * kRegion, q_lo + buf * 3 * (kChunk >> 4), k_lo);
    tc_commit(&C->s_full[buf]);
    tc_commit(&C->q_empty[buf]);
    // K of the loads the next tile no longer reads is free once this score completes
    const uint32_t k_dead_hi = has_next ? Wn.n_lo : W.n_hi;
#pragma unroll 1
    for (uint32_t n = W.n_lo; n < k_dead_hi; ++n) tc_commit(&C->k_empty[n % S::kR]);
    if (t >= 1) {  // PV of the previous tile
      const uint32_t pbuf = buf ^ 1u;
      if (!pk_wait<2>(C, &C->p_full[pbuf], ((t - 1) >> 1) & 1u, lim)) return;
#pragma unroll 1
      for (uint32_t n = max(v_wait, p_lo); n < p_hi; ++n)
        if (!pk_wait<2>(C, &C->v_full[n % S::kR], (n / S::kR) & 1u, lim)) return;
      v_wait = p_hi;
      tc_fence_after_sync();
      issue_pv<G>(tmem + pbuf * kRegion, v_lo, p_lo, p_hi);
      tc_commit(&C->o_full[pbuf]);
#pragma unroll 1
      for (uint32_t n = p_lo; n < W.n_lo; ++n) tc_commit(&C->v_empty[n % S::kR]);
    }
    p_lo = W.n_lo;
    p_hi = W.n_hi;
    if (!has_next) {  // PV of the last tile
      if (!pk_wait<2>(C, &C->p_full[buf], (t >> 1) & 1u, lim)) return;
#pragma unroll 1
      for (uint32_t n = max(v_wait, p_lo); n < p_hi; ++n)
        if (!pk_wait<2>(C, &C->v_full[n % S::kR], (n / S::kR) & 1u, lim)) return;
      tc_fence_after_sync();
      issue_pv<G>(tmem + buf * kRegion, v_lo, p_lo, p_hi);
      tc_commit(&C->o_full[buf]);
    }
    has = has_next;
    W = Wn;  // tile t+1; Wn moves on to t+2 at the top of the next iteration
  }
}

// Softmax + epilogue of the tiles with parity hw; thread r of the warpgroup owns MMA row r.  One
// pass over the score columns (one TMEM load per 32 columns): the row's run of allowed keys is
// selected (others become -inf), and P = exp2(s * scale - m) is formed against a running max m that
// is updated lazily (P stays below 2^8).
template <int G>
__device__ void role_softmax(Ctrl* C, uint32_t tmem, const FwdParams& P, int hw, int r, int wq) {
  using S = Shape<G>;
  const uint64_t lim = P.wait_limit_ns;
  const uint32_t tR = tmem + (static_cast<uint32_t>(wq * 32) << 16) + hw * kRegion;
  const float sl2 = P.scale_log2;
  const int tok = r / G, hsub = r % G;
  TileWalk<G> W(P, C->total_tiles);
  for (uint32_t t = 0; W.next(); ++t) {
    if ((t & 1u) != static_cast<uint32_t>(hw)) continue;
    const int head = W.g * G + hsub;
    const int p = W.i * S::kQT + tok;  // query position in its sequence
    const bool valid = p < W.L;
    // keys [klo, p] in column space: key k sits in column (base + k) mod N
    const int klo = max(0, p - P.window);
    const int len = valid ? p - klo + 1 : 0;
    const int base = (kBlk * static_cast<int>(W.n_lo % S::kR) - kBlk * W.blk_lo) % S::kN + S::kN;
    const int c0 = (base + klo) % S::kN;
    float sink2 = -INFINITY;
    if (P.sink != nullptr) sink2 = (P.hq <= kMaxStagedSinks ? C->sink[head] : __ldg(P.sink + head)) * kLog2e;

    if (!pk_wait<3>(C, &C->s_full[hw], (t >> 1) & 1u, lim)) return;
    tc_fence_after_sync();
    // One pass over S with a lazily updated running max m (log2 units): P = exp2(s * scale - m) stays
    // below 2^8, and when a chunk's max passes m + 8 the P columns already written (a rare event)
    // are scaled down to the new m before going on.  The sink starts the running max and sum.
    float m = sink2, l = (P.sink != nullptr) ? 1.f : 0.f;
    const float2 sl = make_float2(sl2, sl2);
    float2 sm[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) sm[k] = make_float2(0.f, 0.f);
#pragma unroll 1
    for (int j = 0; j < S::kChunks; ++j) {
      const int a = c0 - 32 * j;
      const uint32_t run = bits(a, a + len - 1) | bits(a - S::kN, a - S::kN + len - 1);
      uint32_t s[32];
      tmem_ld32(tR + 32 * j, s);
      tmem_ld_wait(s);
      float mx[8];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const float v0 = ((run >> e) & 1u) ? __uint_as_float(s[e]) : -INFINITY;
        const float v1 = ((run >> (e + 1)) & 1u) ? __uint_as_float(s[e + 1]) : -INFINITY;
        s[e] = __float_as_uint(v0);
        s[e + 1] = __float_as_uint(v1);
        mx[(e >> 1) & 7] = (e < 16) ? fmaxf(v0, v1) : fmax3(mx[(e >> 1) & 7], v0, v1);
      }
      const float cm = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * sl2;
      const bool grow = cm > m + kRescaleThreshold;
      if (__any_sync(0xffffffffu, grow)) {  // warp-uniform: TMEM access is warp-collective
        const float m_new = grow ? cm : m;
        const float corr = grow ? ex2_approx(m - m_new) : 1.f;  // m = -inf -> 0
        l *= corr;
#pragma unroll
        for (int k = 0; k < 4; ++k) sm[k] = make_float2(sm[k].x * corr, sm[k].y * corr);
#pragma unroll 1
        for (int jj = 0; jj < j; ++jj) {  // P columns written so far
          uint32_t pk[16];
          tmem_ld16(tR + 16 * jj, pk);
          tmem_ld16_wait(pk);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 f = unpack_bf16x2(pk[e]);
            pk[e] = pack_bf16x2(f.x * corr, f.y * corr);
          }
          tmem_st16(tR + 16 * jj, pk);
        }
        m = m_new;
      }
      const float mb = (m == -INFINITY) ? 0.f : m;
      const float2 nb = make_float2(-mb, -mb);
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const float2 x = ffma2(make_float2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), sl, nb);
        const float p0 = ex2_approx(x.x);  // exp2(-inf) = 0 outside the run
        const float p1 = ex2_approx(x.y);
        sm[(e >> 1) & 3] = fadd2(sm[(e >> 1) & 3], make_float2(p0, p1));
        pk[e >> 1] = pack_bf16x2(p0, p1);
      }
      tmem_st16(tR + 16 * j, pk);  // P of the chunk's two slots, onto S columns already read
    }
    l += ((sm[0].x + sm[0].y) + (sm[1].x + sm[1].y)) + ((sm[2].x + sm[2].y) + (sm[3].x + sm[3].y));
    tmem_st_wait();
    tc_fence_before_sync();
    mbar_arrive(&C->p_full[hw]);

    // epilogue: O / l times the V scale, BF16 rows; the FP32 LSE
    if (!pk_wait<3>(C, &C->o_full[hw], (t >> 1) & 1u, lim)) return;
    tc_fence_after_sync();
    uint32_t o[4][32];
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld32(tR + S::kColO + 32 * q, o[q]);
    tmem_ld_wait(o[0]);
    reg_fence(o[1]);
    reg_fence(o[2]);
    reg_fence(o[3]);
    tc_fence_before_sync();
    mbar_arrive(&C->o_empty[hw]);
    if (valid) {
      const float inv = P.v_scale / l;
      uint16_t* dst = P.out + (static_cast<size_t>(W.s_b + p) * P.hq + head) * kHeadDimV;
#pragma unroll
      for (int qd = 0; qd < 8; ++qd) {  // 16 dims (32 bytes) per store
        const int q = qd >> 1, e0 = (qd & 1) * 16;
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[q][e0 + 2 * e]) * inv, __uint_as_float(o[q][e0 + 2 * e + 1]) * inv);
        st_global_v8(dst + 16 * qd, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
      }
      P.lse[static_cast<size_t>(head) * P.total_tokens + W.s_b + p] = (m + log2f(l)) * kLn2;
    }
  }
}

// Rotates one row of a Q rope chunk in place (BF16 -> FP16): cos/sin of
// (tile start + token offset) theta_i as base (tile start) x offset.
__device__ __forceinline__ float rope_q_row(uint8_t* chunk, int r, const float2* __restrict__ base,
                                            const float (&oc)[32], const float (&os)[32]) {
  uint8_t* row = chunk + r * 128;
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

// RoPE warpgroup: per tile, the rope chunk of each newly loaded K block (64
// threads: row r / 4, chunk pair r % 4, at the key's position), then the Q
// tile's rope chunk (thread r owns row r: token r / G).
template <int G>
__device__ void role_rope(uint8_t* smem, Ctrl* C, const FwdParams& P, int r) {
  using S = Shape<G>;
  const uint64_t lim = P.wait_limit_ns;
  float oc[32], os[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) rope_sincos(r / G, C->theta[e], os[e], oc[e]);
  float amax = 0.f;
  TileWalk<G> W(P, C->total_tiles);
  bool ok = true;
  for (uint32_t t = 0; ok && W.next(); ++t) {
#pragma unroll 1
    for (uint32_t n = W.n_new; ok && n < W.n_hi; ++n) {
      const uint32_t s = n % S::kR;
      const bool got = pk_wait<4>(C, &C->k_full[s], (n / S::kR) & 1u, lim);
      if (got && r < 64) {
        const int pos = (W.blk_lo + static_cast<int>(n - W.n_lo)) * kBlk + r / 4;
        const float a = rope_rotate_chunk_pair(smem + S::kKOff + s * kSlot, r / 4, r % 4, pos, C->theta);
        if (pos < W.L) amax = fmaxf(amax, a);  // rows past the sequence are never attended
        fence_proxy_async_smem();
      }
      ok = named_bar_and(kRopeBarId, 128, got);
      if (ok && r == 0) mbar_arrive(&C->k_ready[s]);
    }
    if (!ok) break;
    const uint32_t buf = t & 1u;
    if (r < 32) {
      float sn, cs;
      rope_sincos(W.i * S::kQT, C->theta[r], sn, cs);
      C->base_q[r] = make_float2(cs, sn);
    }
    const bool got = pk_wait<4>(C, &C->q_full[buf], (t >> 1) & 1u, lim);
    named_bar_sync(kRopeBarId, 128);  // base_q written
    if (got) {
      const float a = rope_q_row(smem + S::kQOff + 3 * buf * kChunk, r, C->base_q, oc, os);
      if (W.i * S::kQT + r / G < W.L) amax = fmaxf(amax, a);  // rows past the sequence are never stored
      fence_proxy_async_smem();
    }
    ok = named_bar_and(kRopeBarId, 128, got);  // every thread leaves together once any wait fails
    if (ok && r == 0) mbar_arrive(&C->q_ready[buf]);
  }
  if (amax > 65504.f) atomicOr(&g_mimo_error, kErrRange);
}

}  // namespace pk

template <int G>
__global__ void __launch_bounds__(pk::kThreads, 1)
    attn_fwd_swa_packed_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ FwdParams P) {
  using namespace pk;
  using S = Shape<G>;
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctrl* C = reinterpret_cast<Ctrl*>(smem + S::kCtrlOff);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // A recorded timeout makes later launches skip their work until the host clears it.
  int skip = 0;
  if (tid == 0) {
    skip = (*reinterpret_cast<volatile unsigned int*>(&g_mimo_error) & kErrTimeout) != 0;
    if (smem_u32(smem) & 1023u) skip = 1;                         // swizzled operands need a 1 KB aligned base
    if (P.window < 0 || P.window > 128 || P.group != G) skip = 1;  // the host dispatches only these here
  }
  if (__syncthreads_or(skip)) return;

  if (tid == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&C->q_full[h], 1);
      mbar_init(&C->q_ready[h], 1);
      mbar_init(&C->q_empty[h], 1);
      mbar_init(&C->s_full[h], 1);
      mbar_init(&C->p_full[h], 128);
      mbar_init(&C->o_full[h], 1);
      mbar_init(&C->o_empty[h], 128);
    }
    for (int s = 0; s < S::kR; ++s) {
      mbar_init(&C->k_full[s], 1);
      mbar_init(&C->k_ready[s], 1);
      mbar_init(&C->k_empty[s], 1);
      mbar_init(&C->v_full[s], 1);
      mbar_init(&C->v_empty[s], 1);
    }
    C->abort = 0;
#pragma unroll
    for (int e = 0; e < kRopeDims / 2; ++e) C->theta[e] = P.theta[e];
    fence_barrier_init();
  }
  if (P.sink != nullptr && P.hq <= kMaxStagedSinks)
    for (int h = tid; h < P.hq; h += kThreads) C->sink[h] = __ldg(P.sink + h);
  if (warp == 3) {
    const long long tiles = count_tiles<G>(P, lane);
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
      if (warp == 0) role_q_loader<G>(smem, C, &tm_q, P);
      else if (warp == 1) role_mma<G>(smem, C, tmem, P);
      else if (warp == 2) role_kv_loader<G>(smem, C, &tm_k, &tm_v, P);
    }
  } else if (warp < 12) {
    setmaxnreg_inc<kRegsSoftmax>();
    const int hw = (warp - 4) >> 2;
    role_softmax<G>(C, tmem, P, hw, tid - 128 * (1 + hw), warp & 3);
  } else {
    setmaxnreg_dec<kRegsRope>();
    role_rope<G>(smem, C, P, tid - 384);
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
