// attn_decode_tc.cuh -- tensor-core form of the KV-cache attention (decode,
// speculative-draft verification, chunked prefill) with page size 1.
//
// The operation is the one attn_decode.cuh states: query i of sequence b sits
// at position kv_len_b - q_len_b + i and attends the cache keys the forward
// would give it; every CTA writes the same per-split partial (running max in
// log2 units, sum, unnormalised O) that the combine kernel there merges with
// the sink.
//
// Work items are (sequence, KV head, key split); the grid is persistent (at
// most one CTA per SM) and the CTAs share the items through a global counter:
// a producer warp claims the next item, skips items without keys, and
// publishes it in a shared-memory ring that every role reads in the same order
// (items are numbered split-major, so the full-length splits go first and the
// short remainders last).  The q_len x (Hq/Hkv) query rows of an item (row r = query r / group, head
// g*group + r % group) form the M = 128 operand of tcgen05.mma (rows past
// q_len x group are zero and never written out).  K/V rows are gathered by index with cp.async straight
// into the 128-byte-swizzled K-major layout a TMA tile load would produce, so
// the score and PV contractions use the same descriptors as the forward:
//
//   Q      : 3 units of 128 rows x 64 dims (dims 0..63 rotated, FP16; 64..191 BF16)
//   stage  : 64 keys: K dims 0..63 (rotated in place, FP16), 64..127, 128..191
//            (8 KB each, 64 rows x 128 B), then V as 64 keys x 128 dims in two
//            8 KB halves (dims 0..63, 64..127); 4 stages in a ring
//   TMEM   : S/P of chunk t in columns 64 (t & 1) .. +63 (P as BF16 pairs in
//            the first 32), O in columns 128..255
//
// Warp roles (14 warps):
//   warps 0-3   softmax (thread = query row = TMEM lane) and the partial write
//   warps 4-7   K/V fetcher: gathers the chunks of all items, in order, into
//               the ring with cp.async as stages free up; each thread's copies
//               of a chunk arrive on the stage's `landed` barrier when done
//   warp 8      TMEM owner; lane 0 issues the MMAs over the CTA's chunk stream
//               (t counts chunks over all items):
//               S(0) | S(1) PV(0) | S(2) PV(1) | ... | PV(T-1)
//               so the score of the next chunk overlaps the softmax of this one; at an item
//               boundary the previous chunk's PV goes first (the new item's S waits for its Q)
//   warps 9-12  lander: per item, once the previous item's last S has read Q,
//               loads and rotates the item's Q (its own cp.async groups); then,
//               per landed chunk, rotates the first 64 dims of K at the key
//               positions (BF16 -> FP16 in place; angle addition from the
//               chunk's first position) and signals the MMA issuer
//   warp 13     item producer (lane 0)
// Fetching and landing are separate warps, so a chunk is signalled as soon as
// it lands, whatever the fetcher is waiting for: chunk f waits for PV(f-4) to
// release its stage, which needs S(f-3), which needs only chunks already
// fetched.  PV of an item's first chunk (which overwrites O) waits until the
// softmax warps have read the previous item's O.
//
// Softmax: lazy rescale as in the pipelined forward (the running max moves only
// when a chunk's max exceeds it by more than 2^8); O is rescaled in TMEM after
// PV(t-1) has completed, and only a warp that rescales waits for that, so the
// softmax of chunk t otherwise hands its P over without a round trip through
// PV(t-1).  Every wait is bounded (kErrTimeout); the softmax
// warps take each wait's outcome warp-uniformly, since the TMEM loads and
// stores that follow are warp-collective.
#pragma once

#include "attn_decode.cuh"
#include "attn_fwd_swa.cuh"
#include "cp_async.cuh"

namespace mimo {
namespace dtc {

constexpr int kThreads = 448;
constexpr int kChunk = 64;   // keys per step
constexpr int kStages = 4;
constexpr int kAhead = kStages - 1;  // chunks in flight ahead of the one being signalled
constexpr uint32_t kQUnit = 16384;   // 128 rows x 64 dims x 2 B
constexpr uint32_t kKUnit = 8192;    // 64 keys x 64 dims x 2 B
constexpr uint32_t kVOff = 3 * kKUnit;
constexpr uint32_t kStageBytes = 3 * kKUnit + 2 * kKUnit;  // 40 KB
constexpr uint32_t kQOff = 0;
constexpr uint32_t kStageOff = 3 * kQUnit;
constexpr uint32_t kCtrlOff = kStageOff + kStages * kStageBytes;  // 212992
constexpr uint32_t kCtrlBytes = 2048;
constexpr int kRing = 16;  // published items not yet read by every role
constexpr uint32_t kSmemBytes = kCtrlOff + kCtrlBytes;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 128;
constexpr uint32_t kQBar = 3;  // named barrier of the lander warpgroup
constexpr uint32_t kIdescSF16 = make_idesc_f32acc(0, 0, 128, kChunk);
constexpr uint32_t kIdescSBF16 = make_idesc_f32acc(1, 0, 128, kChunk);
static_assert(kStageBytes % 1024 == 0 && kStageOff % 1024 == 0 && kVOff % 1024 == 0, "swizzle atoms");



// One work item: a key split of one (sequence, KV head).
struct Work {
  int q_beg, rows, p0;       // first query row, q_len * group, position of query 0
  int kv_beg, k_beg, k_end;  // index-list offset, key range [k_beg, k_end) of this split
  int n;                     // chunks (0: no key of the split is visible to the tile's rows)
  int g, split;              // KV head, split
  int row0;                  // first query row of the tile (rows row0 .. row0 + rows - 1 of the sequence's)
};

struct Ctrl {
  uint64_t q_ready, q_empty;
  uint64_t full[kStages], empty[kStages];
  uint64_t s_full[2], p_full[2], pv_done, o_full, o_empty;  // p_full by chunk parity: a warp may run a chunk ahead
  uint32_t tmem_base;
  int abort;
  uint64_t landed[kStages];  // the fetcher's copies of the stage's chunk are in
  uint64_t item_full[kRing], item_empty[kRing];
  Work ring[kRing];  // n < 0: no more items
  double theta[kRopeDims / 2];  // RoPE inverse frequencies, staged once per CTA
  float2 k_base[2][kRopeDims / 2];  // cos / sin of theta_i x (first key position of the chunk), by chunk parity
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block too large");

// Fills w for item u (split-major: u = (split * num_seqs + b) * hkv + g); false when the item has no query rows or its sequence is
// inconsistent (reported; the combine kernel skips the same rows).  The checks
// are those of the CUDA-core kernel.
__device__ __forceinline__ bool make_work(const dec::DecParams& P, long long u, Work& w) {
  const long long per_tile = static_cast<long long>(P.hkv) * P.num_seqs;
  const long long per_split = per_tile * P.qtiles;
  w.split = static_cast<int>(u / per_split);
  const long long rt = u % per_split;
  const int qt = static_cast<int>(rt / per_tile);
  const long long r = rt % per_tile;
  w.g = static_cast<int>(r % P.hkv);
  const int b = static_cast<int>(r / P.hkv);
  w.q_beg = __ldg(P.cu_q + b);
  const int q_len = __ldg(P.cu_q + b + 1) - w.q_beg;
  w.kv_beg = __ldg(P.kv_indptr + b);
  const int kv_len = __ldg(P.kv_indptr + b + 1) - w.kv_beg;
  const int all_rows = q_len * P.group;
  const int lo = dec::key_lo(kv_len, q_len, P.window);
  if (q_len < 0 || kv_len < 0 || q_len > kv_len || all_rows > 128 * P.qtiles || w.q_beg < 0 ||
      w.q_beg + q_len > P.total_q || w.kv_beg < 0 || w.kv_beg + kv_len > P.total_kv ||
      kv_len - lo > P.splits * P.split_keys) {
    if (w.split == 0 && w.g == 0 && qt == 0) atomicOr(&g_mimo_error, kErrSeqlens);
    return false;
  }
  w.row0 = 128 * qt;
  w.rows = min(128, all_rows - w.row0);
  if (w.rows <= 0) return false;
  w.p0 = kv_len - q_len;
  // the split's keys, clipped to those the tile's rows may see
  const int pos_first = w.p0 + w.row0 / P.group, pos_last = w.p0 + (w.row0 + w.rows - 1) / P.group;
  const int lo_t = P.window >= 0 ? max(0, pos_first - P.window) : 0;
  const int s_beg = lo + w.split * P.split_keys;
  w.k_beg = max(s_beg, lo_t);
  w.k_end = min(min(kv_len, s_beg + P.split_keys), pos_last + 1);
  w.n = w.k_end > w.k_beg ? (w.k_end - w.k_beg + kChunk - 1) / kChunk : 0;
  return true;
}

// Bounded wait; gives up once another role has aborted (kept inline for the same
// reason as the forward's: every role runs it).
__device__ __forceinline__ bool dwait(Ctrl* C, uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
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

// Reader of the CTA's item ring; every role reads every published item once, in order.
struct Items {
  uint32_t k = 0;
  // The next item (false at the end, or when the wait gave up: then failed is set).
  __device__ __forceinline__ bool next(Ctrl* C, Work& w, bool& failed, uint64_t lim) {
    const int slot = static_cast<int>(k % kRing);
    if (!dwait(C, &C->item_full[slot], (k / kRing) & 1, lim)) {
      failed = true;
      return false;
    }
    w = C->ring[slot];
    mbar_arrive(&C->item_empty[slot]);
    ++k;
    return w.n > 0;
  }
};
constexpr uint32_t kItemReaders = 128 + 128 + 1 + 128;  // softmax, fetcher, MMA issuer, lander

// Claims items from the global counter, skips those without keys (and reports
// inconsistent sequences), and publishes the rest; ends with an n < 0 entry.
__device__ __forceinline__ void role_producer(Ctrl* C, const dec::DecParams& P) {
  const uint64_t lim = P.wait_limit_ns;
  const long long total = static_cast<long long>(P.splits) * P.qtiles * P.hkv * P.num_seqs;
#pragma unroll 1
  for (uint32_t k = 0;; ++k) {
    const int slot = static_cast<int>(k % kRing);
    if (k >= kRing && !dwait(C, &C->item_empty[slot], ((k / kRing) - 1) & 1, lim)) return;
    Work w;
    w.n = -1;
#pragma unroll 1
    while (true) {
      const long long v = static_cast<long long>(atomicAdd(P.item_counter, 1ull));
      if (v >= total) break;
      if (make_work(P, v, w) && w.n > 0) break;
      w.n = -1;
    }
    C->ring[slot] = w;
    mbar_arrive(&C->item_full[slot]);
    if (w.n < 0) return;
  }
}

// S = Q K^T for one 64-key chunk: 4 FP16 K-steps (rotated dims) + 8 BF16 K-steps.
__device__ __forceinline__ void issue_s64(uint32_t d_tmem, uint32_t q_lo, uint32_t k_lo) {
  constexpr uint32_t kQStep = kQUnit >> 4, kKStep = kKUnit >> 4;
#pragma unroll
  for (int sub = 0; sub < 4; ++sub) mma_ss_lo(d_tmem, q_lo + 2 * sub, k_lo + 2 * sub, kIdescSF16, sub > 0 ? 1u : 0u);
#pragma unroll
  for (int u = 1; u < 3; ++u)
#pragma unroll
    for (int sub = 0; sub < 4; ++sub)
      mma_ss_lo(d_tmem, q_lo + u * kQStep + 2 * sub, k_lo + u * kKStep + 2 * sub, kIdescSBF16, 1u);
}

// Cache-row indices of the four keys this loader thread copies in chunk c (-1: none / invalid).
__device__ __forceinline__ void load_idx(const dec::DecParams& P, const Work& w, int c, int rsub, int (&idx)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int key = w.k_beg + c * kChunk + 16 * p + rsub;
    idx[p] = key < w.k_end ? __ldg(P.kv_indices + w.kv_beg + key) : -1;
  }
}

// Issues the copies of chunk c of item w into ring stage `stage` (8 lanes per key row, 16 rows per pass).
__device__ __forceinline__ bool issue_chunk(uint8_t* smem, const dec::DecParams& P, const Work& w, int c, int stage,
                                           int l8, int rsub, const int (&idx)[4]) {
  const uint32_t st = smem_u32(smem + kStageOff + stage * kStageBytes);
  bool bad = false;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int j = 16 * p + rsub;  // key row within the chunk
    const int key = w.k_beg + c * kChunk + j;
    const int row = idx[p];
    const bool in = row >= 0 && row < P.cache_rows;
    bad |= key < w.k_end && !in;  // an index outside the cache: zeros, reported
    const uint16_t* ks = in ? P.k_cache + (static_cast<size_t>(row) * P.hkv + w.g) * kHeadDimQK : P.k_cache;
    const uint16_t* vs = in ? P.v_cache + (static_cast<size_t>(row) * P.hkv + w.g) * kHeadDimV : P.v_cache;
    const uint32_t nb = in ? 16u : 0u;
    const uint32_t sw = static_cast<uint32_t>(j * 128 + ((l8 ^ (j & 7)) << 4));
#pragma unroll
    for (int u = 0; u < 3; ++u) cp_async_16(st + u * kKUnit + sw, ks + 64 * u + 8 * l8, nb);
#pragma unroll
    for (int h = 0; h < 2; ++h) cp_async_16(st + kVOff + h * kKUnit + sw, vs + 64 * h + 8 * l8, nb);
  }
  cp_async_commit();
  return bad;
}

// K/V chunks of every item, in one stream over the ring.
__device__ __forceinline__ void role_fetcher(uint8_t* smem, Ctrl* C, const dec::DecParams& P, int lt) {
  const uint64_t lim = P.wait_limit_ns;
  const int l8 = lt & 7, rsub = lt >> 3;
  Items items;
  Work fw;  // the item being fetched
  bool failed = false, bad = false;
  bool more = items.next(C, fw, failed, lim);
  int fc = 0;  // its next chunk
  int idx[4];
  if (more) load_idx(P, fw, 0, rsub, idx);
#pragma unroll 1
  for (uint32_t f = 0; more; ++f) {
    const int stage = static_cast<int>(f % kStages);
    // the stage's previous chunk f-4 is released by PV(f-4)
    if (f >= kStages && !dwait(C, &C->empty[stage], ((f / kStages) - 1) & 1, lim)) break;
    bad |= issue_chunk(smem, P, fw, fc, stage, l8, rsub, idx);
    cp_async_mbar_arrive_noinc(&C->landed[stage]);
    if (++fc == fw.n) {
      more = items.next(C, fw, failed, lim);
      fc = 0;
    }
    if (more) load_idx(P, fw, fc, rsub, idx);  // in flight while this thread waits for the next stage
  }
  cp_async_wait<0>();  // nothing of ours stays in flight, on every path
  if (bad) atomicOr(&g_mimo_error, kErrSeqlens);
}

// Rotates the chunk pair (c, c + 4) of key row r of a landed stage by angles given as cos / sin pairs:
// base[i] of the chunk's first key position and off[e] of the row's offset from it (frequencies 8c ..
// 8c + 7), combined by angle addition.  Returns the largest |rotated value|.
__device__ __forceinline__ float rope_rotate_chunk_pair_add(uint8_t* block, int r, int c, const float2* base,
                                                           const float2 (&off)[8]) {
  uint8_t* row = block + r * 128;
  uint4* plo = reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4));
  uint4* phi = reinterpret_cast<uint4*>(row + (((c + 4) ^ (r & 7)) << 4));
  const uint4 lo = *plo, hi = *phi;
  const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lo);
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hi);
  uint4 olo, ohi;
  __half2* ol = reinterpret_cast<__half2*>(&olo);
  __half2* oh = reinterpret_cast<__half2*>(&ohi);
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = __bfloat1622float2(l2[e]);
    const float2 y = __bfloat1622float2(h2[e]);
    const float2 b0 = base[8 * c + 2 * e], b1 = base[8 * c + 2 * e + 1];
    const float2 o0 = off[2 * e], o1 = off[2 * e + 1];
    const float c0 = b0.x * o0.x - b0.y * o0.y, s0 = b0.y * o0.x + b0.x * o0.y;
    const float c1 = b1.x * o1.x - b1.y * o1.y, s1 = b1.y * o1.x + b1.x * o1.y;
    const float a0 = x.x * c0 - y.x * s0, d0 = y.x * c0 + x.x * s0;
    const float a1 = x.y * c1 - y.y * s1, d1 = y.y * c1 + x.y * s1;
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a0), fabsf(d0)), fmaxf(fabsf(a1), fabsf(d1))));
    ol[e] = __floats2half2_rn(a0, a1);
    oh[e] = __floats2half2_rn(d0, d1);
  }
  *plo = olo;
  *phi = ohi;
  return amax;
}

// Per item: Q (once the previous item's last S has read Q), then every chunk as it lands.
__device__ __forceinline__ void role_lander(uint8_t* smem, Ctrl* C, const dec::DecParams& P, int qt) {
  const uint64_t lim = P.wait_limit_ns;
  const int l8 = qt & 7, rsub = qt >> 3;
  const int group = P.group;
  Items items;
  Work w;
  float amax = 0.f;
  uint32_t landed = 0;
  bool ok = true;
  // cos / sin of theta_i x (this thread's key row within a chunk), for its two chunk pairs' frequencies
  float2 off[2][8];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float sn, cs;
      rope_sincos(qt & 63, C->theta[8 * (2 * (qt >> 6) + h) + e], sn, cs);
      off[h][e] = make_float2(cs, sn);
    }
#pragma unroll 1
  for (uint32_t item = 0;; ++item) {
    bool failed = false;
    const bool have = items.next(C, w, failed, lim);
    ok = ok && !failed && (!have || item == 0 || dwait(C, &C->q_empty, (item - 1) & 1, lim));
    // every thread leaves here together: a failed wait anywhere ends the loop in all of them
    if (!named_bar_and(kQBar, 128, ok) || !have) break;
#pragma unroll 1
    for (int pass = 0; pass < 8; ++pass) {  // zeros past q_len x group
      const int r = 16 * pass + rsub;
      const bool in = r < w.rows;
      const int i = in ? (w.row0 + r) / group : 0, hh = in ? (w.row0 + r) % group : 0;
      const uint16_t* src =
          in ? P.q + (static_cast<size_t>(w.q_beg + i) * P.hq + w.g * group + hh) * kHeadDimQK : P.q;
      const uint32_t sw = static_cast<uint32_t>(r * 128 + ((l8 ^ (r & 7)) << 4));
#pragma unroll
      for (int u = 0; u < 3; ++u)
        cp_async_16(smem_u32(smem + kQOff + u * kQUnit) + sw, src + 64 * u + 8 * l8, in ? 16u : 0u);
    }
    cp_async_commit();
    cp_async_wait<0>();
    named_bar_sync(kQBar, 128);
    const int pos = qt < w.rows ? w.p0 + (w.row0 + qt) / group : 0;  // one row per thread
#pragma unroll
    for (int c = 0; c < 4; ++c) amax = fmaxf(amax, rope_rotate_chunk_pair(smem + kQOff, qt, c, pos, C->theta));
    fence_proxy_async_smem();
    mbar_arrive(&C->q_ready);
    // the item's chunks: rotated dims of the 64 keys, two chunk pairs per thread, at angles
    // base (the chunk's first key position, FP64-reduced by 32 threads per chunk) + off (the row's offset)
    const int r = qt & 63, c0 = 2 * (qt >> 6);
#pragma unroll 1
    for (int c = 0; c < w.n; ++c, ++landed) {
      const int stage = static_cast<int>(landed % kStages);
      float2* base = C->k_base[landed & 1];
      if (qt < kRopeDims / 2) {
        float sn, cs;
        rope_sincos(w.k_beg + c * kChunk, C->theta[qt], sn, cs);
        base[qt] = make_float2(cs, sn);
      }
      named_bar_sync(kQBar, 128);  // this chunk's bases written; the bases of two chunks back are read
      if (ok) ok = dwait(C, &C->landed[stage], (landed / kStages) & 1, lim);
      if (!ok) continue;  // the same trips as the others, without the work, up to the barrier above
      uint8_t* kr = smem + kStageOff + stage * kStageBytes;
#pragma unroll
      for (int h = 0; h < 2; ++h) amax = fmaxf(amax, rope_rotate_chunk_pair_add(kr, r, c0 + h, base, off[h]));
      fence_proxy_async_smem();  // the fetcher's copies and these writes, before the MMA reads the stage
      mbar_arrive(&C->full[stage]);
    }
  }
  cp_async_wait<0>();
  if (amax > 65504.f) atomicOr(&g_mimo_error, kErrRange);
}

__device__ __forceinline__ void role_mma(uint8_t* smem, Ctrl* C, uint32_t tmem, const dec::DecParams& P) {
  const uint64_t lim = P.wait_limit_ns;
  const uint32_t qd = sdesc_lo(smem_u32(smem + kQOff), 16);
  Items items;
  Work w;
  w.n = 0;
  int c = 0;
  bool failed = false;
  uint32_t item = 0;  // busy items started so far
  bool prev = false, prev_first = false, prev_last = false;
  uint32_t prev_item = 0;
#pragma unroll 1
  for (uint32_t t = 0;; ++t) {
    bool have = true;
    if (c == w.n) {
      have = items.next(C, w, failed, lim);
      if (failed) return;
      c = 0;
      if (have) ++item;
    }
    // PV of the previous chunk; at an item boundary it goes before the new item's first score, so that
    // the previous item's epilogue does not wait for this item's Q to load and rotate
    auto pv_prev = [&]() -> bool {
      const uint32_t u = t - 1;
      const int s = static_cast<int>(u % kStages);
      if (!dwait(C, &C->p_full[u & 1], (u >> 1) & 1, lim)) return false;
      if (prev_first && prev_item > 1 && !dwait(C, &C->o_empty, (prev_item - 2) & 1, lim)) return false;
      tc_fence_after_sync();
      issue_pv_half(tmem + kColO, tmem + 64u * (u & 1),
                    sdesc_lo(smem_u32(smem + kStageOff + s * kStageBytes + kVOff), kKUnit), prev_first);
      tc_commit(&C->pv_done);
      tc_commit(&C->empty[s]);
      if (prev_last) tc_commit(&C->o_full);
      return true;
    };
    const bool pv_first = prev && (!have || c == 0);
    if (pv_first && !pv_prev()) return;
    if (have) {
      if (c == 0) {
        if (!dwait(C, &C->q_ready, (item - 1) & 1, lim)) return;
        tc_fence_after_sync();
      }
      const int s = static_cast<int>(t % kStages);
      if (!dwait(C, &C->full[s], (t / kStages) & 1, lim)) return;
      tc_fence_after_sync();
      issue_s64(tmem + 64u * (t & 1), qd, sdesc_lo(smem_u32(smem + kStageOff + s * kStageBytes), 16));
      tc_commit(&C->s_full[t & 1]);
      if (c == w.n - 1) tc_commit(&C->q_empty);  // the item's last S has read Q
    }
    if (prev && !pv_first && !pv_prev()) return;
    if (!have) break;
    prev = true;
    prev_first = c == 0;
    prev_last = c == w.n - 1;
    prev_item = item;
    ++c;
  }
}

// Writes an item's partial for row r: (m, l) and the unnormalised O row.
__device__ __forceinline__ float4* partial_row(const dec::DecParams& P, const Work& w, int r, size_t& slot) {
  const int i = (w.row0 + r) / P.group, hh = (w.row0 + r) % P.group;
  slot = (static_cast<size_t>(w.q_beg + i) * P.hq + w.g * P.group + hh) * P.splits + w.split;
  return reinterpret_cast<float4*>(P.part_o + slot * kHeadDimV);
}

__device__ __forceinline__ void role_softmax(Ctrl* C, uint32_t tmem, const dec::DecParams& P, int r, int wq) {
  const uint64_t lim = P.wait_limit_ns;
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t tO = tmem + lane_base + kColO;
  const float sl2 = P.scale_log2;
  Items items;
  Work w;
  uint32_t t = 0, item = 0;  // chunks and items so far
#pragma unroll 1
  while (true) {
    bool failed = false;
    const bool have = items.next(C, w, failed, lim);
    if (!__all_sync(0xffffffffu, !failed) || !have) break;
    const bool valid = r < w.rows;
    const int pos = valid ? w.p0 + (w.row0 + r) / P.group : -1;  // rows past the queries see no key
    const int last = min(w.k_end - 1, pos);           // last key this row may see
    const int first = P.window >= 0 ? pos - P.window : w.k_beg;
    float m = -INFINITY, l = 0.f;
#pragma unroll 1
    for (int c = 0; c < w.n; ++c, ++t) {
      const uint32_t tS = tmem + lane_base + 64u * (t & 1);
      if (!__all_sync(0xffffffffu, dwait(C, &C->s_full[t & 1], (t >> 1) & 1, lim))) return;
      tc_fence_after_sync();
      uint32_t s[2][32];
      tmem_ld32(tS, s[0]);
      tmem_ld32(tS + 32, s[1]);
      tmem_ld_wait(s[0]);
      reg_fence(s[1]);
      const int c0 = w.k_beg + c * kChunk;
      const int hi = last - c0, lo = max(first - c0, 0);  // allowed columns lo..hi of this chunk
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
      for (int q = 0; q < 2; ++q) {  // masked keys become -inf in place (their exp is 0)
        const uint32_t run = swa::run_mask(lo - 32 * q, hi - 32 * q);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x = ((run >> i) & 1u) ? __uint_as_float(s[q][i]) : -INFINITY;
          s[q][i] = __float_as_uint(x);
          mx[i & 7] = fmaxf(mx[i & 7], x);
        }
      }
      const float mt =
          fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
      const bool grow = mt > m + pipe::kRescaleThreshold;
      const float m_new = grow ? mt : m;
      const float corr = grow ? ex2_approx(m - m_new) : 1.f;  // m = -inf -> 0
      const float base = (m_new == -INFINITY) ? 0.f : m_new;
      float sm[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) sm[k] = 0.f;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(s[q][i]), sl2, -base));
          const float p1 = ex2_approx(fmaf(__uint_as_float(s[q][i + 1]), sl2, -base));
          sm[i & 7] += p0;
          sm[(i + 1) & 7] += p1;
          pk[i >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + 16 * q, pk);
      }
      l = l * corr + (((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7])));
      m = m_new;
      if (c > 0 && __any_sync(0xffffffffu, grow)) {
        // O holds PV of chunks 0 .. c-1 once PV(c-1) has completed: rescale it.  Only a warp that
        // rescales waits; pv_done cannot run two phases ahead of any waiter, since PV(t) needs
        // this chunk's P.
        if (!__all_sync(0xffffffffu, dwait(C, &C->pv_done, (t - 1) & 1, lim))) return;
        tc_fence_after_sync();
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
      mbar_arrive(&C->p_full[t & 1]);
    }
    if (!__all_sync(0xffffffffu, dwait(C, &C->o_full, item & 1, lim))) return;
    tc_fence_after_sync();
    if (P.splits == 1) {
      // One split: the item holds every key its rows see, so the row's output and LSE are final here,
      // with the sink folded into the running max and sum as the combine kernel would (no combine).
      const int i = (w.row0 + r) / P.group, head = w.g * P.group + (w.row0 + r) % P.group;
      const float sg = P.sink != nullptr ? __ldg(P.sink + head) * dec::kLog2e : -INFINITY;
      const float M = fmaxf(m, sg);
      const float mb = (M == -INFINITY) ? 0.f : M;
      const float wgt = ex2_approx(m - mb);  // m = -inf -> 0
      const float L = l * wgt + (P.sink != nullptr ? ex2_approx(sg - mb) : 0.f);
      const float scale = P.v_scale * wgt / L;
      uint16_t* dst = valid ? P.out + (static_cast<size_t>(w.q_beg + i) * P.hq + head) * kHeadDimV : nullptr;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {  // 32 columns at a time (warp-collective loads: every row takes part)
        uint32_t o[32];
        tmem_ld32(tO + 32 * q, o);
        tmem_ld_wait(o);
        if (valid) {
#pragma unroll
          for (int hv = 0; hv < 2; ++hv) {
            uint32_t b[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              b[e] = pack_bf16x2(__uint_as_float(o[16 * hv + 2 * e]) * scale,
                                 __uint_as_float(o[16 * hv + 2 * e + 1]) * scale);
            st_global_v8(dst + 32 * q + 16 * hv, b[0], b[1], b[2], b[3], b[4], b[5], b[6], b[7]);
          }
        }
      }
      tc_fence_before_sync();
      mbar_arrive(&C->o_empty);  // the next item's first PV may overwrite O
      if (valid) P.lse[static_cast<size_t>(head) * P.total_q + w.q_beg + i] = (M + log2f(L)) * dec::kLn2;
      ++item;
      continue;
    }
    size_t slot = 0;
    float4* dst = valid ? partial_row(P, w, r, slot) : nullptr;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {  // 32 columns at a time (the loads are warp-collective: every row takes part)
      uint32_t o[32];
      tmem_ld32(tO + 32 * q, o);
      tmem_ld_wait(o);
      if (valid) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[8 * q + e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                       __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
      }
    }
    tc_fence_before_sync();
    mbar_arrive(&C->o_empty);  // the next item's first PV may overwrite O
    if (valid) {
      P.part_ml[2 * slot] = m;
      P.part_ml[2 * slot + 1] = l;
    }
    ++item;
  }
}

}  // namespace dtc

__global__ void __launch_bounds__(dtc::kThreads, 1) attn_decode_tc_kernel(const __grid_constant__ dec::DecParams P) {
  using namespace dtc;
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctrl* C = reinterpret_cast<Ctrl*>(smem + kCtrlOff);
  const int tid = threadIdx.x, warp = tid >> 5;

  int skip = 0;
  if (tid == 0) {
    skip = (*reinterpret_cast<volatile unsigned int*>(&g_mimo_error) & kErrTimeout) != 0;
    if (smem_u32(smem) & 1023u) skip = 1;  // swizzled operands need a 1 KB aligned base
  }
  if (__syncthreads_or(skip)) return;

  if (tid == 0) {
    mbar_init(&C->q_ready, 128);
    mbar_init(&C->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&C->landed[s], 128);  // one cp.async arrival per fetcher thread
      mbar_init(&C->full[s], 128);
      mbar_init(&C->empty[s], 1);
    }
    mbar_init(&C->s_full[0], 1);
    mbar_init(&C->s_full[1], 1);
    mbar_init(&C->p_full[0], 128);
    mbar_init(&C->p_full[1], 128);
    mbar_init(&C->pv_done, 1);
    mbar_init(&C->o_full, 1);
    mbar_init(&C->o_empty, 128);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&C->item_full[i], 1);
      mbar_init(&C->item_empty[i], kItemReaders);
    }
    C->abort = 0;
    fence_barrier_init();
  }
  if (tid < kRopeDims / 2) C->theta[tid] = P.theta[tid];
  if (warp == 8) {
    tmem_alloc(&C->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = C->tmem_base;

  if (warp < 4) {
    role_softmax(C, tmem, P, tid, warp);
  } else if (warp < 8) {
    role_fetcher(smem, C, P, tid - 128);
  } else if (warp == 8) {
    if ((tid & 31) == 0) role_mma(smem, C, tmem, P);
  } else if (warp < 13) {
    role_lander(smem, C, P, tid - 288);
  } else if ((tid & 31) == 0) {
    role_producer(C, P);
  }
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mimo
