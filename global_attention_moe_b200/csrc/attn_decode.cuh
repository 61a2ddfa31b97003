// attn_decode.cuh -- attention of new query tokens against a KV cache with
// page size 1: decode, speculative-draft verification (up to 8 new tokens per
// sequence) and chunked prefill, for the MiMo-V2 sliding-window (sink) and
// global layers.
//
// Sequence b owns kv_len_b cache entries, listed in position order by
// kv_indices[kv_indptr[b] .. kv_indptr[b+1]) (page size 1: one cache row per
// token), and q_len_b <= kv_len_b new query tokens, rows cu_q[b] .. cu_q[b+1]
// of q.  The new tokens' K and V are already in the cache (its last q_len_b
// entries), so query i sits at position kv_len_b - q_len_b + i and attends
// keys j <= its position (and within the window for the sliding layer).  The
// cache holds K as the forward takes it (not rotated); the kernel rotates the
// first 64 dims of Q and K at their positions.  The result equals the
// forward's output rows for those positions.
//
// This file holds the FP32 CUDA-core form of the per-split kernel (the
// cross-check of the tensor-core kernel in attn_decode_tc.cuh, and the kernel
// for chunked prefill) and the combine kernel both use.  The q_len x (Hq/Hkv)
// query rows that share a KV head are cut into tiles of 128 rows; one CTA per
// (key split, row tile, KV head, sequence) holds the tile's rows, walks the
// split's keys that those rows may see 32 at a time (one key per lane, rows
// spread over the warps) with an online softmax, and writes a partial (max,
// sum, O) per row.  The combine kernel merges, per token and head, the splits
// that overlap its tile's keys with the sink and writes BF16 out and the FP32
// LSE.
#pragma once

#include "params.cuh"
#include "rope_smem.cuh"
#include "sm100.cuh"

namespace mimo {
namespace dec {

constexpr int kThreads = 256;  // 8 warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = 32;                        // keys per step, one per lane
constexpr int kMaxRows = 128;                     // query rows per CTA (one row tile)
constexpr int kRowsPerWarp = kMaxRows / kWarps;   // row r belongs to warp r % kWarps
constexpr int kQStride = kHeadDimQK;              // Q rows are read as broadcast 16-byte loads
constexpr int kKStride = kHeadDimQK + 4;          // 16-byte aligned, lane stride of 4 banks: conflict-free
constexpr int kDimsPerPass = 48;                  // key dims held in registers per pass of the score loop
constexpr int kPStride = kChunk + 1;
constexpr uint32_t kSmemBytes =
    (kMaxRows * kQStride + kChunk * kKStride + kChunk * kHeadDimV + kWarps * kRowsPerWarp * kPStride) * 4;

struct DecParams {
  const uint16_t* q;          // bf16 [Tq, hq, 192]
  const uint16_t* k_cache;    // bf16 [cache_rows, hkv, 192]
  const uint16_t* v_cache;    // bf16 [cache_rows, hkv, 128]
  const int32_t* kv_indices;  // [total_kv] cache row of each key, per sequence in position order
  const int32_t* kv_indptr;   // [num_seqs + 1]
  const int32_t* cu_q;        // [num_seqs + 1]
  const float* sink;          // [hq] or nullptr
  float* part_o;              // [Tq, hq, splits, 128]
  float* part_ml;             // [Tq, hq, splits, 2]: running max (log2 units), sum
  unsigned long long* item_counter;  // zero before the tensor-core kernel: items claimed so far
  uint16_t* out;              // bf16 [Tq, hq, 128]
  float* lse;                 // [hq, Tq]
  int32_t num_seqs, total_q, total_kv, cache_rows;
  int32_t hq, hkv, group;
  int32_t window;             // < 0: global causal layer
  int32_t splits, split_keys;
  int32_t qtiles;             // row tiles per sequence and KV head (CUDA-core kernel; 1 for the tensor-core one)
  float scale_log2;           // log2(e) / sqrt(192)
  float v_scale;
  uint64_t wait_limit_ns;     // bound of every barrier wait (tensor-core kernel)
  double theta[kRopeDims / 2];
};

// The sequence's keys that any of its queries may see: [lo, kv_len).
__device__ __forceinline__ int key_lo(int kv_len, int q_len, int window) {
  const int p0 = kv_len - q_len;  // first query's position
  return (window >= 0 && p0 - window > 0) ? p0 - window : 0;
}

// Keys [lo_t, hi_t) that the query rows row0 .. row0 + rows - 1 of a sequence may see (row r is query
// r / group, at position p0 + r / group).
__device__ __forceinline__ void tile_keys(int p0, int row0, int rows, int group, int window, int& lo_t, int& hi_t) {
  const int pos_first = p0 + row0 / group, pos_last = p0 + (row0 + rows - 1) / group;
  lo_t = (window >= 0 && pos_first - window > 0) ? pos_first - window : 0;
  hi_t = pos_last + 1;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = __bfloat1622float2(h[e]);
    f[2 * e] = x.x;
    f[2 * e + 1] = x.y;
  }
}

// Rotates the first 64 dims of an FP32 row in shared memory (pairs (i, i+32)) at position pos.
__device__ __forceinline__ void rope_pair_f32(float* row, int i, int pos, double theta) {
  float s, c;
  rope_sincos(pos, theta, s, c);
  const float x = row[i], y = row[i + kRopeDims / 2];
  row[i] = x * c - y * s;
  row[i + kRopeDims / 2] = y * c + x * s;
}

__global__ void __launch_bounds__(kThreads) attn_decode_partial_kernel(const __grid_constant__ DecParams P) {
  extern __shared__ __align__(16) float sm[];
  float* sQ = sm;                                // [kMaxRows][kQStride]
  float* sK = sQ + kMaxRows * kQStride;          // [kChunk][kKStride]
  float* sV = sK + kChunk * kKStride;            // [kChunk][128]
  float* sP = sV + kChunk * kHeadDimV;           // [kWarps][kRowsPerWarp][kPStride]
  const int split = blockIdx.x % P.splits, qt = blockIdx.x / P.splits, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int q_beg = __ldg(P.cu_q + b), q_len = __ldg(P.cu_q + b + 1) - q_beg;
  const int kv_beg = __ldg(P.kv_indptr + b), kv_len = __ldg(P.kv_indptr + b + 1) - kv_beg;
  const int all_rows = q_len * P.group;
  // Inconsistent bounds: report and touch nothing (the combine kernel skips the same rows).
  if (q_len < 0 || kv_len < 0 || q_len > kv_len || all_rows > kMaxRows * P.qtiles || q_beg < 0 ||
      q_beg + q_len > P.total_q || kv_beg < 0 || kv_beg + kv_len > P.total_kv) {
    if (tid == 0 && split == 0 && qt == 0 && g == 0) atomicOr(&g_mimo_error, kErrSeqlens);
    return;
  }
  const int row0 = kMaxRows * qt;  // the tile's rows: row0 .. row0 + rows - 1 of the sequence's
  const int rows = min(kMaxRows, all_rows - row0);
  if (rows <= 0) return;
  const int p0 = kv_len - q_len;
  const int lo = key_lo(kv_len, q_len, P.window);
  if (kv_len - lo > P.splits * P.split_keys) {  // more keys than the launch covers (max_kv_len too small)
    if (tid == 0 && split == 0 && qt == 0 && g == 0) atomicOr(&g_mimo_error, kErrSeqlens);
    return;
  }
  // the split's keys, clipped to those the tile's rows may see; a split with none is not read back
  int lo_t, hi_t;
  tile_keys(p0, row0, rows, P.group, P.window, lo_t, hi_t);
  const int s_beg = lo + split * P.split_keys;
  const int k_beg = max(s_beg, lo_t);
  const int k_end = min(min(kv_len, s_beg + P.split_keys), hi_t);
  if (k_end <= k_beg) return;

  // Q rows r = row0 + tile row = i * group + hh (query i of the sequence, head g * group + hh), rotated
  // at p0 + i.
  for (int e = tid; e < rows * (kHeadDimQK / 8); e += kThreads) {
    const int r = e / (kHeadDimQK / 8), c = e % (kHeadDimQK / 8);
    const int i = (row0 + r) / P.group, hh = (row0 + r) % P.group;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(
        P.q + (static_cast<size_t>(q_beg + i) * P.hq + g * P.group + hh) * kHeadDimQK) + c);
    bf16x8_to_f32(u, sQ + r * kQStride + 8 * c);
  }
  __syncthreads();
  for (int e = tid; e < rows * (kRopeDims / 2); e += kThreads) {
    const int r = e / (kRopeDims / 2), i = e % (kRopeDims / 2);
    rope_pair_f32(sQ + r * kQStride, i, p0 + (row0 + r) / P.group, P.theta[i]);
  }

  // Per-row state of this warp's rows r = warp + kWarps * k.
  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][4];
#pragma unroll
  for (int k = 0; k < kRowsPerWarp; ++k) {
    m[k] = -INFINITY;
    l[k] = 0.f;
#pragma unroll
    for (int d = 0; d < 4; ++d) o[k][d] = 0.f;
  }
  float* myP = sP + warp * kRowsPerWarp * kPStride;
  bool bad_index = false;

  for (int c0 = k_beg; c0 < k_end; c0 += kChunk) {
    __syncthreads();  // previous chunk's K/V fully used (and Q rotated, on the first pass)
    const int n = min(kChunk, k_end - c0);
    // gather K and V rows of keys c0 .. c0+n-1 (page size 1: one index per key)
    for (int e = tid; e < n * (kHeadDimQK / 8 + kHeadDimV / 8); e += kThreads) {
      const int jj = e / (kHeadDimQK / 8 + kHeadDimV / 8), c = e % (kHeadDimQK / 8 + kHeadDimV / 8);
      int row = __ldg(P.kv_indices + kv_beg + c0 + jj);
      if (row < 0 || row >= P.cache_rows) {  // out-of-range index: report, read row 0 instead
        bad_index = true;
        row = 0;
      }
      if (c < kHeadDimQK / 8) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(
            P.k_cache + (static_cast<size_t>(row) * P.hkv + g) * kHeadDimQK) + c);
        bf16x8_to_f32(u, sK + jj * kKStride + 8 * c);
      } else {
        const int cv = c - kHeadDimQK / 8;
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(
            P.v_cache + (static_cast<size_t>(row) * P.hkv + g) * kHeadDimV) + cv);
        bf16x8_to_f32(u, sV + jj * kHeadDimV + 8 * cv);
      }
    }
    __syncthreads();
    for (int e = tid; e < n * (kRopeDims / 2); e += kThreads) {
      const int jj = e / (kRopeDims / 2), i = e % (kRopeDims / 2);
      rope_pair_f32(sK + jj * kKStride, i, c0 + jj, P.theta[i]);
    }
    __syncthreads();

    // scores: lane = key c0 + lane, against the warp's rows.  The key's dims sit in registers
    // 48 at a time and every Q value comes from a broadcast 16-byte load, so the loop is bound by
    // the FMA pipe rather than by shared-memory loads.
    const int j = c0 + lane;
    float acc[kRowsPerWarp];
#pragma unroll
    for (int k = 0; k < kRowsPerWarp; ++k) acc[k] = 0.f;
#pragma unroll 1
    for (int d0 = 0; d0 < kHeadDimQK; d0 += kDimsPerPass) {
      float4 kv[kDimsPerPass / 4];
#pragma unroll
      for (int c = 0; c < kDimsPerPass / 4; ++c)
        kv[c] = *reinterpret_cast<const float4*>(sK + lane * kKStride + d0 + 4 * c);
#pragma unroll
      for (int k = 0; k < kRowsPerWarp; ++k) {
        const int r = warp + kWarps * k;
        if (r >= rows) break;  // warp-uniform
        const float4* qr = reinterpret_cast<const float4*>(sQ + r * kQStride + d0);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int c = 0; c < kDimsPerPass / 4; c += 2) {
          const float4 x = qr[c], y = qr[c + 1];
          a0 = fmaf(x.x, kv[c].x, a0);
          a0 = fmaf(x.y, kv[c].y, a0);
          a0 = fmaf(x.z, kv[c].z, a0);
          a0 = fmaf(x.w, kv[c].w, a0);
          a1 = fmaf(y.x, kv[c + 1].x, a1);
          a1 = fmaf(y.y, kv[c + 1].y, a1);
          a1 = fmaf(y.z, kv[c + 1].z, a1);
          a1 = fmaf(y.w, kv[c + 1].w, a1);
        }
        acc[k] += a0 + a1;
      }
    }
#pragma unroll
    for (int k = 0; k < kRowsPerWarp; ++k) {  // unrolled: the per-row state stays in registers
      const int r = warp + kWarps * k;
      if (r >= rows) break;  // warp-uniform
      const int pos = p0 + (row0 + r) / P.group;
      const bool ok = lane < n && j <= pos && (P.window < 0 || pos - j <= P.window);
      const float s = ok ? acc[k] * P.scale_log2 : -INFINITY;
      float mx = s;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[k], mx);
      const float base = (m_new == -INFINITY) ? 0.f : m_new;
      const float corr = ex2_approx(m[k] - base);  // m = -inf -> 0
      const float p = ok ? ex2_approx(s - base) : 0.f;
      float ps = p;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[k] = l[k] * corr + ps;
      m[k] = m_new;
#pragma unroll
      for (int d = 0; d < 4; ++d) o[k][d] *= corr;
      myP[k * kPStride + lane] = p;
    }
    __syncwarp();
    // O += P V: lane owns dims lane, lane+32, lane+64, lane+96
#pragma unroll 1
    for (int jj = 0; jj < n; ++jj) {
      float vv[4];
#pragma unroll
      for (int d = 0; d < 4; ++d) vv[d] = sV[jj * kHeadDimV + lane + 32 * d];
#pragma unroll
      for (int k = 0; k < kRowsPerWarp; ++k) {
        if (warp + kWarps * k >= rows) break;
        const float pk = myP[k * kPStride + jj];
#pragma unroll
        for (int d = 0; d < 4; ++d) o[k][d] = fmaf(pk, vv[d], o[k][d]);
      }
    }
  }
  if (bad_index) atomicOr(&g_mimo_error, kErrSeqlens);

  // partials of this split for the warp's rows
#pragma unroll
  for (int k = 0; k < kRowsPerWarp; ++k) {
    const int r = warp + kWarps * k;
    if (r >= rows) break;
    const int i = (row0 + r) / P.group, hh = (row0 + r) % P.group;
    const size_t slot = (static_cast<size_t>(q_beg + i) * P.hq + g * P.group + hh) * P.splits + split;
#pragma unroll
    for (int d = 0; d < 4; ++d) P.part_o[slot * kHeadDimV + lane + 32 * d] = o[k][d];
    if (lane == 0) {
      P.part_ml[2 * slot] = m[k];
      P.part_ml[2 * slot + 1] = l[k];
    }
  }
}

// One warp per (query token, query head): merges the splits and the sink.
__global__ void __launch_bounds__(kThreads) attn_decode_combine_kernel(const __grid_constant__ DecParams P) {
  const long long wid = (static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<long long>(P.total_q) * P.hq) return;
  const int t = static_cast<int>(wid / P.hq), h = static_cast<int>(wid % P.hq);
  // the sequence of token t must be consistent, as the partial kernel checked
  int lo_b = 0, hi_b = P.num_seqs - 1;
  while (lo_b < hi_b) {
    const int mid = (lo_b + hi_b + 1) >> 1;
    if (__ldg(P.cu_q + mid) <= t) lo_b = mid; else hi_b = mid - 1;
  }
  const int q_beg = __ldg(P.cu_q + lo_b), q_len = __ldg(P.cu_q + lo_b + 1) - q_beg;
  const int kv_beg = __ldg(P.kv_indptr + lo_b), kv_len = __ldg(P.kv_indptr + lo_b + 1) - kv_beg;
  // the partial kernel's checks: such rows were reported there and stay unwritten
  if (q_len <= 0 || q_len > kv_len || q_len * P.group > kMaxRows * P.qtiles || q_beg < 0 ||
      q_beg + q_len > P.total_q || kv_beg < 0 || kv_beg + kv_len > P.total_kv)
    return;
  const int lo = key_lo(kv_len, q_len, P.window);
  if (kv_len - lo > P.splits * P.split_keys) return;
  // The token's row tile and the keys its rows may see: exactly the splits overlapping [lo_t, hi_t)
  // hold written partials for the tile (one tile: every split that holds keys).
  const int row = (t - q_beg) * P.group + h % P.group;
  const int row0 = row / kMaxRows * kMaxRows;
  int lo_t, hi_t;
  tile_keys(kv_len - q_len, row0, min(kMaxRows, q_len * P.group - row0), P.group, P.window, lo_t, hi_t);
  const int s_lo = (lo_t - lo) / P.split_keys, s_hi = (hi_t - 1 - lo) / P.split_keys;
  const size_t base = (static_cast<size_t>(t) * P.hq + h) * P.splits;
  float M = P.sink != nullptr ? __ldg(P.sink + h) * kLog2e : -INFINITY;
  for (int s = s_lo; s <= s_hi; ++s) M = fmaxf(M, P.part_ml[2 * (base + s)]);
  const float mb = (M == -INFINITY) ? 0.f : M;
  float L = P.sink != nullptr ? ex2_approx(__ldg(P.sink + h) * kLog2e - mb) : 0.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = s_lo; s <= s_hi; ++s) {
    const float w = ex2_approx(P.part_ml[2 * (base + s)] - mb);
    L += P.part_ml[2 * (base + s) + 1] * w;
#pragma unroll
    for (int d = 0; d < 4; ++d) acc[d] = fmaf(P.part_o[(base + s) * kHeadDimV + lane + 32 * d], w, acc[d]);
  }
  const float inv = P.v_scale / L;
  uint16_t* dst = P.out + (static_cast<size_t>(t) * P.hq + h) * kHeadDimV;
#pragma unroll
  for (int d = 0; d < 4; ++d) {
    const __nv_bfloat16 x = __float2bfloat16_rn(acc[d] * inv);
    dst[lane + 32 * d] = *reinterpret_cast<const uint16_t*>(&x);
  }
  if (lane == 0) P.lse[static_cast<size_t>(h) * P.total_q + t] = (M + log2f(L)) * kLn2;
}

}  // namespace dec
}  // namespace mimo
