// attn_bwd_simple.cuh -- backward of the MiMo-V2 attention forward (sliding
// window with sink, global causal), FP32 on the CUDA cores: the first correct
// form, the cross-check for a tensor-core backward.
//
// Given the forward's out (BF16) and lse (FP32, natural log, sink included),
// the upstream dO = dL/dout and dLSE = dL/dlse, with P_j = exp(s_j - lse),
// P_sink = exp(sigma_h - lse), D = dO . out:
//   dL/ds_j      = P_j (dO . v'_j - D + dLSE)              (v' = v_scale v)
//   dL/dsigma_h  = sum over the head's rows of P_sink (dLSE - D)
//   dL/dv_j      = v_scale sum over the rows that attend j of P_j dO
//   dL/dq~ = sum_j dL/ds_j k~_j / sqrt(192),  dL/dk~_j = sum over rows of dL/ds_j q~ / sqrt(192)
//   dL/dq = R(-pos) dL/dq~, dL/dk = R(-pos) dL/dk~ (the transpose of the rotation)
// (~ marks the rotated first 64 dims; the rest pass through).
//
// Kernels:
//   bwd_prep_kernel      D[h, t] = dO . out (one warp per (token, head)); zeroes dk, dv, dsink
//   bwd_main_kernel      one CTA per (64-query tile, sequence, query head): recomputes P
//                        chunk by chunk (32 keys) from the rotated Q tile and the forward's
//                        lse, writes dq for its rows (rotated back), and adds the tile's
//                        dk~ / dv contributions to dk / dv with FP32 atomics
//   bwd_finalize_kernel  rotates dk~ back to dk in place (key positions)
#pragma once

#include "params.cuh"
#include "rope_smem.cuh"
#include "sm100.cuh"

namespace mimo {
namespace bwd {

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr int kRows = 64;                // query rows per CTA
constexpr int kRowsPerWarp = kRows / kWarps;
constexpr int kChunk = 32;               // keys per step (one per lane)
constexpr int kQS = kHeadDimQK;          // Q and dO rows: broadcast 16-byte loads
constexpr int kOS = kHeadDimV;
constexpr int kKS = kHeadDimQK + 4;      // K rows: one per lane, 16-byte aligned, 4-bank lane stride
constexpr int kVS = kHeadDimV + 4;
constexpr int kPS = kChunk + 1;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kSmemBytes =
    (kRows * kQS + kRows * kOS + kChunk * kKS + kChunk * kVS + 2 * kRows * kPS + 2 * kRows) * 4;

struct BwdParams {
  const uint16_t* q;     // bf16 [T, hq, 192]
  const uint16_t* k;     // bf16 [T, hkv, 192]
  const uint16_t* v;     // bf16 [T, hkv, 128]
  const float* sink;     // [hq] or nullptr
  const int32_t* cu_seqlens;
  const uint16_t* out;   // bf16 [T, hq, 128] (the forward's)
  const float* lse;      // [hq, T] (the forward's, natural log)
  const uint16_t* dout;  // bf16 [T, hq, 128]
  const float* dlse;     // [hq, T] or nullptr
  float* D;              // scratch [hq, T]
  float* dq;             // [T, hq, 192]
  float* dk;             // [T, hkv, 192]
  float* dv;             // [T, hkv, 128]
  float* dsink;          // [hq] or nullptr (needs sink)
  int32_t num_seqs, total_tokens, max_seqlen, hq, hkv, group;
  int32_t window;        // < 0: global causal layer
  float scale;           // 1 / sqrt(192)
  float v_scale;
  double theta[kRopeDims / 2];
};

__device__ __forceinline__ float bf(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

__device__ __forceinline__ void bf8(const uint16_t* p, float* f) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = __bfloat1622float2(h[e]);
    f[2 * e] = x.x;
    f[2 * e + 1] = x.y;
  }
}

// Rotates the pair (i, i + 32) of an FP32 row in shared memory by +pos (sgn = 1) or -pos (sgn = -1).
__device__ __forceinline__ void rot_pair(float* row, int i, int pos, double theta, float sgn) {
  float s, c;
  rope_sincos(pos, theta, s, c);
  s *= sgn;
  const float x = row[i], y = row[i + kRopeDims / 2];
  row[i] = x * c - y * s;
  row[i + kRopeDims / 2] = y * c + x * s;
}

// D = dO . out per (token, head); zeroes the accumulated outputs.
__global__ void __launch_bounds__(kThreads) bwd_prep_kernel(const __grid_constant__ BwdParams P) {
  const long long gtid = static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x;
  const long long nthreads = static_cast<long long>(gridDim.x) * kThreads;
  const long long T = P.total_tokens;
  for (long long e = gtid; e < T * P.hkv * kHeadDimQK; e += nthreads) P.dk[e] = 0.f;
  for (long long e = gtid; e < T * P.hkv * kHeadDimV; e += nthreads) P.dv[e] = 0.f;
  if (P.dsink != nullptr)
    for (long long e = gtid; e < P.hq; e += nthreads) P.dsink[e] = 0.f;
  const int lane = threadIdx.x & 31;
  for (long long w = gtid >> 5; w < T * P.hq; w += nthreads >> 5) {
    const long long t = w / P.hq;
    const int h = static_cast<int>(w % P.hq);
    const size_t base = (static_cast<size_t>(t) * P.hq + h) * kHeadDimV;
    float acc = 0.f;
#pragma unroll
    for (int d = 0; d < kHeadDimV / 32; ++d) acc += bf(P.dout[base + lane + 32 * d]) * bf(P.out[base + lane + 32 * d]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) P.D[static_cast<size_t>(h) * T + t] = acc;
  }
}

__global__ void __launch_bounds__(kThreads) bwd_main_kernel(const __grid_constant__ BwdParams P) {
  extern __shared__ __align__(16) float sm[];
  float* sQ = sm;                         // [kRows][kQS] rotated q
  float* sO = sQ + kRows * kQS;           // [kRows][kOS] dO
  float* sK = sO + kRows * kOS;           // [kChunk][kKS] rotated k
  float* sV = sK + kChunk * kKS;          // [kChunk][kVS]
  float* sP = sV + kChunk * kVS;          // [kRows][kPS] P of the chunk (row r at r)
  float* sS = sP + kRows * kPS;           // [kRows][kPS] dL/ds of the chunk
  float* sRow = sS + kRows * kPS;         // [2][kRows]: lse (log2 units), dLSE - D
  const int tile = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s_b = __ldg(P.cu_seqlens + b), e_b = __ldg(P.cu_seqlens + b + 1);
  if (s_b < 0 || e_b < s_b || e_b > P.total_tokens) {
    if (tid == 0 && tile == 0 && h == 0) atomicOr(&g_mimo_error, kErrSeqlens);
    return;
  }
  const int L = e_b - s_b;
  const int q0 = tile * kRows;
  if (q0 >= L) return;
  const int nrows = min(kRows, L - q0);
  const int g = h / P.group;
  const size_t T = static_cast<size_t>(P.total_tokens);

  // Q (rotated at the row positions) and dO; per-row lse and dLSE - D
  for (int e = tid; e < kRows * (kHeadDimQK / 8); e += kThreads) {
    const int r = e / (kHeadDimQK / 8), c = e % (kHeadDimQK / 8);
    float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (r < nrows) bf8(P.q + (static_cast<size_t>(s_b + q0 + r) * P.hq + h) * kHeadDimQK + 8 * c, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) sQ[r * kQS + 8 * c + i] = f[i];
  }
  for (int e = tid; e < kRows * (kHeadDimV / 8); e += kThreads) {
    const int r = e / (kHeadDimV / 8), c = e % (kHeadDimV / 8);
    float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (r < nrows) bf8(P.dout + (static_cast<size_t>(s_b + q0 + r) * P.hq + h) * kHeadDimV + 8 * c, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) sO[r * kOS + 8 * c + i] = f[i];
  }
  for (int r = tid; r < kRows; r += kThreads) {
    float l2 = 0.f, dd = 0.f;
    if (r < nrows) {
      const size_t i = static_cast<size_t>(h) * T + s_b + q0 + r;
      l2 = __ldg(P.lse + i) * kLog2e;
      dd = (P.dlse != nullptr ? __ldg(P.dlse + i) : 0.f) - P.D[i];
    }
    sRow[r] = l2;
    sRow[kRows + r] = dd;
  }
  __syncthreads();
  for (int e = tid; e < kRows * (kRopeDims / 2); e += kThreads) {
    const int r = e / (kRopeDims / 2), i = e % (kRopeDims / 2);
    rot_pair(sQ + r * kQS, i, q0 + r, P.theta[i], 1.f);
  }

  // dq~ accumulators: row warp + 8 k, dims lane + 32 m
  float dq[kRowsPerWarp][kHeadDimQK / 32];
#pragma unroll
  for (int k = 0; k < kRowsPerWarp; ++k)
#pragma unroll
    for (int m = 0; m < kHeadDimQK / 32; ++m) dq[k][m] = 0.f;
  const float sl2 = P.scale * kLog2e;

  const int last_key = q0 + nrows - 1;
  const int first_key = P.window >= 0 ? max(0, q0 - P.window) : 0;
#pragma unroll 1
  for (int c0 = first_key; c0 <= last_key; c0 += kChunk) {
    __syncthreads();  // previous chunk fully used (and Q rotated, on the first pass)
    const int n = min(kChunk, last_key + 1 - c0);
    for (int e = tid; e < kChunk * (kHeadDimQK / 8 + kHeadDimV / 8); e += kThreads) {
      const int j = e / (kHeadDimQK / 8 + kHeadDimV / 8), c = e % (kHeadDimQK / 8 + kHeadDimV / 8);
      float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (c < kHeadDimQK / 8) {
        if (j < n) bf8(P.k + (static_cast<size_t>(s_b + c0 + j) * P.hkv + g) * kHeadDimQK + 8 * c, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) sK[j * kKS + 8 * c + i] = f[i];
      } else {
        const int cv = c - kHeadDimQK / 8;
        if (j < n) bf8(P.v + (static_cast<size_t>(s_b + c0 + j) * P.hkv + g) * kHeadDimV + 8 * cv, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) sV[j * kVS + 8 * cv + i] = f[i];
      }
    }
    __syncthreads();
    for (int e = tid; e < kChunk * (kRopeDims / 2); e += kThreads) {
      const int j = e / (kRopeDims / 2), i = e % (kRopeDims / 2);
      rot_pair(sK + j * kKS, i, c0 + j, P.theta[i], 1.f);
    }
    __syncthreads();

    // P and dL/ds for the warp's rows; lane = key c0 + lane
    const int kpos = c0 + lane;
#pragma unroll
    for (int k = 0; k < kRowsPerWarp; ++k) {
      const int r = warp + kWarps * k;
      const int pos = q0 + r;
      float s = 0.f, dp = 0.f;
#pragma unroll 4
      for (int d = 0; d < kHeadDimQK; d += 4) {
        const float4 a = *reinterpret_cast<const float4*>(sQ + r * kQS + d);
        const float4 kk = *reinterpret_cast<const float4*>(sK + lane * kKS + d);
        s = fmaf(a.x, kk.x, fmaf(a.y, kk.y, fmaf(a.z, kk.z, fmaf(a.w, kk.w, s))));
      }
#pragma unroll 4
      for (int d = 0; d < kHeadDimV; d += 4) {
        const float4 a = *reinterpret_cast<const float4*>(sO + r * kOS + d);
        const float4 vv = *reinterpret_cast<const float4*>(sV + lane * kVS + d);
        dp = fmaf(a.x, vv.x, fmaf(a.y, vv.y, fmaf(a.z, vv.z, fmaf(a.w, vv.w, dp))));
      }
      const bool ok = r < nrows && lane < n && kpos <= pos && (P.window < 0 || pos - kpos <= P.window);
      const float p = ok ? exp2f(s * sl2 - sRow[r]) : 0.f;
      sP[r * kPS + lane] = p;
      sS[r * kPS + lane] = p * (P.v_scale * dp + sRow[kRows + r]);
    }
    __syncthreads();

    // dq~ += dL/ds . k~ (scale applied at the end)
#pragma unroll 1
    for (int j = 0; j < n; ++j) {
      float kk[kHeadDimQK / 32];
#pragma unroll
      for (int m = 0; m < kHeadDimQK / 32; ++m) kk[m] = sK[j * kKS + lane + 32 * m];
#pragma unroll
      for (int k = 0; k < kRowsPerWarp; ++k) {
        const float ds = sS[(warp + kWarps * k) * kPS + j];
#pragma unroll
        for (int m = 0; m < kHeadDimQK / 32; ++m) dq[k][m] = fmaf(ds, kk[m], dq[k][m]);
      }
    }
    // dk~_j += scale sum_r dL/ds_rj q~_r : thread = 4 keys x 6 dims
    {
      const int jb = tid & 7, db = tid >> 3;  // keys 4 jb .. 4 jb + 3, dims 6 db .. 6 db + 5
      float acc[4][6];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int i = 0; i < 6; ++i) acc[a][i] = 0.f;
#pragma unroll 2
      for (int r = 0; r < nrows; ++r) {
        float ds[4], qv[6];
#pragma unroll
        for (int a = 0; a < 4; ++a) ds[a] = sS[r * kPS + 4 * jb + a];
#pragma unroll
        for (int i = 0; i < 6; ++i) qv[i] = sQ[r * kQS + 6 * db + i];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int i = 0; i < 6; ++i) acc[a][i] = fmaf(ds[a], qv[i], acc[a][i]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int j = 4 * jb + a;
        if (j < n) {
          float* dst = P.dk + (static_cast<size_t>(s_b + c0 + j) * P.hkv + g) * kHeadDimQK + 6 * db;
#pragma unroll
          for (int i = 0; i < 6; ++i) atomicAdd(dst + i, acc[a][i] * P.scale);
        }
      }
    }
    // dv_j += v_scale sum_r P_rj dO_r : thread = 4 keys x 4 dims
    {
      const int jb = tid & 7, db = tid >> 3;  // keys 4 jb .. 4 jb + 3, dims 4 db .. 4 db + 3
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[a][i] = 0.f;
#pragma unroll 2
      for (int r = 0; r < nrows; ++r) {
        float pv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) pv[a] = sP[r * kPS + 4 * jb + a];
        const float4 o = *reinterpret_cast<const float4*>(sO + r * kOS + 4 * db);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          acc[a][0] = fmaf(pv[a], o.x, acc[a][0]);
          acc[a][1] = fmaf(pv[a], o.y, acc[a][1]);
          acc[a][2] = fmaf(pv[a], o.z, acc[a][2]);
          acc[a][3] = fmaf(pv[a], o.w, acc[a][3]);
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int j = 4 * jb + a;
        if (j < n) {
          float* dst = P.dv + (static_cast<size_t>(s_b + c0 + j) * P.hkv + g) * kHeadDimV + 4 * db;
#pragma unroll
          for (int i = 0; i < 4; ++i) atomicAdd(dst + i, acc[a][i] * P.v_scale);
        }
      }
    }
  }

  // dq: scale, rotate back at -pos (pairs (i, i+32) are dims lane and lane + 32 of this lane), write
#pragma unroll
  for (int k = 0; k < kRowsPerWarp; ++k) {
    const int r = warp + kWarps * k;
    if (r >= nrows) continue;
    float v0 = dq[k][0] * P.scale, v1 = dq[k][1] * P.scale;
    float s, c;
    rope_sincos(q0 + r, P.theta[lane], s, c);
    const float a = v0 * c + v1 * s, bb = v1 * c - v0 * s;  // rotation by -pos
    float* dst = P.dq + (static_cast<size_t>(s_b + q0 + r) * P.hq + h) * kHeadDimQK;
    dst[lane] = a;
    dst[lane + 32] = bb;
#pragma unroll
    for (int m = 2; m < kHeadDimQK / 32; ++m) dst[lane + 32 * m] = dq[k][m] * P.scale;
  }
  // dsink_h += sum over rows of P_sink (dLSE - D)
  if (P.sink != nullptr && P.dsink != nullptr && warp == 0) {
    const float sig2 = __ldg(P.sink + h) * kLog2e;
    float acc = 0.f;
    for (int r = lane; r < nrows; r += 32) acc += exp2f(sig2 - sRow[r]) * sRow[kRows + r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) atomicAdd(P.dsink + h, acc);
  }
}

// dk = R(-pos) dk~ in place: one thread per (token, KV head, rope pair).
__global__ void __launch_bounds__(kThreads) bwd_finalize_kernel(const __grid_constant__ BwdParams P) {
  const long long e = static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x;
  const long long n = static_cast<long long>(P.total_tokens) * P.hkv * (kRopeDims / 2);
  if (e >= n) return;
  const int i = static_cast<int>(e % (kRopeDims / 2));
  const long long th = e / (kRopeDims / 2);
  const int t = static_cast<int>(th / P.hkv);
  // the key's position within its sequence
  int lo = 0, hi = P.num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(P.cu_seqlens + mid) <= t) lo = mid; else hi = mid - 1;
  }
  const int pos = t - __ldg(P.cu_seqlens + lo);
  float* row = P.dk + th * kHeadDimQK;
  float s, c;
  rope_sincos(pos, P.theta[i], s, c);
  const float x = row[i], y = row[i + kRopeDims / 2];
  row[i] = x * c + y * s;
  row[i + kRopeDims / 2] = y * c - x * s;
}

}  // namespace bwd
}  // namespace mimo
