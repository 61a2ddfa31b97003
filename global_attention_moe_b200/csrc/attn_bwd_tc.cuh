// attn_bwd_tc.cuh -- backward of the MiMo-V2 attention forward on the tensor cores (tcgen05 MMAs with
// TMEM accumulators, TMA tile loads): the same gradients as attn_bwd_simple.cuh,
//   dL/ds_j = P_j (dO . v'_j - D + dLSE), P_j = exp(s_j - lse), D = dO . out,
//   dV = v_scale P^T dO, dK~ = scale dS^T Q~, dQ~ = scale dS K~, dq / dk = R(-pos) applied after,
// with every contraction on the tensor cores.
//
// One CTA (128 threads) per (128-key tile, sequence, query head).  Keys are the M = 128 rows:
//   for each 128-query tile that sees the key tile (causal; within the window on sliding layers):
//     S^T = K~ Q~^T and dP^T = V dO^T, in two halves of 64 queries (N = 64; TMEM columns 0..127),
//     P^T and dS^T formed per (key, query) by the thread that owns the key (TMEM lane), written as
//     BF16 into shared memory as [keys][queries] rows in 128-byte-swizzled 64-query boxes;
//     dV += P^T dO and dK~ += dS^T Q~ accumulate in TMEM (columns 192..319, 320..511) across the
//     query tiles: A = P / dS K-major (rows = keys), B = dO / Q~ MN-major (their row-major tiles);
//     dQ~ = dS K~ for this query tile (columns 0..191, reusing S / dP): A = the same dS buffer read
//     MN-major (M = queries), B = K~ MN-major; the tile's R(-pos) scale dQ~ rows are staged in shared
//     memory and added to dq with 16-byte vector reductions along each row (other key tiles add
//     theirs).
//   at the end v_scale dV and R(-pos) scale dK~ of the key rows are added to dv / dk the same way
//   (the query heads of a KV group add to the same rows).
// The rotated Q / K dims enter the MMAs as BF16 (one rounding of the rotation), P and dS as BF16.
// bwdtc_prep_kernel: D - dLSE per (token, head) and the sink gradient; it also zeroes dq, dk, dv
// (dsink is zeroed by the host before).  The work is serialised inside a CTA (load, MMA, softmax-side math, MMA);
// overlap comes from the CTAs resident on other SMs.
#pragma once

#include "attn_bwd_simple.cuh"
#include "params.cuh"
#include "rope_smem.cuh"
#include "sm100.cuh"

namespace mimo {
namespace bwdtc {

constexpr int kThreads = 128;
constexpr uint32_t kBox = 16384;            // 128 rows x 64 bf16, 128-byte swizzled
constexpr uint32_t kOffK = 0;               // K~ (rotated, bf16): 3 boxes
constexpr uint32_t kOffV = 3 * kBox;        // V: 2 boxes
constexpr uint32_t kOffQ = 5 * kBox;        // Q~: 3 boxes
constexpr uint32_t kOffO = 8 * kBox;        // dO: 2 boxes
constexpr uint32_t kOffP = 10 * kBox;       // P^T [keys][queries]: 2 boxes of 64 queries
constexpr uint32_t kOffS = 12 * kBox;       // dS^T [keys][queries]: 2 boxes
constexpr uint32_t kOffRow = 14 * kBox;     // lse (log2 units) [128], D - dLSE [128]
constexpr uint32_t kOffBar = kOffRow + 1024;
constexpr uint32_t kSmemBytes = kOffBar + 64 + 1024;  // + slack to align the base to 1024
// Gradient rows staged for the vector reductions: row per thread, 4 floats of padding per row (so the
// threads' 16-byte writes spread over the banks), over the Q / dO / P boxes (free once the MMAs that
// read them have completed).
constexpr uint32_t kOffStage = kOffQ;
constexpr int kStrideQK = kHeadDimQK + 4, kStrideV = kHeadDimV + 4;
static_assert(kOffStage + 128 * kStrideQK * 4 <= kOffS, "staging overlaps dS");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColDP = 64, kColDQ = 0, kColDV = 192, kColDK = 320;
constexpr uint32_t kIdescS = make_idesc_f32acc(1, 0, 128, 64);       // S^T / dP^T halves
constexpr uint32_t kIdescDV = make_idesc_f32acc(1, 1, 128, 128);     // B = dO, MN-major
constexpr uint32_t kIdescDK = make_idesc_f32acc(1, 1, 128, 192);     // B = Q~, MN-major
constexpr uint32_t kIdescDQ = make_idesc_f32acc(1, 1, 128, 192) | (1u << 15);  // A = dS read MN-major
constexpr float kLog2e = 1.4426950408889634f;

// Rotates the chunk pair (c, c + 4) of row r of a swizzled box (the 64 rope dims) by +pos, in place,
// and stores the result as BF16.
__device__ __forceinline__ void rope_rotate_bf16(uint8_t* box, int r, int c, int pos, const double* theta) {
  uint8_t* row = box + r * 128;
  uint4* plo = reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4));
  uint4* phi = reinterpret_cast<uint4*>(row + (((c + 4) ^ (r & 7)) << 4));
  uint4 lo = *plo, hi = *phi;
  const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lo);
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hi);
  uint32_t ol[4], oh[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = __bfloat1622float2(l2[e]);
    const float2 y = __bfloat1622float2(h2[e]);
    const int i0 = 8 * c + 2 * e;
    float s0, c0, s1, c1;
    rope_sincos(pos, theta[i0], s0, c0);
    rope_sincos(pos, theta[i0 + 1], s1, c1);
    ol[e] = pack_bf16x2(x.x * c0 - y.x * s0, x.y * c1 - y.y * s1);
    oh[e] = pack_bf16x2(y.x * c0 + x.x * s0, y.y * c1 + x.y * s1);
  }
  *plo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
  *phi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
}

// Eight BF16 values into the 16-byte chunk q8 (queries 8 q8 .. 8 q8 + 7 of a 64-query box) of key row r.
__device__ __forceinline__ void store_chunk(uint8_t* box, int r, int q8, const uint32_t (&w)[4]) {
  *reinterpret_cast<uint4*>(box + r * 128 + ((q8 ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint64_t desc(uint32_t saddr, uint32_t lbo) { return sdesc_sw128(saddr, lbo, 1024); }

// Row r of a staged tile (kCols floats, stride kCols + 4): the thread that owns the row writes it
// 4 floats at a time.
template <int kCols>
__device__ __forceinline__ void stage4(float* stage, int r, int c4, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(stage + r * (kCols + 4) + 4 * c4) = make_float4(a, b, c, d);
}

// Adds the first nrows staged rows to global rows dst0 + r * row_stride: warp w takes rows w, w + 4,
// ..., its lanes 16-byte pieces of the row, so each reduction instruction covers consecutive floats.
template <int kCols>
__device__ __forceinline__ void flush_rows(const float* stage, int nrows, float* dst0, size_t row_stride, int warp,
                                           int lane) {
  for (int r = warp; r < nrows; r += 4) {
    const float* src = stage + r * (kCols + 4);
    float* dst = dst0 + r * row_stride;
#pragma unroll
    for (int c = lane; c < kCols / 4; c += 32) {
      const float4 v = *reinterpret_cast<const float4*>(src + 4 * c);
      red_add_f32x4(dst + 4 * c, v.x, v.y, v.z, v.w);
    }
  }
}

// Stages this thread's gradient row R(-pos) scale x, x read from its TMEM lane at columns taddr ..
// taddr + 191 (the 192 Q/K dims) 64 columns at a time; the rotate-half pairs (i, i + 32) of the first
// 64 are turned back by -pos.
__device__ __forceinline__ void stage_rotated_row(float* stage, int r, uint32_t taddr, int pos, float scale,
                                                  const double* theta) {
  {
    uint32_t x[2][32];
    tmem_ld32(taddr, x[0]);
    tmem_ld32(taddr + 32, x[1]);
    tmem_ld_wait(x[0]);
    reg_fence(x[1]);
#pragma unroll
    for (int c4 = 0; c4 < 8; ++c4) {
      float lo[4], hi[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = 4 * c4 + u;
        float sn, cs;
        rope_sincos(pos, theta[i], sn, cs);
        const float a = __uint_as_float(x[0][i]) * scale, b = __uint_as_float(x[1][i]) * scale;
        lo[u] = a * cs + b * sn;
        hi[u] = b * cs - a * sn;
      }
      stage4<kHeadDimQK>(stage, r, c4, lo[0], lo[1], lo[2], lo[3]);
      stage4<kHeadDimQK>(stage, r, 8 + c4, hi[0], hi[1], hi[2], hi[3]);
    }
  }
#pragma unroll
  for (int j = 2; j < 6; j += 2) {
    uint32_t x[2][32];
    tmem_ld32(taddr + 32 * j, x[0]);
    tmem_ld32(taddr + 32 * (j + 1), x[1]);
    tmem_ld_wait(x[0]);
    reg_fence(x[1]);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4)
        stage4<kHeadDimQK>(stage, r, 8 * (j + h) + c4, __uint_as_float(x[h][4 * c4]) * scale,
                           __uint_as_float(x[h][4 * c4 + 1]) * scale, __uint_as_float(x[h][4 * c4 + 2]) * scale,
                           __uint_as_float(x[h][4 * c4 + 3]) * scale);
  }
}

}  // namespace bwdtc

// D - dLSE per (token, head) into P.D, and dL/dsink_h += exp(sigma_h - lse)(dLSE - D).  Work items are
// (head, token stride class): a warp keeps one head, sums its tokens' sink terms in a register and adds
// them with one atomic per item (atomics per token and head would all land on Hq addresses).
__global__ void __launch_bounds__(256) bwdtc_prep_kernel(const __grid_constant__ bwd::BwdParams P) {
  const long long warp = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const long long nwarps = static_cast<long long>(gridDim.x) * 8;
  const long long T = P.total_tokens;
  const int lane = threadIdx.x & 31;
  const long long classes = nwarps / P.hq > 0 ? nwarps / P.hq : 1;  // token stride classes per head
  const bool sink = P.sink != nullptr && P.dsink != nullptr;
  {  // dq, dk, dv zeroed (16-byte aligned, whole rows of 4-float groups); the main kernel adds into them
    const long long i0 = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x, n = static_cast<long long>(gridDim.x) * 256;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    const long long nq = T * P.hq * (kHeadDimQK / 4), nk = T * P.hkv * (kHeadDimQK / 4), nv = T * P.hkv * (kHeadDimV / 4);
    for (long long i = i0; i < nq; i += n) reinterpret_cast<float4*>(P.dq)[i] = z;
    for (long long i = i0; i < nk; i += n) reinterpret_cast<float4*>(P.dk)[i] = z;
    for (long long i = i0; i < nv; i += n) reinterpret_cast<float4*>(P.dv)[i] = z;
  }
  for (long long item = warp; item < classes * P.hq; item += nwarps) {
    const int h = static_cast<int>(item / classes);
    float ds = 0.f;
    for (long long t = item % classes; t < T; t += classes) {
      const size_t base = (static_cast<size_t>(t) * P.hq + h) * kHeadDimV;
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < kHeadDimV / 32; ++d)
        acc += bwd::bf(P.dout[base + lane + 32 * d]) * bwd::bf(P.out[base + lane + 32 * d]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const size_t i = static_cast<size_t>(h) * T + t;
      const float dl = P.dlse != nullptr ? P.dlse[i] : 0.f;
      if (lane == 0) P.D[i] = acc - dl;
      if (sink) ds += ex2_approx((P.sink[h] - P.lse[i]) * bwdtc::kLog2e) * (dl - acc);
    }
    if (sink && lane == 0) atomicAdd(P.dsink + h, ds);
  }
}

__global__ void __launch_bounds__(bwdtc::kThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const __grid_constant__ bwd::BwdParams P, const int heads_per_cta,
                       const uint64_t wait_limit_ns) {
  using namespace bwdtc;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem) + 1023) & ~uintptr_t(1023));
  float* s_lse = reinterpret_cast<float*>(sm + kOffRow);
  float* s_dlt = s_lse + 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);  // 0: K/V, 1: Q/dO, 2: MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);

  const int tid = threadIdx.x, warp = tid >> 5;
  // heads h0 .. h0 + heads_per_cta - 1, all of KV group g: K / V loaded and rotated once, dK / dV
  // accumulated over them in TMEM and added to global memory once
  const int kt = blockIdx.x, b = blockIdx.y, h0 = blockIdx.z * heads_per_cta;
  const int s_b = __ldg(P.cu_seqlens + b), e_b = __ldg(P.cu_seqlens + b + 1);
  if (s_b < 0 || e_b < s_b || e_b > P.total_tokens) {
    if (tid == 0 && kt == 0 && h0 == 0) atomicOr(&g_mimo_error, kErrSeqlens);
    return;
  }
  const int L = e_b - s_b;
  const int k0 = kt * 128;
  if (k0 >= L) return;
  const int nk = min(128, L - k0);
  const int g = h0 / P.group;
  const uint32_t base = smem_u32(sm);

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  bool fail = false;
  uint32_t qo_phase = 0, mma_phase = 0;

  do {
    if (tid == 0) {
      mbar_arrive_expect_tx(&bars[0], 5 * kBox);
      for (int c = 0; c < 3; ++c) tma_load_2d(sm + kOffK + c * kBox, &tm_k, &bars[0], g * kHeadDimQK + 64 * c, s_b + k0);
      for (int c = 0; c < 2; ++c) tma_load_2d(sm + kOffV + c * kBox, &tm_v, &bars[0], g * kHeadDimV + 64 * c, s_b + k0);
    }
    fail = !mbar_wait(&bars[0], 0, wait_limit_ns);
    if (__syncthreads_or(fail)) { fail = true; break; }
#pragma unroll
    for (int c = 0; c < 4; ++c) rope_rotate_bf16(sm + kOffK, tid, c, k0 + tid, P.theta);

    const int q_last = P.window >= 0 ? min(L - 1, k0 + nk - 1 + P.window) : L - 1;
    const int key = k0 + tid;  // this thread's key (S / dP / dV / dK rows)
    const float sl2 = P.scale * kLog2e;
#pragma unroll 1
    for (int h = h0; h < h0 + heads_per_cta; ++h) {
    for (int q0 = k0 / 128 * 128, first = h == h0; q0 <= q_last; q0 += 128, first = 0) {
      const int nq = min(128, L - q0);
      fence_proxy_async_smem();
      __syncthreads();  // the previous tile's MMAs and reads are done; K~ rotated (first pass)
      if (tid == 0) {
        mbar_arrive_expect_tx(&bars[1], 5 * kBox);
        for (int c = 0; c < 3; ++c) tma_load_2d(sm + kOffQ + c * kBox, &tm_q, &bars[1], h * kHeadDimQK + 64 * c, s_b + q0);
        for (int c = 0; c < 2; ++c) tma_load_2d(sm + kOffO + c * kBox, &tm_o, &bars[1], h * kHeadDimV + 64 * c, s_b + q0);
      }
      {
        const bool in = tid < nq;
        const size_t i = static_cast<size_t>(h) * P.total_tokens + s_b + q0 + tid;
        s_lse[tid] = in ? __ldg(P.lse + i) * kLog2e : 0.f;
        s_dlt[tid] = in ? P.D[i] : 0.f;
      }
      fail = !mbar_wait(&bars[1], qo_phase, wait_limit_ns);
      qo_phase ^= 1;
      if (__syncthreads_or(fail)) { fail = true; break; }
#pragma unroll
      for (int c = 0; c < 4; ++c) rope_rotate_bf16(sm + kOffQ, tid, c, q0 + tid, P.theta);
      fence_proxy_async_smem();
      __syncthreads();

      for (int half = 0; half < 2; ++half) {
        if (tid == 0) {
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < 12; ++kk) {  // S^T = K~ Q~^T over 192 dims
            const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
            mma_ss(tmem + kColS, desc(base + kOffK + off, 16), desc(base + kOffQ + off + half * 8192, 16), kIdescS,
                   kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // dP^T = V dO^T over 128 dims
            const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
            mma_ss(tmem + kColDP, desc(base + kOffV + off, 16), desc(base + kOffO + off + half * 8192, 16), kIdescS,
                   kk > 0 ? 1u : 0u);
          }
          tc_commit(&bars[2]);
        }
        fail = !mbar_wait(&bars[2], mma_phase, wait_limit_ns);
        mma_phase ^= 1;
        if (__syncthreads_or(fail)) { fail = true; break; }
        tc_fence_after_sync();
        uint32_t s[2][32], dp[2][32];
        tmem_ld32(tmem + lane_base + kColS, s[0]);
        tmem_ld32(tmem + lane_base + kColS + 32, s[1]);
        tmem_ld32(tmem + lane_base + kColDP, dp[0]);
        tmem_ld32(tmem + lane_base + kColDP + 32, dp[1]);
        tmem_ld_wait(s[0]);
        reg_fence(s[1]);
        reg_fence(dp[0]);
        reg_fence(dp[1]);
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
          uint32_t pw[4], dw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float pv[2], dv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int c = 8 * q8 + 2 * e + u;  // query column of the half
              const int ql = half * 64 + c;       // query row of the tile
              const int q = q0 + ql;
              const bool ok = tid < nk && ql < nq && q >= key && (P.window < 0 || q - key <= P.window);
              const float sv = __uint_as_float(s[c >> 5][c & 31]);
              const float dpv = __uint_as_float(dp[c >> 5][c & 31]);
              pv[u] = ok ? ex2_approx(sv * sl2 - s_lse[ql]) : 0.f;
              dv[u] = pv[u] * (P.v_scale * dpv - s_dlt[ql]);
            }
            pw[e] = pack_bf16x2(pv[0], pv[1]);
            dw[e] = pack_bf16x2(dv[0], dv[1]);
          }
          bwdtc::store_chunk(sm + kOffP + half * kBox, tid, q8, pw);
          bwdtc::store_chunk(sm + kOffS + half * kBox, tid, q8, dw);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
      }
      if (fail) break;

      if (tid == 0) {
        tc_fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // dV += P^T dO (K = 128 queries)
          const uint32_t a_off = (kk >> 2) * kBox + (kk & 3) * 32;
          mma_ss(tmem + kColDV, desc(base + kOffP + a_off, 16), desc(base + kOffO + kk * 2048, kBox), kIdescDV,
                 (kk > 0 || !first) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // dK~ += dS^T Q~
          const uint32_t a_off = (kk >> 2) * kBox + (kk & 3) * 32;
          mma_ss(tmem + kColDK, desc(base + kOffS + a_off, 16), desc(base + kOffQ + kk * 2048, kBox), kIdescDK,
                 (kk > 0 || !first) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // dQ~ = dS K~ (K = 128 keys; A read MN-major)
          mma_ss(tmem + kColDQ, desc(base + kOffS + kk * 2048, kBox), desc(base + kOffK + kk * 2048, kBox), kIdescDQ,
                 kk > 0 ? 1u : 0u);
        tc_commit(&bars[2]);
      }
      fail = !mbar_wait(&bars[2], mma_phase, wait_limit_ns);
      mma_phase ^= 1;
      if (__syncthreads_or(fail)) { fail = true; break; }
      tc_fence_after_sync();
      // dq for the tile's query rows (TMEM lane = query): R(-pos) scale dQ~, staged then added row-wise
      {
        float* stage = reinterpret_cast<float*>(sm + kOffStage);
        stage_rotated_row(stage, tid, tmem + lane_base + kColDQ, q0 + tid, P.scale, P.theta);
        __syncthreads();
        flush_rows<kHeadDimQK>(stage, nq, P.dq + (static_cast<size_t>(s_b + q0) * P.hq + h) * kHeadDimQK,
                               static_cast<size_t>(P.hq) * kHeadDimQK, warp, tid & 31);
      }
      tc_fence_before_sync();
    }
    if (fail) break;
    }
    if (fail) break;

    // dV and R(-pos) scale dK~ of the tile's key rows, staged then added row-wise
    tc_fence_after_sync();
    float* stage = reinterpret_cast<float*>(sm + kOffStage);
    __syncthreads();  // every warp has read the last dq rows out of the staging area
    {
      uint32_t r[4][32];
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld32(tmem + lane_base + kColDV + 32 * j, r[j]);
      tmem_ld_wait(r[0]);
#pragma unroll
      for (int j = 1; j < 4; ++j) reg_fence(r[j]);
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4)
          stage4<kHeadDimV>(stage, tid, 8 * j + c4, __uint_as_float(r[j][4 * c4]) * P.v_scale,
                            __uint_as_float(r[j][4 * c4 + 1]) * P.v_scale, __uint_as_float(r[j][4 * c4 + 2]) * P.v_scale,
                            __uint_as_float(r[j][4 * c4 + 3]) * P.v_scale);
      __syncthreads();
      flush_rows<kHeadDimV>(stage, nk, P.dv + (static_cast<size_t>(s_b + k0) * P.hkv + g) * kHeadDimV,
                            static_cast<size_t>(P.hkv) * kHeadDimV, warp, tid & 31);
      __syncthreads();
    }
    {
      stage_rotated_row(stage, tid, tmem + lane_base + kColDK, key, P.scale, P.theta);
      __syncthreads();
      flush_rows<kHeadDimQK>(stage, nk, P.dk + (static_cast<size_t>(s_b + k0) * P.hkv + g) * kHeadDimQK,
                             static_cast<size_t>(P.hkv) * kHeadDimQK, warp, tid & 31);
    }
  } while (0);

  if (fail && tid == 0) atomicOr(&g_mimo_error, kErrTimeout);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mimo
