// attn_fwd_simple.cuh -- straightforward tcgen05 attention forward: one CTA
// (4 warps) per (128-query tile, query head), every step serialised.  It uses
// the same building blocks as the pipelined kernel (TMA tiles, RoPE in shared
// memory, tcgen05.mma into TMEM, online softmax in registers) and serves as
// the cross-check path for it.
//
// Per KV tile:  TMA K,V -> RoPE(K) -> S = Q K^T (TMEM) -> mask, online softmax
// with the sink folded into the initial max/sum -> P (bf16) into TMEM over S
// -> O += P V (TMEM) ; epilogue out = v_scale * O / l, lse = m + ln l.
#pragma once

#include "params.cuh"
#include "rope_smem.cuh"
#include "sm100.cuh"

namespace mimo {

namespace simple {
constexpr int kThreads = 128;
constexpr uint32_t kBoxBytes = 128 * 64 * 2;  // one 128-row x 64-col bf16 box, 128B swizzled
constexpr uint32_t kQBytes = 3 * kBoxBytes;
constexpr uint32_t kKBytes = 3 * kBoxBytes;
constexpr uint32_t kVBytes = 2 * kBoxBytes;
constexpr uint32_t kSmemBytes = kQBytes + kKBytes + kVBytes + 256 + 1024;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;    // S (fp32, 128 cols); P (bf16x2, 64 cols) aliases it
constexpr uint32_t kColO = 128;  // O (fp32, 128 cols)
constexpr uint32_t kIdescSF16 = make_idesc_f32acc(0, 0, 128, 128);
constexpr uint32_t kIdescSBF16 = make_idesc_f32acc(1, 0, 128, 128);
constexpr uint32_t kIdescPV = make_idesc_f32acc(1, 1, 128, 128);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
}  // namespace simple

// S = Q K^T over 192 dims: 4 FP16 K-steps on the rotated block, 8 BF16 K-steps
// on the two pass-through blocks.  Issued by one thread.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t sq, uint32_t sk, uint32_t idesc_f16,
                                         uint32_t idesc_bf16) {
#pragma unroll
  for (int kk = 0; kk < 12; ++kk) {
    const uint32_t off = (kk >> 2) * simple::kBoxBytes + (kk & 3) * 32;
    mma_ss(d_tmem, sdesc_sw128(sq + off, 16, 1024), sdesc_sw128(sk + off, 16, 1024),
           (kk < 4) ? idesc_f16 : idesc_bf16, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V with P (bf16, 128 x 128) in TMEM and V (128 keys x 128 dims,
// dims contiguous = MN-major B operand) in shared memory: two 64-dim boxes
// 16 KB apart (LBO), 8-key groups 1 KB apart (SBO), 16 keys per K-step.
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t sv, uint32_t idesc,
                                         bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    mma_ts(d_tmem, p_tmem + kk * 8, sdesc_sw128(sv + kk * 2048, simple::kBoxBytes, 1024), idesc,
           (kk > 0 || accumulate) ? 1u : 0u);
  }
}

__global__ void __launch_bounds__(simple::kThreads, 1)
    attn_fwd_simple_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ FwdParams P) {
  using namespace simple;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kQBytes;
  uint8_t* sV = sK + kKBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kVBytes);  // 0: Q, 1: K/V, 2: MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int b = blockIdx.y;
  const int h = blockIdx.z;
  const int q0 = blockIdx.x * kBlockM;

  // A recorded timeout makes later CTAs skip their work until the host clears it.
  int abort_now = 0;
  if (tid == 0) abort_now = (*reinterpret_cast<volatile unsigned int*>(&g_mimo_error) & kErrTimeout) != 0;
  if (__syncthreads_or(abort_now)) return;
  const int s_b = P.cu_seqlens[b];
  const int e_b = P.cu_seqlens[b + 1];
  const int L = e_b - s_b;
  if (s_b < 0 || L < 0 || e_b > P.total_tokens) {
    if (tid == 0 && blockIdx.x == 0 && h == 0) atomicOr(&g_mimo_error, kErrSeqlens);
    return;
  }
  if (L > P.max_seqlen && tid == 0 && blockIdx.x == 0 && h == 0) atomicOr(&g_mimo_error, kErrSeqlens);
  if (q0 >= L) return;
  const int g = h / P.group;

  if (tid == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
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
  const uint32_t sq = smem_u32(sQ), sk = smem_u32(sK), sv = smem_u32(sV);

  // KV tiles touched by this query tile (window: keys >= q0 - window).
  const int kt_hi = q0 / kBlockN;
  int kt_lo = 0;
  if (P.window >= 0) {
    const int lo_key = q0 - P.window;
    kt_lo = lo_key > 0 ? lo_key / kBlockN : 0;
  }

  const int r = tid;  // query row of this thread = TMEM lane
  float m_run = -INFINITY, l_run = 0.f;
  if (P.sink != nullptr) {
    m_run = P.sink[h] * kLog2e;  // sink folded into the initial max and sum
    l_run = 1.f;
  }
  float amax = 0.f;
  bool fail = false;

  do {
    if (tid == 0) {
      mbar_arrive_expect_tx(&bars[0], kQBytes);
#pragma unroll
      for (int c = 0; c < 3; ++c) tma_load_2d(sQ + c * kBoxBytes, &tm_q, &bars[0], h * kHeadDimQK + 64 * c, s_b + q0);
    }
    fail = !mbar_wait(&bars[0], 0, P.wait_limit_ns);
    if (__syncthreads_or(fail)) { fail = true; break; }
#pragma unroll
    for (int c = 0; c < 4; ++c) amax = fmaxf(amax, rope_rotate_chunk_pair(sQ, r, c, q0 + r, P.theta));
    fence_proxy_async_smem();
    __syncthreads();

    uint32_t kv_phase = 0, mma_phase = 0;
    for (int kt = kt_lo; kt <= kt_hi; ++kt) {
      const bool first = (kt == kt_lo);
      if (tid == 0) {
        mbar_arrive_expect_tx(&bars[1], kKBytes + kVBytes);
#pragma unroll
        for (int c = 0; c < 3; ++c)
          tma_load_2d(sK + c * kBoxBytes, &tm_k, &bars[1], g * kHeadDimQK + 64 * c, s_b + kt * kBlockN);
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tma_load_2d(sV + c * kBoxBytes, &tm_v, &bars[1], g * kHeadDimV + 64 * c, s_b + kt * kBlockN);
      }
      fail = !mbar_wait(&bars[1], kv_phase, P.wait_limit_ns);
      kv_phase ^= 1;
      if (__syncthreads_or(fail)) { fail = true; break; }
#pragma unroll
      for (int c = 0; c < 4; ++c) amax = fmaxf(amax, rope_rotate_chunk_pair(sK, r, c, kt * kBlockN + r, P.theta));
      fence_proxy_async_smem();
      __syncthreads();

      if (tid == 0) {
        tc_fence_after_sync();
        issue_qk(tmem + kColS, sq, sk, kIdescSF16, kIdescSBF16);
        tc_commit(&bars[2]);
      }
      fail = !mbar_wait(&bars[2], mma_phase, P.wait_limit_ns);
      mma_phase ^= 1;
      if (__syncthreads_or(fail)) { fail = true; break; }
      tc_fence_after_sync();

      uint32_t s[4][32];
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld32(tmem + lane_base + kColS + 32 * j, s[j]);
      tmem_ld_wait(s[0]);
      reg_fence(s[1]);
      reg_fence(s[2]);
      reg_fence(s[3]);

      // key column c is allowed iff d - window <= c <= d, d = query pos - first key pos of the tile
      const int d = q0 - kt * kBlockN + r;
      const int cmin = (P.window >= 0) ? d - P.window : -1;
      float mt = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int c = 32 * j + i;
          const float x = (c <= d && c >= cmin) ? __uint_as_float(s[j][i]) * P.scale_log2 : -INFINITY;
          s[j][i] = __float_as_uint(x);
          mt = fmaxf(mt, x);
        }
      }
      const float m_new = fmaxf(m_run, mt);
      const float base = (m_new == -INFINITY) ? 0.f : m_new;
      const float corr = ex2_approx(m_run - base);
      float sum = 0.f;
      uint32_t pk[2][32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = ex2_approx(__uint_as_float(s[j][i]) - base);
          const float p1 = ex2_approx(__uint_as_float(s[j][i + 1]) - base);
          sum += p0 + p1;
          pk[j >> 1][(j & 1) * 16 + (i >> 1)] = pack_bf16x2(p0, p1);
        }
      }
      l_run = l_run * corr + sum;
      m_run = m_new;
      if (!first && __any_sync(0xffffffffu, corr != 1.f)) {
        // rescale O (the previous P V has completed: its commit was waited on)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + kColO + 32 * j, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
          tmem_st32(tmem + lane_base + kColO + 32 * j, o);
        }
      }
      tmem_st32(tmem + lane_base + kColS, pk[0]);
      tmem_st32(tmem + lane_base + kColS + 32, pk[1]);
      tmem_st_wait();
      tc_fence_before_sync();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after_sync();
        issue_pv(tmem + kColO, tmem + kColS, sv, kIdescPV, !first);
        tc_commit(&bars[2]);
      }
      fail = !mbar_wait(&bars[2], mma_phase, P.wait_limit_ns);
      mma_phase ^= 1;
      if (__syncthreads_or(fail)) { fail = true; break; }
      tc_fence_after_sync();
    }
    if (fail) break;

    // epilogue
    uint32_t o[4][32];
#pragma unroll
    for (int j = 0; j < 4; ++j) tmem_ld32(tmem + lane_base + kColO + 32 * j, o[j]);
    tmem_ld_wait(o[0]);
    reg_fence(o[1]);
    reg_fence(o[2]);
    reg_fence(o[3]);
    const int p = q0 + r;
    if (p < L) {
      const float inv = P.v_scale / l_run;
      uint4* dst = reinterpret_cast<uint4*>(P.out + (static_cast<size_t>(s_b + p) * P.hq + h) * kHeadDimV);
#pragma unroll
      for (int qd = 0; qd < 16; ++qd) {
        const int j = qd >> 2, i = (qd & 3) * 8;
        uint4 val;
        val.x = pack_bf16x2(__uint_as_float(o[j][i + 0]) * inv, __uint_as_float(o[j][i + 1]) * inv);
        val.y = pack_bf16x2(__uint_as_float(o[j][i + 2]) * inv, __uint_as_float(o[j][i + 3]) * inv);
        val.z = pack_bf16x2(__uint_as_float(o[j][i + 4]) * inv, __uint_as_float(o[j][i + 5]) * inv);
        val.w = pack_bf16x2(__uint_as_float(o[j][i + 6]) * inv, __uint_as_float(o[j][i + 7]) * inv);
        dst[qd] = val;
      }
      P.lse[static_cast<size_t>(h) * P.total_tokens + s_b + p] = (m_run + log2f(l_run)) * kLn2;
    }
  } while (0);

  if (amax > 65504.f) atomicOr(&g_mimo_error, kErrRange);
  if (fail && tid == 0) atomicOr(&g_mimo_error, kErrTimeout);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mimo
