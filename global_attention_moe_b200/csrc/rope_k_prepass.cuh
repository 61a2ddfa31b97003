// rope_k_prepass.cuh -- rotates the rope dims of K once per launch.
//
// Every K row is used by many query tiles and heads, so its partial RoPE
// (first 64 of 192 dims, rotate-half pairs (i, i+32), position = index within
// its sequence) is applied here once, to FP16, into a scratch tensor
// k_rope [T, Hkv, 64] that the attention kernel loads in place of K's first
// 64 dims.  The remaining 128 dims are read from K unchanged.
//
// One thread handles one 16-byte chunk pair (c, c+4) of one (token, KV head)
// row: 8 rotations.  Four consecutive threads cover a row's 128 bytes.
#pragma once

#include "params.cuh"
#include "rope_smem.cuh"
#include "sm100.cuh"

namespace mimo {

struct RopeKParams {
  const uint16_t* k;          // bf16 [T, hkv, 192]
  uint16_t* k_rope;           // fp16 [T, hkv, 64]
  const int32_t* cu_seqlens;  // [num_seqs + 1]
  int32_t num_seqs;
  int32_t total_tokens;
  int32_t hkv;
  double theta[kRopeDims / 2];
};

__global__ void __launch_bounds__(256) rope_k_prepass_kernel(const __grid_constant__ RopeKParams P) {
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(P.total_tokens) * P.hkv;
  if (gid >= rows * 4) return;
  const int c = static_cast<int>(gid & 3);
  const long long row = gid >> 2;  // (t, g) row index
  const int t = static_cast<int>(row / P.hkv);
  // sequence containing token t: largest b with cu[b] <= t (empty sequences skipped)
  int lo = 0, hi = P.num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(P.cu_seqlens + mid) <= t) lo = mid; else hi = mid - 1;
  }
  const int pos = t - __ldg(P.cu_seqlens + lo);
  const uint4* src = reinterpret_cast<const uint4*>(P.k + row * kHeadDimQK);
  const uint4 a = __ldg(src + c);
  const uint4 b = __ldg(src + c + 4);
  const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* y2 = reinterpret_cast<const __nv_bfloat162*>(&b);
  uint4 oa, ob;
  __half2* o1 = reinterpret_cast<__half2*>(&oa);
  __half2* o2 = reinterpret_cast<__half2*>(&ob);
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = __bfloat1622float2(x2[e]);
    const float2 y = __bfloat1622float2(y2[e]);
    const int i0 = 8 * c + 2 * e;
    float s0, c0, s1, c1;
    rope_sincos(pos, P.theta[i0], s0, c0);
    rope_sincos(pos, P.theta[i0 + 1], s1, c1);
    const float a0 = x.x * c0 - y.x * s0, b0 = y.x * c0 + x.x * s0;
    const float a1 = x.y * c1 - y.y * s1, b1 = y.y * c1 + x.y * s1;
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a0), fabsf(b0)), fmaxf(fabsf(a1), fabsf(b1))));
    o1[e] = __floats2half2_rn(a0, a1);
    o2[e] = __floats2half2_rn(b0, b1);
  }
  uint4* dst = reinterpret_cast<uint4*>(P.k_rope + row * kRopeDims);
  dst[c] = oa;
  dst[c + 4] = ob;
  if (amax > 65504.f) atomicOr(&g_mimo_error, kErrRange);
}

}  // namespace mimo
