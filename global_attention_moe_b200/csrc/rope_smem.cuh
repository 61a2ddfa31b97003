// rope_smem.cuh -- partial RoPE applied in shared memory to a tile that TMA
// has just landed.
//
// Partial rotary embedding on the first 64 of the 192 Q/K dims (miles docs
// "MiMo-V2.6-Flash", section 1 Model Introduction; Megatron-Bridge API doc
// "mimo_v2_flash_bridge", "only 33.4% of head dims get RoPE"), rotate-half
// pairs (i, i+32), theta_i = base^(-2i/64), position = token index within its
// sequence.
//
// Layout: the 64 rotary dims of a 128-row tile are one 128-byte-swizzled TMA
// box: row r occupies bytes [128 r, 128 r + 128) and its 16-byte chunk c
// (elements 8c .. 8c+7) sits at chunk position c ^ (r & 7).  Pair partners
// i and i+32 are chunks c and c+4 of the same row.  Input is BF16; the rotated
// values are written back in place as FP16 (11 significant bits), so that the
// score contraction over these dims runs on FP16 tensor-core operands.
#pragma once

#include "sm100.cuh"

namespace mimo {

constexpr double kTwoPi = 6.283185307179586476925286766559;
constexpr double kInvTwoPi = 0.15915494309189533576888376337251;

// sin/cos of pos * theta.  The angle is formed and reduced to [-pi, pi] in
// FP64 (positions reach 2^17 and beyond, where an FP32 product would be off
// by ~1e-2 rad), then evaluated in FP32.
__device__ __forceinline__ void rope_sincos(int pos, double theta, float& s, float& c) {
  const double ang = static_cast<double>(pos) * theta;
  const double n = rint(ang * kInvTwoPi);
  const double red = fma(-n, kTwoPi, ang);
  __sincosf(static_cast<float>(red), &s, &c);
}

// Rotates chunk pair (c, c+4) of row r of a swizzled 128-row block.  Returns
// the largest |rotated value| (to detect FP16 overflow).
__device__ __forceinline__ float rope_rotate_chunk_pair(uint8_t* block, int r, int c, int pos,
                                                        const double* __restrict__ theta) {
  uint8_t* row = block + r * 128;
  uint4* plo = reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4));
  uint4* phi = reinterpret_cast<uint4*>(row + (((c + 4) ^ (r & 7)) << 4));
  uint4 lo = *plo;
  uint4 hi = *phi;
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
    const int i0 = 8 * c + 2 * e;
    float s0, c0, s1, c1;
    rope_sincos(pos, theta[i0], s0, c0);
    rope_sincos(pos, theta[i0 + 1], s1, c1);
    const float a0 = x.x * c0 - y.x * s0;
    const float b0 = y.x * c0 + x.x * s0;
    const float a1 = x.y * c1 - y.y * s1;
    const float b1 = y.y * c1 + x.y * s1;
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a0), fabsf(b0)), fmaxf(fabsf(a1), fabsf(b1))));
    ol[e] = __floats2half2_rn(a0, a1);
    oh[e] = __floats2half2_rn(b0, b1);
  }
  *plo = olo;
  *phi = ohi;
  return amax;
}

}  // namespace mimo
