// neighbors.cuh -- the steps on either side of the MiMo-V2 attention kernel:
// FP8 blockwise dequant of a weight (out = fp8 * scale_inv per block), the
// split of the kv-head-interleaved fused QKV output into q, k, v, and top-8
// sigmoid routing with a score-correction bias.  All three are bound by HBM.
//
// Sources (page title and section): miles docs "MiMo-V2.6-Flash", section 1
// Model Introduction (FP8 block-quantized weights, fused kv-head-interleaved
// qkv_proj; 256 routed experts, top-8 sigmoid routing with a fixed
// score-correction bias) and section 3.1 (split into q/k/v in head order);
// Megatron-Bridge API doc "mimo_v2_flash_bridge" (_dequant_fp8_blockwise:
// out = fp8 value times scale_inv; MiMoV2FlashQKVMapping: 192-dim Q/K, 128-dim
// V); SGLang cookbook "MiMo-V2.6", section 2 (router logits in FP32).
// Readings where the pages are silent: E4M3 elements; 128 x 128 scale blocks
// (a parameter); per KV group the fused row holds its query heads, then its K
// head, then its V head; the bias enters the choice only and the weights are
// the chosen sigmoid scores normalised to sum to one; ties go to the lower
// expert index.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace mimo {
namespace nb {

constexpr int kThreads = 256;

// ---------------------------------------------------------------- FP8 dequant
// out = bf16_rne(decode(code) * scale_inv[block]), the exact product rounded once.  The product is
// formed in FP32 (round to nearest) and rounded to BF16 two at a time.  Every BF16 midpoint is an
// FP32 number, so rounding to FP32 first cannot carry the product across one: the two roundings
// differ only when the FP32 product lands exactly on a midpoint (its low 16 bits 0x8000) without
// being exact.  A chunk with such a product forms its products in FP64 instead.  Codes are decoded
// through a 256-entry table in shared memory.

// The scale blocks a chunk of 16 columns starting at j0 touches: b0 (and b1 when it crosses into the
// next block at column `edge`; blocks of at least 16 columns give at most two).
struct DequantCols {
  int j0, b0, b1, edge;
  bool one_block;
};

__device__ __forceinline__ DequantCols dequant_cols(int j0, int block_n) {
  DequantCols c;
  c.j0 = j0;
  c.b0 = j0 / block_n;
  c.edge = (c.b0 + 1) * block_n;
  c.one_block = j0 + 15 < c.edge;
  c.b1 = c.one_block ? c.b0 : (j0 + 15) / block_n;
  return c;
}

__device__ __forceinline__ float dequant_code(const float* lut, uint32_t word, int byte) {
  return lut[(word >> (8 * byte)) & 0xFFu];
}

// Thread = 16 consecutive codes of one row (N % 16 == 0: 16-byte loads, 32-byte stores).
__device__ __forceinline__ void fp8_dequant_chunk(const uint4 u, const float* __restrict__ srow, const DequantCols& c,
                                                  int block_n, const float* lut, uint16_t* __restrict__ dst) {
  const uint32_t cw[4] = {u.x, u.y, u.z, u.w};
  const float s0 = __ldg(srow + c.b0);
  uint32_t w[8];
  bool mid = false;
  if (c.one_block) {
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const float a = __fmul_rn(dequant_code(lut, cw[p >> 1], 2 * (p & 1)), s0);
      const float b = __fmul_rn(dequant_code(lut, cw[p >> 1], 2 * (p & 1) + 1), s0);
      mid |= (__float_as_uint(a) & 0xFFFFu) == 0x8000u;
      mid |= (__float_as_uint(b) & 0xFFFFu) == 0x8000u;
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(a, b);
      w[p] = *reinterpret_cast<const uint32_t*>(&b2);
    }
  } else {
    mid = true;  // a chunk across a block edge (only with blocks that are not multiples of 16 wide)
  }
  if (mid) {
    const float s1 = __ldg(srow + c.b1);
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      uint32_t h[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int jj = 2 * p + k;
        const int j = c.j0 + jj;
        // narrower blocks than 16 columns take the division per column
        const float sc = c.one_block ? s0 : (block_n >= 16 ? (j < c.edge ? s0 : s1) : __ldg(srow + j / block_n));
        const __nv_bfloat16 r = __double2bfloat16(static_cast<double>(dequant_code(lut, cw[jj >> 2], jj & 3)) *
                                                  static_cast<double>(sc));
        h[k] = *reinterpret_cast<const uint16_t*>(&r);
      }
      w[p] = h[0] | (h[1] << 16);
    }
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(w[0], w[1], w[2], w[3]);
  d[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// Rows of at most kThreads chunks: a CTA takes G = kThreads / chunks-per-row whole rows per step, so
// every thread keeps one column chunk (its scale-block columns found once) and walks rows; two row
// groups per loop trip with both loads issued first.  Wider rows: a CTA walks rows, its threads the
// row's chunks.  The only per-chunk index arithmetic left is the row's scale row, i / block_m, in
// 32 bits while M allows.
__global__ void __launch_bounds__(kThreads) fp8_dequant_kernel(const uint8_t* __restrict__ codes,
                                                               const float* __restrict__ scale_inv,
                                                               uint16_t* __restrict__ out, int64_t M, int64_t N,
                                                               int block_m, int block_n) {
  static_assert(kThreads == 256, "one decode-table entry per thread");
  __shared__ float lut[256];
  lut[threadIdx.x] = __half2float(__half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(threadIdx.x),
                                                                 __NV_E4M3)));
  __syncthreads();
  const int64_t per_row = N / 16;
  const int64_t scale_cols = (N + block_n - 1) / block_n;
  const bool m32 = M <= 0x7FFFFFFF;
  auto scale_row = [&](int64_t i) {
    const int64_t r = m32 ? static_cast<int64_t>(static_cast<uint32_t>(i) / static_cast<uint32_t>(block_m))
                          : i / block_m;
    return scale_inv + r * scale_cols;
  };
  const uint4* src = reinterpret_cast<const uint4*>(codes);  // chunk e starts at byte 16 e
  if (per_row <= kThreads) {
    const int pr = static_cast<int>(per_row);
    const int G = kThreads / pr;
    const int r_off = static_cast<int>(threadIdx.x) / pr;
    if (r_off >= G) return;  // no CTA-wide synchronisation follows
    const int jc = static_cast<int>(threadIdx.x) - r_off * pr;
    const DequantCols cols = dequant_cols(16 * jc, block_n);
    const int64_t groups = (M + G - 1) / G;
    const int64_t gstep = gridDim.x;
    for (int64_t g = blockIdx.x; g < groups; g += 2 * gstep) {
      const int64_t i0 = g * G + r_off, i1 = (g + gstep) * G + r_off;
      const int64_t e0 = i0 * per_row + jc, e1 = i1 * per_row + jc;
      const bool has0 = i0 < M, has1 = i1 < M;
      uint4 u0 = make_uint4(0, 0, 0, 0), u1 = make_uint4(0, 0, 0, 0);
      if (has0) u0 = __ldg(src + e0);
      if (has1) u1 = __ldg(src + e1);
      if (has0) fp8_dequant_chunk(u0, scale_row(i0), cols, block_n, lut, out + e0 * 16);
      if (has1) fp8_dequant_chunk(u1, scale_row(i1), cols, block_n, lut, out + e1 * 16);
    }
  } else {
    for (int64_t i = blockIdx.x; i < M; i += gridDim.x) {
      const float* srow = scale_row(i);
      for (int64_t jc = threadIdx.x; jc < per_row; jc += 2 * kThreads) {
        const int64_t jc1 = jc + kThreads;
        const bool has1 = jc1 < per_row;
        const uint4 u0 = __ldg(src + i * per_row + jc);
        uint4 u1 = make_uint4(0, 0, 0, 0);
        if (has1) u1 = __ldg(src + i * per_row + jc1);
        fp8_dequant_chunk(u0, srow, dequant_cols(static_cast<int>(16 * jc), block_n), block_n, lut,
                          out + (i * per_row + jc) * 16);
        if (has1)
          fp8_dequant_chunk(u1, srow, dequant_cols(static_cast<int>(16 * jc1), block_n), block_n, lut,
                            out + (i * per_row + jc1) * 16);
      }
    }
  }
}

// ---------------------------------------------------------------- fused QKV split
// Thread = one 16-byte chunk (8 bf16) of the fused row; every head boundary is a multiple of 8.
__global__ void __launch_bounds__(kThreads) qkv_split_kernel(const uint16_t* __restrict__ fused,
                                                             uint16_t* __restrict__ q, uint16_t* __restrict__ k,
                                                             uint16_t* __restrict__ v, int64_t T, int hq, int hkv) {
  const int group = hq / hkv;
  const int per_group = group * 192 + 192 + 128;  // elements
  const int chunks_per_group = per_group / 8;
  const int64_t chunks_per_row = static_cast<int64_t>(hkv) * chunks_per_group;
  const int64_t n = T * chunks_per_row;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t t = e / chunks_per_row;
    const int rem = static_cast<int>(e % chunks_per_row);
    const int g = rem / chunks_per_group;
    const int o = (rem % chunks_per_group) * 8;  // element offset inside the group
    const uint4 val = __ldg(reinterpret_cast<const uint4*>(fused) + e);
    uint16_t* dst;
    if (o < group * 192) {
      dst = q + (t * hq + g * group + o / 192) * 192 + o % 192;
    } else if (o < group * 192 + 192) {
      dst = k + (t * hkv + g) * 192 + (o - group * 192);
    } else {
      dst = v + (t * hkv + g) * 128 + (o - group * 192 - 192);
    }
    *reinterpret_cast<uint4*>(dst) = val;
  }
}

// ---------------------------------------------------------------- MoE router
// One warp per token (E <= 256, E % 32 == 0): lane holds experts lane + 32 m.  The choice is taken on
// FP32 keys fp32(sigmoid) + bias with the sigmoid formed in FP64; the weights are the chosen FP64
// scores normalised in FP64, stored as FP32.
//
// Only the keys near the top k decide anything, so the FP64 sigmoid is formed for those alone:
//   1. approximate keys from an FP32 sigmoid whose error is bounded (below);
//   2. a lower bound L on the k-th largest approximate key: the k-th largest of the lanes' maxima
//      (k of the keys are at least that);
//   3. candidates: experts whose approximate key is at least L less the error margin.  Every
//      expert of the exact top k is one: an expert below that has k exact keys strictly above it;
//   4. exact keys for the candidates (FP64 sigmoid, the same expression as the exact loop), then
//      each candidate's rank by (key descending, expert ascending).
// A token with more than 32 candidates (many keys within the margin of L) or a NaN among them takes
// the exact loop over all its experts, which gives the same result by definition.

__device__ __forceinline__ double route_sigmoid_f64(double x) {
  return x >= 0 ? 1.0 / (1.0 + exp(-x)) : exp(x) / (1.0 + exp(x));
}

// Approximate sigmoid 1 / (1 + e), e = __expf(-x): e is within (2 + 1.173 |x|) ulp of exp(-x) and
// __fdividef within 2 ulp for divisors up to 2^126 (CUDA's documented bounds).  With s the exact
// sigmoid, e's relative error d moves the result by at most s d e / (1 + e): for x >= 0 that is
// (2 + 1.173 x) e^-x / (1 + e^-x)^2 2^-23 <= 0.65 2^-23; for x < 0 it is below (2 + 1.173 |x|) /
// (1 + e^|x|) 2^-23 <= 2^-23.  The rounding of 1 + e adds at most 2^-24 and the division 2 ulp of s
// (<= 2^-23), so the absolute error is below 2^-21.  Past the divisor's range (x below about -87)
// the result is 0 against an exact value below 2^-126.
__device__ __forceinline__ float route_sigmoid_approx(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

// The exact choice for one token over all its experts.
template <int kMaxPerLane>
__device__ __forceinline__ void route_token_exact(const float* __restrict__ lrow, const float* __restrict__ bias,
                                                  int per_lane, int lane, int top_k, int normalize,
                                                  int32_t* __restrict__ ids, float* __restrict__ weights) {
  double sc[kMaxPerLane];
  float key[kMaxPerLane];
#pragma unroll
  for (int m = 0; m < kMaxPerLane; ++m) {
    if (m < per_lane) {
      const int e = lane + 32 * m;
      sc[m] = route_sigmoid_f64(static_cast<double>(__ldg(lrow + e)));
      key[m] = static_cast<float>(sc[m]) + __ldg(bias + e);
    } else {
      sc[m] = 0.0;
      key[m] = -INFINITY;
    }
  }
  double chosen = 0.0, total = 0.0;
  int my_id = -1;  // lane k keeps choice k
  uint32_t taken = 0;
#pragma unroll 1
  for (int c = 0; c < top_k; ++c) {
    // this lane's best remaining (largest key, then lowest expert)
    float bk = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int m = 0; m < kMaxPerLane; ++m) {
      const int e = lane + 32 * m;
      if (m < per_lane && !((taken >> m) & 1u) && (key[m] > bk || (key[m] == bk && e < be))) {
        bk = key[m];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ok > bk || (ok == bk && oe < be)) {
        bk = ok;
        be = oe;
      }
    }
    // the owner marks it and broadcasts its score
    double s = 0.0;
    if ((be & 31) == lane) {
      const int m = be >> 5;
#pragma unroll
      for (int mm = 0; mm < kMaxPerLane; ++mm)
        if (mm == m) s = sc[mm];
      taken |= 1u << m;
    }
    s = __shfl_sync(0xffffffffu, s, be & 31);
    total += s;
    if (lane == c) {
      my_id = be;
      chosen = s;
    }
  }
  if (lane < top_k) {
    ids[lane] = my_id;
    weights[lane] = static_cast<float>(normalize ? chosen / total : chosen);
  }
}

template <int kMaxPerLane>
__global__ void __launch_bounds__(kThreads) route_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                                                         int32_t* __restrict__ ids, float* __restrict__ weights,
                                                         int64_t T, int E, int top_k, int normalize) {
  extern __shared__ __align__(16) float sm[];  // per warp: 32 candidates' logits, experts, exact keys
  const int lane = threadIdx.x & 31;
  float* c_x = sm + (threadIdx.x >> 5) * 96;
  int* c_id = reinterpret_cast<int*>(c_x + 32);
  float* c_key = c_x + 64;
  const int per_lane = E / 32;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  float bl[kMaxPerLane], xn[kMaxPerLane];  // this lane's biases; the next token's logits
#pragma unroll
  for (int m = 0; m < kMaxPerLane; ++m) bl[m] = m < per_lane ? __ldg(bias + lane + 32 * m) : 0.f;
  int64_t t = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
#pragma unroll
  for (int m = 0; m < kMaxPerLane; ++m) xn[m] = (t < T && m < per_lane) ? __ldg(logits + t * E + lane + 32 * m) : 0.f;
  for (; t < T; t += warps) {
    const float* lrow = logits + t * E;
    float x[kMaxPerLane], ka[kMaxPerLane];
    const int64_t tn = t + warps;
#pragma unroll
    for (int m = 0; m < kMaxPerLane; ++m) {
      x[m] = xn[m];
      xn[m] = (tn < T && m < per_lane) ? __ldg(logits + tn * E + lane + 32 * m) : 0.f;  // in flight meanwhile
    }
    float lmax = -INFINITY;
#pragma unroll
    for (int m = 0; m < kMaxPerLane; ++m) {
      ka[m] = -INFINITY;
      if (m < per_lane) {
        const float k = route_sigmoid_approx(x[m]) + bl[m];
        ka[m] = (k == k) ? k : -INFINITY;  // a NaN key is never a candidate here
      }
      lmax = fmaxf(lmax, ka[m]);
    }
    // L: the k-th largest lane maximum (bitonic sort of the 32 maxima, descending)
    float v = lmax;
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, v, stride);
        v = (((lane & stride) == 0) == ((lane & size) == 0)) ? fmaxf(v, o) : fminf(v, o);
      }
    const float kth = __shfl_sync(0xffffffffu, v, top_k - 1);
    // candidates: an exact key differs from its approximate one by at most 2^-19 + 2^-22 |key| (the
    // sigmoid bound, the FP32 rounding of the exact sigmoid and of the sum), so twice that, with room,
    // is the margin
    const float cut = kth - (0x1p-17f + 0x1p-19f * fabsf(kth));
    unsigned cand[kMaxPerLane];
    int n_cand = 0;
#pragma unroll
    for (int m = 0; m < kMaxPerLane; ++m) {
      cand[m] = __ballot_sync(0xffffffffu, ka[m] >= cut);
      n_cand += __popc(cand[m]);
    }
    bool fast = n_cand >= top_k && n_cand <= 32;  // warp-uniform
    if (fast) {
      int at = 0;
#pragma unroll
      for (int m = 0; m < kMaxPerLane; ++m) {
        if ((cand[m] >> lane) & 1u) {
          const int pos = at + __popc(cand[m] & ((1u << lane) - 1u));
          c_x[pos] = x[m];
          c_id[pos] = lane + 32 * m;
        }
        at += __popc(cand[m]);
      }
      __syncwarp();
      double sc = 0.0;
      float key = -INFINITY;
      int id = 0;
      if (lane < n_cand) {
        id = c_id[lane];
        sc = route_sigmoid_f64(static_cast<double>(c_x[lane]));
        key = static_cast<float>(sc) + __ldg(bias + id);  // as in the exact loop
        c_key[lane] = key;
      }
      __syncwarp();
      fast = !__any_sync(0xffffffffu, lane < n_cand && key != key);
      if (fast) {
        int rank = 0;
        if (lane < n_cand)
          for (int j = 0; j < n_cand; ++j) {
            const float kj = c_key[j];
            rank += (kj > key || (kj == key && c_id[j] < id)) ? 1 : 0;
          }
        const bool chosen = lane < n_cand && rank < top_k;
        double total = chosen ? sc : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        if (chosen) {
          ids[t * top_k + rank] = id;
          weights[t * top_k + rank] = static_cast<float>(normalize ? sc / total : sc);
        }
      }
      __syncwarp();  // the candidate buffers are rewritten for the next token
    }
    if (!fast)
      route_token_exact<kMaxPerLane>(lrow, bias, per_lane, lane, top_k, normalize, ids + t * top_k,
                                     weights + t * top_k);
  }
}

// Two tokens per warp (top_k <= 16), one per half-warp: lane hl = lane & 15 of half h holds experts
// hl + 16 m.  The steps of route_kernel on 16 lanes: the threshold is the k-th largest of the half's
// 16 lane maxima, and a token takes the fast path with at most 16 candidates (one per lane of its
// half for the FP64 sigmoid).  The warp-wide steps -- the sort of the lane maxima, the FP64 sigmoid,
// the rank loop and the sums -- then serve both tokens at once.  Each lane packs its candidates as a
// bit mask; a scan over the half gives each lane its slot, and the candidates' logits are read again
// (from L1) by the lanes that evaluate them.  A token with more than 16 candidates, fewer than k, or
// a NaN among their keys takes the exact loop over all its experts, run by the whole warp.
template <int kMaxPerLane, bool kFull>  // kFull: E == 16 kMaxPerLane, every lane holds kMaxPerLane experts
__global__ void __launch_bounds__(kThreads) route_pair_kernel(const float* __restrict__ logits,
                                                              const float* __restrict__ bias,
                                                              int32_t* __restrict__ ids, float* __restrict__ weights,
                                                              int64_t T, int E, int top_k, int normalize) {
  // per half-warp: 16 candidates' experts, then their keys; after all warps' buffers, the E biases
  extern __shared__ __align__(16) float sm[];
  float* s_bias = sm + (kThreads / 32) * 96;
  for (int e = threadIdx.x; e < E; e += kThreads) s_bias[e] = __ldg(bias + e);
  __syncthreads();  // the only CTA-wide barrier
  const int lane = threadIdx.x & 31;
  const int hl = lane & 15, hbase = lane & 16;
  int* c_id = reinterpret_cast<int*>(sm) + (threadIdx.x >> 5) * 96 + 3 * hbase;
  // a candidate's (key, expert) as one integer that orders like (key descending, expert ascending)
  unsigned long long* c_ord = reinterpret_cast<unsigned long long*>(c_id + 16);
  const int per_lane = kFull ? kMaxPerLane : E / 16;
  const int64_t pair_step = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  float xn[kMaxPerLane];  // the next token's logits
  int64_t pr = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;  // warp-uniform
  {
    const int64_t t = 2 * pr + (hbase >> 4);
#pragma unroll
    for (int m = 0; m < kMaxPerLane; ++m)
      xn[m] = (t < T && m < per_lane) ? __ldg(logits + t * E + hl + 16 * m) : 0.f;
  }
  for (; 2 * pr < T; pr += pair_step) {
    const int64_t t = 2 * pr + (hbase >> 4);
    const bool live = t < T;
    const int64_t tn = t + 2 * pair_step;
    float ka[kMaxPerLane];
    float lmax = -INFINITY;
#pragma unroll
    for (int m = 0; m < kMaxPerLane; ++m) {
      const float x = xn[m];
      xn[m] = (tn < T && m < per_lane) ? __ldg(logits + tn * E + hl + 16 * m) : 0.f;  // in flight meanwhile
      // a NaN key compares false below: never a candidate, and fmaxf passes it over
      ka[m] = m < per_lane ? route_sigmoid_approx(x) + s_bias[hl + 16 * m] : -INFINITY;
      lmax = fmaxf(lmax, ka[m]);
    }
    // L: the k-th largest lane maximum of the half (bitonic sort of its 16 maxima, descending)
    float v = lmax;
#pragma unroll
    for (int size = 2; size <= 16; size <<= 1)
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, v, stride);
        v = (((hl & stride) == 0) == ((hl & size) == 0)) ? fmaxf(v, o) : fminf(v, o);
      }
    const float kth = __shfl_sync(0xffffffffu, v, hbase + top_k - 1);
    // the margin of route_kernel: twice the bound on |exact key - approximate key|, with room
    const float cut = kth - (0x1p-17f + 0x1p-19f * fabsf(kth));
    uint32_t mask = 0;
#pragma unroll
    for (int m = 0; m < kMaxPerLane; ++m)
      if (ka[m] >= cut) mask |= 1u << m;
    if (!live) mask = 0;
    // this lane's first slot: an exclusive scan of the candidate counts over the half
    const int cnt = __popc(mask);
    int scan = cnt;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, scan, o);
      if (hl >= o) scan += y;
    }
    const int n_cand = __shfl_sync(0xffffffffu, scan, hbase + 15);
    bool fast = live && n_cand >= top_k && n_cand <= 16;
    if (fast) {
      int pos = scan - cnt;
      for (uint32_t mm = mask; mm; mm &= mm - 1) c_id[pos++] = hl + 16 * (__ffs(mm) - 1);
    }
    __syncwarp();
    const bool mine = fast && hl < n_cand;
    double sc = 0.0;
    float key = -INFINITY;
    int id = 0;
    if (mine) {
      id = c_id[hl];
      sc = route_sigmoid_f64(static_cast<double>(__ldg(logits + t * E + id)));
      key = static_cast<float>(sc) + s_bias[id];  // as in the exact loop
    }
    // the key's bits made order-preserving as an unsigned integer (-0 taken as +0, which the FP32
    // comparisons of the exact loop treat as equal), above the complemented expert index
    const uint32_t kb = __float_as_uint(key + 0.f);
    const uint32_t ko = (kb & 0x80000000u) ? ~kb : (kb | 0x80000000u);
    const unsigned long long ord = (static_cast<unsigned long long>(ko) << 32) | static_cast<uint32_t>(~id);
    if (mine) c_ord[hl] = ord;
    __syncwarp();
    if ((__ballot_sync(0xffffffffu, mine && key != key) >> hbase) & 0xFFFFu) fast = false;
    int rank = 0;
    if (mine)
      for (int j = 0; j < n_cand; ++j) rank += c_ord[j] > ord ? 1 : 0;
    const bool chosen = fast && mine && rank < top_k;
    double total = chosen ? sc : 0.0;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
    if (chosen) {
      ids[t * top_k + rank] = id;
      weights[t * top_k + rank] = static_cast<float>(normalize ? sc / total : sc);
    }
    const uint32_t slow = __ballot_sync(0xffffffffu, live && !fast);
    __syncwarp();  // the candidate buffers are rewritten for the next pair
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh)
      if ((slow >> (16 * hh)) & 0xFFFFu) {
        const int64_t ts = 2 * pr + hh;
        route_token_exact<(kMaxPerLane + 1) / 2>(logits + ts * E, bias, E / 32, lane, top_k, normalize,
                                                 ids + ts * top_k, weights + ts * top_k);
      }
  }
}

// Dynamic shared memory of route_pair_kernel: per warp two halves of 16 experts and 16 ordering
// keys (8 bytes each), then the biases of at most 256 experts.
constexpr uint32_t kRoutePairSmemBytes = ((kThreads / 32) * 96 + 256) * 4;

// Dynamic shared memory of route_kernel: per warp 32 logits, 32 expert indices and 32 keys.
constexpr uint32_t kRouteSmemBytes = (kThreads / 32) * 96 * 4;

}  // namespace nb
}  // namespace mimo
