// params.cuh -- launch parameters shared by the attention forward kernels.
#pragma once

#include <stdint.h>

namespace mimo {

// Per-device error word written by the kernels (bits: kErrTimeout, kErrRange,
// kErrSeqlens) and read/cleared by mimo_attn_check.  Defined once: every
// kernel and the host API are compiled in one translation unit.
static __device__ unsigned int g_mimo_error = 0;

constexpr int kHeadDimQK = 192;
constexpr int kHeadDimV = 128;
constexpr int kRopeDims = 64;
constexpr int kBlockM = 128;  // queries per tile
constexpr int kBlockN = 128;  // keys per tile

struct FwdParams {
  const int32_t* cu_seqlens;  // [num_seqs + 1]
  const float* sink;          // [hq] or nullptr
  uint16_t* out;              // bf16 [T, hq, 128]
  float* lse;                 // [hq, T]
  int32_t num_seqs;
  int32_t total_tokens;
  int32_t max_seqlen;
  int32_t hq;
  int32_t hkv;
  int32_t group;              // hq / hkv
  int32_t window;             // < 0: unbounded (global causal layer)
  float scale_log2;           // log2(e) / sqrt(192)
  float v_scale;
  uint64_t wait_limit_ns;     // bound on every mbarrier wait
  double theta[kRopeDims / 2];  // RoPE inverse frequencies base^(-2i/64)
};

}  // namespace mimo
