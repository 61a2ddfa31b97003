// device_model/cp_async.cuh -- host model of the library's cp_async.cuh: the 16-byte copy lands at
// once (zero fill past src_bytes); the completion arrival is a plain arrival on the barrier.
#pragma once

#include "sm100.cuh"

namespace mimo {
inline void cp_async_16(uint32_t dst_smem, const void* src, uint32_t src_bytes) {
  uint8_t* d = smem_at(dst_smem);
  if (src_bytes) std::memcpy(d, src, src_bytes);
  std::memset(d + src_bytes, 0, 16 - src_bytes);
}
inline void cp_async_commit() {}
inline void cp_async_mbar_arrive_noinc(uint64_t* bar) { mbar_arrive_at(bar); }
template <int N>
inline void cp_async_wait() {}
}  // namespace mimo
