// cudart_host.h -- host definitions of the CUDA runtime calls the library's host code makes, for its
// host build in tests (which links no CUDA runtime): one device with 148 SMs, memory from guarded host
// allocations, copies as memcpy, tensor maps from tensormap_host.h.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdlib>

namespace hemu {
inline bool g_launch_failed = false;
CUresult host_encode_tiled(CUtensorMap* m, CUtensorMapDataType dt, cuuint32_t rank, void* base, const cuuint64_t* dims,
                           const cuuint64_t* strides, const cuuint32_t* box, const cuuint32_t*, CUtensorMapInterleave,
                           CUtensorMapSwizzle sw, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
}

extern "C" {
cudaError_t cudaGetDevice(int* d) { *d = 0; return cudaSuccess; }
cudaError_t cudaDeviceGetAttribute(int* v, enum cudaDeviceAttr a, int) {
  // HEMU_SMS: fewer SMs, so that the persistent kernels' CTAs walk several work units each
  const char* sms = std::getenv("HEMU_SMS");
  *v = a == cudaDevAttrMultiProcessorCount ? (sms ? std::atoi(sms) : 148) : (1 << 20);
  return cudaSuccess;
}
cudaError_t cudaFuncSetAttribute(const void*, enum cudaFuncAttribute, int) { return cudaSuccess; }
cudaError_t cudaMemPoolCreate(cudaMemPool_t* p, const struct cudaMemPoolProps*) {
  *p = reinterpret_cast<cudaMemPool_t>(0x1);
  return cudaSuccess;
}
cudaError_t cudaMemPoolSetAttribute(cudaMemPool_t, enum cudaMemPoolAttr, void*) { return cudaSuccess; }
cudaError_t cudaMemPoolDestroy(cudaMemPool_t) { return cudaSuccess; }
cudaError_t cudaMallocFromPoolAsync(void** p, size_t n, cudaMemPool_t, cudaStream_t) {
  *p = hemu::guarded_alloc(n);
  return cudaSuccess;
}
cudaError_t cudaFreeAsync(void* p, cudaStream_t) { hemu::guarded_free(p); return cudaSuccess; }
cudaError_t cudaGetLastError(void) {
  const bool f = hemu::g_launch_failed;
  hemu::g_launch_failed = false;
  return f ? cudaErrorLaunchFailure : cudaSuccess;
}
cudaError_t cudaMemsetAsync(void* p, int v, size_t n, cudaStream_t) { std::memset(p, v, n); return cudaSuccess; }
cudaError_t cudaMemcpyAsync(void* d, const void* s, size_t n, enum cudaMemcpyKind, cudaStream_t) {
  std::memmove(d, s, n);
  return cudaSuccess;
}
cudaError_t cudaStreamSynchronize(cudaStream_t) { return cudaSuccess; }
cudaError_t cudaEventCreate(cudaEvent_t* e) { *e = reinterpret_cast<cudaEvent_t>(0x1); return cudaSuccess; }
cudaError_t cudaEventRecord(cudaEvent_t, cudaStream_t) { return cudaSuccess; }
cudaError_t cudaEventSynchronize(cudaEvent_t) { return cudaSuccess; }
cudaError_t cudaEventElapsedTime(float* ms, cudaEvent_t, cudaEvent_t) { *ms = 0.f; return cudaSuccess; }
cudaError_t cudaEventDestroy(cudaEvent_t) { return cudaSuccess; }
cudaError_t cudaGetDriverEntryPoint(const char* sym, void** fn, unsigned long long, enum cudaDriverEntryPointQueryResult* q) {
  *fn = std::strcmp(sym, "cuTensorMapEncodeTiled") == 0 ? reinterpret_cast<void*>(&hemu::host_encode_tiled) : nullptr;
  if (q) *q = *fn ? cudaDriverEntryPointSuccess : cudaDriverEntryPointSymbolNotFound;
  return cudaSuccess;
}
cudaError_t cudaGetSymbolAddress(void** p, const void* sym) { *p = const_cast<void*>(sym); return cudaSuccess; }
cudaError_t cudaMemcpyFromSymbol(void* d, const void* sym, size_t n, size_t off, enum cudaMemcpyKind) {
  std::memcpy(d, static_cast<const char*>(sym) + off, n);
  return cudaSuccess;
}
cudaError_t cudaMemcpyToSymbol(const void* sym, const void* s, size_t n, size_t off, enum cudaMemcpyKind) {
  std::memcpy(const_cast<char*>(static_cast<const char*>(sym)) + off, s, n);
  return cudaSuccess;
}
}

// the C++ overloads taking a symbol or a kernel (declared by the runtime header for nvcc only)
template <class T>
cudaError_t cudaMemcpyFromSymbol(void* d, const T& sym, size_t n, size_t off = 0,
                                 enum cudaMemcpyKind k = cudaMemcpyDeviceToHost) {
  return cudaMemcpyFromSymbol(d, static_cast<const void*>(&sym), n, off, k);
}
template <class T>
cudaError_t cudaMemcpyToSymbol(const T& sym, const void* s, size_t n, size_t off = 0,
                               enum cudaMemcpyKind k = cudaMemcpyHostToDevice) {
  return cudaMemcpyToSymbol(static_cast<const void*>(&sym), s, n, off, k);
}
template <class T>
cudaError_t cudaGetSymbolAddress(void** p, const T& sym) {
  *p = const_cast<void*>(static_cast<const void*>(&sym));
  return cudaSuccess;
}
template <class T>
cudaError_t cudaFuncSetAttribute(T*, enum cudaFuncAttribute, int) { return cudaSuccess; }

extern "C" cudaError_t cudaOccupancyMaxActiveClusters(int* n, const void*, const cudaLaunchConfig_t* cfg) {
  *n = static_cast<int>(cfg->gridDim.x / 2);  // one two-CTA cluster per SM pair
  return cudaSuccess;
}
