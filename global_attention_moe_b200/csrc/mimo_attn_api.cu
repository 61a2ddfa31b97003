// mimo_attn_api.cu -- host side of the C ABI declared in include/mimo_attn.h:
// argument validation (before any CUDA call), TMA tensor-map encoding, kernel
// launch, the device error word and the host-buffer end-to-end entry point.
#include <cublas_v2.h>  // types only: cuBLAS itself is loaded at the first output projection
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <dlfcn.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/mimo_attn.h"
#include "attn_fwd_pipelined.cuh"
#include "attn_fwd_simple.cuh"
#include "attn_fwd_swa.cuh"
#include "attn_fwd_swa_packed.cuh"
#include "attn_decode.cuh"
#include "attn_decode_tc.cuh"
#include "attn_bwd_simple.cuh"
#include "attn_bwd_tc.cuh"
#include "neighbors.cuh"
#include "rope_k_prepass.cuh"
#include "params.cuh"

using namespace mimo;

namespace {

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s bound on any single wait
constexpr int kBwdHeadsPerCta = 2;  // tensor-core backward: query heads of one KV group per CTA (a power of 2)

PFN_cuTensorMapEncodeTiled_v12000 tensormap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D 16-bit view [rows, inner] (row-major) with a {64, box_rows} box and 128-byte swizzle.
bool encode_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows = 128,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto enc = tensormap_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D BF16 view of q [T, Hq, 192] as (dims, heads, tokens) with a {64, G, 128/G} box: one box is a
// 128-row tile of 128/G tokens x the G query heads of one KV group (heads fastest), 128-byte swizzle.
bool encode_q_packed(CUtensorMap* m, const void* q, int hq, int total_tokens, int group) {
  auto enc = tensormap_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kHeadDimQK, (cuuint64_t)hq, (cuuint64_t)total_tokens};
  cuuint64_t strides[2] = {(cuuint64_t)kHeadDimQK * 2, (cuuint64_t)hq * kHeadDimQK * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)(128 / group)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }  // 32-byte row stores

int validate(const void* q, const void* k, const void* v, const float* sink, const int32_t* cu,
             const mimo_attn_dims* d, int layer_kind, int window, double rope_base, int rope_dims, float v_scale,
             const void* out, const float* lse) {
  if (!d) return MIMO_ERR_INVALID_ARG;
  if (layer_kind != MIMO_LAYER_SWA && layer_kind != MIMO_LAYER_GLOBAL) return MIMO_ERR_INVALID_ARG;
  if (d->num_seqs < 1 || d->total_tokens < 0 || d->max_seqlen < 0 || d->num_q_heads < 1 || d->num_kv_heads < 1)
    return MIMO_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads != 0) return MIMO_ERR_INVALID_ARG;
  if (d->max_seqlen > d->total_tokens) return MIMO_ERR_INVALID_ARG;
  if (d->head_dim_qk < 1 || d->head_dim_v < 1) return MIMO_ERR_INVALID_ARG;
  if (d->head_dim_qk != kHeadDimQK || d->head_dim_v != kHeadDimV) return MIMO_ERR_UNSUPPORTED;
  if (rope_dims < 0 || rope_dims % 2 != 0 || rope_dims > d->head_dim_qk) return MIMO_ERR_INVALID_ARG;
  if (rope_dims != kRopeDims) return MIMO_ERR_UNSUPPORTED;
  if (!(rope_base > 0.0) || !std::isfinite(rope_base)) return MIMO_ERR_INVALID_ARG;
  if (!std::isfinite(v_scale)) return MIMO_ERR_INVALID_ARG;
  if (layer_kind == MIMO_LAYER_SWA && window < 0) return MIMO_ERR_INVALID_ARG;
  if (layer_kind == MIMO_LAYER_GLOBAL && sink != nullptr) return MIMO_ERR_INVALID_ARG;
  if ((int64_t)d->num_q_heads * d->total_tokens > INT32_MAX) return MIMO_ERR_UNSUPPORTED;
  // unit indices of the two-head kernels stay below 2^31
  if ((int64_t)(d->num_q_heads / 2 + 1) * ((int64_t)d->total_tokens / kBlockM + 1 + d->num_seqs) > INT32_MAX)
    return MIMO_ERR_UNSUPPORTED;
  if (!cu) return MIMO_ERR_INVALID_ARG;
  if (d->total_tokens > 0) {
    if (!q || !k || !v || !out || !lse) return MIMO_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned32(out) || !aligned16(lse))
      return MIMO_ERR_INVALID_ARG;
  }
  if (sink && (reinterpret_cast<uintptr_t>(sink) & 3u)) return MIMO_ERR_INVALID_ARG;
  return MIMO_OK;
}

void fill_params(FwdParams& P, const float* sink, const int32_t* cu, const mimo_attn_dims* d, int layer_kind,
                 int window, double rope_base, float v_scale, void* out, float* lse) {
  std::memset(&P, 0, sizeof P);
  P.cu_seqlens = cu;
  P.sink = sink;
  P.out = static_cast<uint16_t*>(out);
  P.lse = lse;
  P.num_seqs = d->num_seqs;
  P.total_tokens = d->total_tokens;
  P.max_seqlen = d->max_seqlen;
  P.hq = d->num_q_heads;
  P.hkv = d->num_kv_heads;
  P.group = d->num_q_heads / d->num_kv_heads;
  P.window = (layer_kind == MIMO_LAYER_GLOBAL) ? -1 : window;
  P.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHeadDimQK)));
  P.v_scale = v_scale;
  P.wait_limit_ns = kDefaultWaitLimitNs;
  for (int i = 0; i < kRopeDims / 2; ++i) P.theta[i] = std::pow(rope_base, -2.0 * i / kRopeDims);
}

std::atomic<int> g_kernel_choice{MIMO_KERNEL_AUTO};

enum class Path { Simple, Pipelined, Window, Packed };

// Chooses the kernel for one call from the process-wide choice and the shape.
int select_path(const FwdParams& P, Path& path) {
  const bool even = P.group % 2 == 0;
  const bool short_window = P.window >= 0 && P.window <= kBlockN;
  const bool packs = short_window && (P.group == 4 || P.group == 8);
  switch (g_kernel_choice.load()) {
    case MIMO_KERNEL_SIMPLE: path = Path::Simple; return MIMO_OK;
    case MIMO_KERNEL_PIPELINED: path = Path::Pipelined; return even ? MIMO_OK : MIMO_ERR_UNSUPPORTED;
    case MIMO_KERNEL_WINDOW: path = Path::Window; return (even && short_window) ? MIMO_OK : MIMO_ERR_UNSUPPORTED;
    case MIMO_KERNEL_WINDOW_PACKED: path = Path::Packed; return packs ? MIMO_OK : MIMO_ERR_UNSUPPORTED;
    default:
      path = packs ? Path::Packed : !even ? Path::Simple : (short_window ? Path::Window : Path::Pipelined);
      return MIMO_OK;
  }
}

// Raises the dynamic shared memory limit of every kernel (once per device).
bool set_smem_attributes() {
  return cudaFuncSetAttribute(attn_fwd_simple_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              simple::kSmemBytes) == cudaSuccess &&
         cudaFuncSetAttribute(attn_fwd_pipelined_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              pipe::kSmemBytes) == cudaSuccess &&
         cudaFuncSetAttribute(attn_fwd_swa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              pipe::kSmemBytes) == cudaSuccess &&
         cudaFuncSetAttribute(attn_fwd_swa_packed_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              pk::Shape<4>::kSmemBytes) == cudaSuccess &&
         cudaFuncSetAttribute(attn_fwd_swa_packed_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              pk::Shape<8>::kSmemBytes) == cudaSuccess &&
         cudaFuncSetAttribute(dec::attn_decode_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              dec::kSmemBytes) == cudaSuccess &&
         cudaFuncSetAttribute(attn_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              dtc::kSmemBytes) == cudaSuccess;
}

// The backward's shared-memory limit, raised on its first call on each device (so that a failure here
// concerns the backward only).
bool bwd_attributes_ready(int dev) {
  static std::atomic<int> state[64];  // 0 unknown, 1 ready, -1 failed
  if (dev < 0 || dev >= 64) return false;
  if (state[dev].load() == 0)
    state[dev].store(cudaFuncSetAttribute(bwd::bwd_main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          bwd::kSmemBytes) == cudaSuccess &&
                             cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  bwdtc::kSmemBytes) == cudaSuccess
                         ? 1
                         : -1);
  return state[dev].load() == 1;
}

std::atomic<int> g_decode_choice{MIMO_DECODE_AUTO};
std::atomic<int> g_bwd_choice{0};  // 0 auto (tensor cores), 1 CUDA cores, 2 tensor cores

// Persistent grid of the two-head kernels: one CTA per SM, at most one per unit.
int persistent_grid(const FwdParams& P, int sms) {
  const long long units = (long long)(P.hq / 2) * ((P.total_tokens + kBlockM - 1) / kBlockM + P.num_seqs);
  return (int)std::min<long long>(units, sms);
}

void launch_two_head(Path path, int grid, const CUtensorMap& tq, const CUtensorMap& tkr, const CUtensorMap& tk,
                     const CUtensorMap& tv, const FwdParams& P, cudaStream_t stream) {
  if (path == Path::Window)
    attn_fwd_swa_kernel<<<grid, pipe::kThreads, pipe::kSmemBytes, stream>>>(tq, tkr, tk, tv, P);
  else
    attn_fwd_pipelined_kernel<<<grid, pipe::kThreads, pipe::kSmemBytes, stream>>>(tq, tkr, tk, tv, P);
}

// The packed window kernel: no scratch, one persistent CTA per SM (at most one per tile).
int launch_packed(const void* q, const void* k, const void* v, const FwdParams& P, int sms,
                  std::pair<cudaEvent_t, cudaEvent_t>* ev, cudaStream_t stream) {
  const int qt = 128 / P.group;
  CUtensorMap tq, tk, tv;
  if (!encode_q_packed(&tq, q, P.hq, P.total_tokens, P.group) ||
      !encode_2d(&tk, k, (uint64_t)P.hkv * kHeadDimQK, P.total_tokens, pk::kBlk) ||
      !encode_2d(&tv, v, (uint64_t)P.hkv * kHeadDimV, P.total_tokens, pk::kBlk))
    return MIMO_ERR_CUDA;
  const long long tiles = (long long)P.hkv * ((long long)P.total_tokens / qt + P.num_seqs);
  const int grid = (int)std::min<long long>(tiles, sms);
  if (ev) cudaEventRecord(ev->first, stream);
  if (P.group == 8)
    attn_fwd_swa_packed_kernel<8><<<grid, pk::kThreads, pk::Shape<8>::kSmemBytes, stream>>>(tq, tk, tv, P);
  else
    attn_fwd_swa_packed_kernel<4><<<grid, pk::kThreads, pk::Shape<4>::kSmemBytes, stream>>>(tq, tk, tv, P);
  const bool ok = cudaGetLastError() == cudaSuccess;
  if (ev) cudaEventRecord(ev->second, stream);
  return ok ? MIMO_OK : MIMO_ERR_CUDA;
}

// Kernel timing: while enabled, each forward records an event pair around its
// attention kernel (library-owned events, per device, reused across sessions).
struct ProfileState {
  std::mutex mu;
  bool enabled = false;
  int stride = 1;         // record every stride-th launch
  long long launches = 0;  // launches seen since profiling started
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pairs[64];
  size_t used[64] = {};
};
ProfileState& profile_state() {
  static ProfileState st;
  return st;
}

// Returns the event pair to record around the next attention kernel, or null when not profiling.
std::pair<cudaEvent_t, cudaEvent_t>* profile_slot(int dev) {
  ProfileState& st = profile_state();
  std::lock_guard<std::mutex> lock(st.mu);
  if (!st.enabled || dev < 0 || dev >= 64) return nullptr;
  if (st.launches++ % st.stride != 0) return nullptr;
  auto& v = st.pairs[dev];
  if (st.used[dev] == v.size()) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess) return nullptr;
    if (cudaEventCreate(&b) != cudaSuccess) {
      cudaEventDestroy(a);
      return nullptr;
    }
    v.emplace_back(a, b);
  }
  return &v[st.used[dev]++];
}

struct DeviceInfo {
  int sms = 0;
  bool kernels_ready = false;  // dynamic shared memory limits raised
  cudaMemPool_t pool = nullptr;  // stream-ordered scratch; returned to the device at the next synchronization
};

DeviceInfo* device_info(int dev) {
  static DeviceInfo infos[64];
  static std::mutex mu;
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo& d = infos[dev];
  if (d.sms == 0) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
    d.kernels_ready = set_smem_attributes();
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof props);
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    // Release threshold 0: memory freed (stream-ordered) by a call is reused by later calls on the same
    // stream without synchronizing, and goes back to the device at the next synchronization, so the
    // library keeps no scratch between synchronized calls.
    if (cudaMemPoolCreate(&d.pool, &props) == cudaSuccess) {
      uint64_t keep = 0;
      if (cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) {
        cudaMemPoolDestroy(d.pool);
        d.pool = nullptr;
      }
    } else {
      d.pool = nullptr;
    }
  }
  return &d;
}

// cuBLAS for the output projection (a plain BF16 GEMM), loaded with dlopen at its first call so that
// nothing else in the library depends on it; one handle per device, used under the lock.
struct CublasApi {
  bool tried = false, ok = false;
  decltype(&cublasCreate_v2) create = nullptr;
  decltype(&cublasSetStream_v2) set_stream = nullptr;
  // the C symbol (the header adds a C++ overload taking the compute type as a cudaDataType)
  cublasStatus_t (*gemm_ex)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int, const void*,
                            const void*, cudaDataType, int, const void*, cudaDataType, int, const void*, void*,
                            cudaDataType, int, cublasComputeType_t, cublasGemmAlgo_t) = nullptr;
  cublasHandle_t handles[64] = {};
};

// y[T, N] = x[T, K] . w[N, K]^T, BF16 in and out, FP32 accumulation (row-major operands; in cuBLAS's
// column-major terms y^T = w . x^T with w read transposed).
int gemm_bf16_nt(const void* x, const void* w, int T, int K, int N, void* y, cudaStream_t stream) {
  static CublasApi a;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MIMO_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!a.tried) {
    a.tried = true;
    if (void* lib = dlopen("libcublas.so.12", RTLD_NOW | RTLD_LOCAL)) {
      a.create = reinterpret_cast<decltype(a.create)>(dlsym(lib, "cublasCreate_v2"));
      a.set_stream = reinterpret_cast<decltype(a.set_stream)>(dlsym(lib, "cublasSetStream_v2"));
      a.gemm_ex = reinterpret_cast<decltype(a.gemm_ex)>(dlsym(lib, "cublasGemmEx"));
      a.ok = a.create && a.set_stream && a.gemm_ex;
    }
  }
  if (!a.ok) return MIMO_ERR_CUDA;
  if (!a.handles[dev] && a.create(&a.handles[dev]) != CUBLAS_STATUS_SUCCESS) {
    a.handles[dev] = nullptr;
    return MIMO_ERR_CUDA;
  }
  if (a.set_stream(a.handles[dev], stream) != CUBLAS_STATUS_SUCCESS) return MIMO_ERR_CUDA;
  const float alpha = 1.f, beta = 0.f;
  const cublasStatus_t st = a.gemm_ex(a.handles[dev], CUBLAS_OP_T, CUBLAS_OP_N, N, T, K, &alpha, w, CUDA_R_16BF, K, x,
                                      CUDA_R_16BF, K, &beta, y, CUDA_R_16BF, N, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
  return st == CUBLAS_STATUS_SUCCESS ? MIMO_OK : MIMO_ERR_CUDA;
}

int launch(const void* q, const void* k, const void* v, const FwdParams& P, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MIMO_ERR_CUDA;
  DeviceInfo* info = device_info(dev);
  if (!info) return MIMO_ERR_CUDA;
  if (P.max_seqlen == 0) return MIMO_OK;
  Path path;
  if (const int sel = select_path(P, path); sel != MIMO_OK) return sel;
  if (!info->kernels_ready) return MIMO_ERR_CUDA;
  if (path == Path::Packed) return launch_packed(q, k, v, P, info->sms, profile_slot(dev), stream);
  const bool two_head = path != Path::Simple;
  CUtensorMap tq, tk, tv;
  if (!encode_2d(&tq, q, (uint64_t)P.hq * kHeadDimQK, P.total_tokens) ||
      !encode_2d(&tk, k, (uint64_t)P.hkv * kHeadDimQK, P.total_tokens) ||
      !encode_2d(&tv, v, (uint64_t)P.hkv * kHeadDimV, P.total_tokens, two_head ? 64 : 128))
    return MIMO_ERR_CUDA;
  if (!info->kernels_ready) return MIMO_ERR_CUDA;
  if (!two_head) {
    dim3 grid((P.max_seqlen + kBlockM - 1) / kBlockM, P.num_seqs, P.hq);
    attn_fwd_simple_kernel<<<grid, simple::kThreads, simple::kSmemBytes, stream>>>(tq, tk, tv, P);
    return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
  }
  if (!info->pool) return MIMO_ERR_CUDA;
  // K's rope dims, rotated once: transient scratch from the library's stream-ordered pool
  const size_t kr_rows = (size_t)P.total_tokens * P.hkv;
  void* k_rope = nullptr;
  if (cudaMallocFromPoolAsync(&k_rope, kr_rows * kRopeDims * 2, info->pool, stream) != cudaSuccess)
    return MIMO_ERR_CUDA;
  RopeKParams R;
  std::memset(&R, 0, sizeof R);
  R.k = static_cast<const uint16_t*>(k);
  R.k_rope = static_cast<uint16_t*>(k_rope);
  R.cu_seqlens = P.cu_seqlens;
  R.num_seqs = P.num_seqs;
  R.total_tokens = P.total_tokens;
  R.hkv = P.hkv;
  for (int i = 0; i < kRopeDims / 2; ++i) R.theta[i] = P.theta[i];
  const long long threads = (long long)kr_rows * 4;
  rope_k_prepass_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(R);
  int st = cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
  CUtensorMap tkr;
  if (st == MIMO_OK && !encode_2d(&tkr, k_rope, (uint64_t)P.hkv * kRopeDims, P.total_tokens, 128,
                                  CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
    st = MIMO_ERR_CUDA;
  if (st == MIMO_OK) {
    auto* ev = profile_slot(dev);
    if (ev) cudaEventRecord(ev->first, stream);
    launch_two_head(path, persistent_grid(P, info->sms), tq, tkr, tk, tv, P, stream);
    if (cudaGetLastError() != cudaSuccess) st = MIMO_ERR_CUDA;
    if (ev) cudaEventRecord(ev->second, stream);
  }
  if (cudaFreeAsync(k_rope, stream) != cudaSuccess) st = MIMO_ERR_CUDA;
  return st;
}

__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the bounded wait must give up.
  const bool ok = mbar_wait(&bar, 0, limit_ns);
  if (!ok && threadIdx.x == 0) atomicOr(&g_mimo_error, kErrTimeout);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------------------
// Scratch for mimo_attn_fwd_noalloc.  Some callers cannot allocate device
// memory while they run: a framework that has already reserved the device
// for its own caching allocator, or a serving loop that forbids allocation on
// its hot path.  For them the rotated-K scratch lives in this file-scope
// array instead of the stream-ordered pool.  Every GPU that loads the library
// holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB: T * Hkv <= 262144 rows of 64 FP16 dims
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocInfo {
  int sms = 0;
  bool ready = false;
  void* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};

// Per-device set-up, done by the first no-alloc call on that device with the
// device current: kernel attributes, SM count and the scratch array's device
// address (in host code the array's name is only a host-side stand-in).
NoAllocInfo* noalloc_info(int dev) {
  static NoAllocInfo infos[64];
  static std::mutex mu;
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  NoAllocInfo& d = infos[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
    if (!set_smem_attributes()) return nullptr;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return nullptr;
    d.scratch = ptr;
    d.ready = true;
  }
  return &d;
}

int launch_noalloc(const void* q, const void* k, const void* v, const FwdParams& P, cudaStream_t stream) {
  Path path;
  if (const int sel = select_path(P, path); sel != MIMO_OK) return sel;
  const bool pipelined = path == Path::Pipelined || path == Path::Window;  // the kernels that read pre-rotated K
  const size_t kr_rows = (size_t)P.total_tokens * P.hkv;
  // The size check comes before any CUDA call, so that it holds on a machine without a GPU too.
  if (pipelined && kr_rows * kRopeDims * 2 > kNoAllocScratchBytes) return MIMO_ERR_SCRATCH_LIMIT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MIMO_ERR_CUDA;
  NoAllocInfo* info = noalloc_info(dev);
  if (!info) return MIMO_ERR_CUDA;
  if (P.max_seqlen == 0) return MIMO_OK;
  if (path == Path::Packed) return launch_packed(q, k, v, P, info->sms, nullptr, stream);  // needs no scratch
  CUtensorMap tq, tk, tv;
  if (!encode_2d(&tq, q, (uint64_t)P.hq * kHeadDimQK, P.total_tokens) ||
      !encode_2d(&tk, k, (uint64_t)P.hkv * kHeadDimQK, P.total_tokens) ||
      !encode_2d(&tv, v, (uint64_t)P.hkv * kHeadDimV, P.total_tokens, pipelined ? 64 : 128))
    return MIMO_ERR_CUDA;
  if (!pipelined) {
    dim3 grid((P.max_seqlen + kBlockM - 1) / kBlockM, P.num_seqs, P.hq);
    attn_fwd_simple_kernel<<<grid, simple::kThreads, simple::kSmemBytes, stream>>>(tq, tk, tv, P);
    return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
  }
  // The pre-pass overwrites every scratch row the attention kernel reads, so
  // nothing needs clearing between calls.
  RopeKParams R;
  std::memset(&R, 0, sizeof R);
  R.k = static_cast<const uint16_t*>(k);
  R.k_rope = static_cast<uint16_t*>(info->scratch);
  R.cu_seqlens = P.cu_seqlens;
  R.num_seqs = P.num_seqs;
  R.total_tokens = P.total_tokens;
  R.hkv = P.hkv;
  for (int i = 0; i < kRopeDims / 2; ++i) R.theta[i] = P.theta[i];
  const long long threads = (long long)kr_rows * 4;
  rope_k_prepass_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(R);
  if (cudaGetLastError() != cudaSuccess) return MIMO_ERR_CUDA;
  CUtensorMap tkr;
  if (!encode_2d(&tkr, info->scratch, (uint64_t)P.hkv * kRopeDims, P.total_tokens, 128,
                 CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
    return MIMO_ERR_CUDA;
  launch_two_head(path, persistent_grid(P, info->sms), tq, tkr, tk, tv, P, stream);
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}

// Query rows per KV head (q_len x Hq/Hkv) that one decode call accepts: 8192 row tiles of the CUDA-core
// kernel (prefill chunks of up to 65536 tokens at 16 query heads per KV head).
constexpr int64_t kMaxDecodeRows = INT64_C(1) << 20;

int validate_decode(const void* q, const void* kc, const void* vc, const int32_t* idx, const int32_t* indptr,
                    const int32_t* cu_q, const float* sink, const mimo_decode_dims* d, int layer_kind, int window,
                    double rope_base, int rope_dims, float v_scale, const void* out, const float* lse) {
  if (!d) return MIMO_ERR_INVALID_ARG;
  if (layer_kind != MIMO_LAYER_SWA && layer_kind != MIMO_LAYER_GLOBAL) return MIMO_ERR_INVALID_ARG;
  if (d->num_seqs < 1 || d->total_q < 0 || d->total_kv < 0 || d->cache_rows < 0 || d->max_q_len < 0 ||
      d->max_kv_len < 0 || d->num_q_heads < 1 || d->num_kv_heads < 1)
    return MIMO_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads != 0) return MIMO_ERR_INVALID_ARG;
  if (d->max_q_len > d->max_kv_len || d->max_q_len > d->total_q || d->max_kv_len > d->total_kv)
    return MIMO_ERR_INVALID_ARG;
  if (d->total_kv > 0 && d->cache_rows < 1) return MIMO_ERR_INVALID_ARG;
  if (d->head_dim_qk < 1 || d->head_dim_v < 1) return MIMO_ERR_INVALID_ARG;
  if (d->head_dim_qk != kHeadDimQK || d->head_dim_v != kHeadDimV) return MIMO_ERR_UNSUPPORTED;
  if (rope_dims < 0 || rope_dims % 2 != 0 || rope_dims > d->head_dim_qk) return MIMO_ERR_INVALID_ARG;
  if (rope_dims != kRopeDims) return MIMO_ERR_UNSUPPORTED;
  if (!(rope_base > 0.0) || !std::isfinite(rope_base)) return MIMO_ERR_INVALID_ARG;
  if (!std::isfinite(v_scale)) return MIMO_ERR_INVALID_ARG;
  if (layer_kind == MIMO_LAYER_SWA && window < 0) return MIMO_ERR_INVALID_ARG;
  if (layer_kind == MIMO_LAYER_GLOBAL && sink != nullptr) return MIMO_ERR_INVALID_ARG;
  if ((int64_t)d->max_q_len * (d->num_q_heads / d->num_kv_heads) > kMaxDecodeRows) return MIMO_ERR_UNSUPPORTED;
  if ((int64_t)d->cache_rows * d->num_kv_heads * kHeadDimQK > INT64_C(1) << 40) return MIMO_ERR_UNSUPPORTED;
  if (!indptr || !cu_q) return MIMO_ERR_INVALID_ARG;
  if (d->total_q > 0) {
    if (!q || !out || !lse || (d->total_kv > 0 && (!kc || !vc || !idx))) return MIMO_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned32(out) || !aligned16(lse) || (kc && !aligned16(kc)) || (vc && !aligned16(vc)))
      return MIMO_ERR_INVALID_ARG;
  }
  if (sink && (reinterpret_cast<uintptr_t>(sink) & 3u)) return MIMO_ERR_INVALID_ARG;
  return MIMO_OK;
}

int launch_decode(const void* q, const void* kc, const void* vc, const int32_t* idx, const int32_t* indptr,
                  const int32_t* cu_q, const float* sink, const mimo_decode_dims* d, int layer_kind, int window,
                  double rope_base, float v_scale, void* out, float* lse, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MIMO_ERR_CUDA;
  DeviceInfo* info = device_info(dev);
  if (!info || !info->kernels_ready || !info->pool) return MIMO_ERR_CUDA;
  dec::DecParams P;
  std::memset(&P, 0, sizeof P);
  P.q = static_cast<const uint16_t*>(q);
  P.k_cache = static_cast<const uint16_t*>(kc);
  P.v_cache = static_cast<const uint16_t*>(vc);
  P.kv_indices = idx;
  P.kv_indptr = indptr;
  P.cu_q = cu_q;
  P.sink = sink;
  P.out = static_cast<uint16_t*>(out);
  P.lse = lse;
  P.num_seqs = d->num_seqs;
  P.total_q = d->total_q;
  P.total_kv = d->total_kv;
  P.cache_rows = d->cache_rows;
  P.hq = d->num_q_heads;
  P.hkv = d->num_kv_heads;
  P.group = d->num_q_heads / d->num_kv_heads;
  P.window = (layer_kind == MIMO_LAYER_GLOBAL) ? -1 : window;
  P.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHeadDimQK)));
  P.v_scale = v_scale;
  P.wait_limit_ns = kDefaultWaitLimitNs;
  for (int i = 0; i < kRopeDims / 2; ++i) P.theta[i] = std::pow(rope_base, -2.0 * i / kRopeDims);
  // The query rows of a KV head are cut into 128-row tiles (one M = 128 accumulator of the tensor-core
  // kernel): chunked prefill runs on either kernel with the tile as one more dimension of its work.
  const long long all_rows = (long long)d->max_q_len * P.group;
  const int choice = g_decode_choice.load();
  const bool tensor = choice != MIMO_DECODE_CUDA_CORES;
  P.qtiles = (int)std::max<long long>(1, (all_rows + dec::kMaxRows - 1) / dec::kMaxRows);
  // Keys one sequence's queries can see, at most; split them so that the work covers the SMs a few
  // times over (tensor-core kernel: persistent, one CTA per SM walking about six (sequence, KV head,
  // split) items; CUDA-core kernel: one CTA per (split, row tile) item, about two per SM).
  const long long span = (P.window >= 0) ? std::min<long long>(d->max_kv_len, (long long)P.window + d->max_q_len)
                                         : (long long)d->max_kv_len;
  const long long base_ctas = (long long)d->num_seqs * P.hkv * P.qtiles;  // both kernels tile the rows
  const long long chunk = tensor ? dtc::kChunk : dec::kChunk;
  const long long target = (tensor ? 6LL : 2LL) * info->sms;
  long long splits = std::max<long long>(1, (target + base_ctas - 1) / base_ctas);
  const long long min_split = tensor ? 256 : 64;  // fewer keys per CTA do not pay for its set-up
  splits = std::min<long long>(splits, std::max<long long>(1, (span + min_split - 1) / min_split));
  long long split_keys = (span + splits - 1) / splits;
  split_keys = std::max<long long>(chunk, (split_keys + chunk - 1) / chunk * chunk);
  splits = std::max<long long>(1, (span + split_keys - 1) / split_keys);
  if (splits > 65535 || d->num_seqs > 65535 || P.hkv > 65535) return MIMO_ERR_UNSUPPORTED;  // grid limits
  P.splits = (int)splits;
  P.split_keys = (int)split_keys;
  const size_t slots = (size_t)d->total_q * P.hq * splits;
  const size_t part_bytes = align256(slots * (kHeadDimV * 4 + 8));
  void* part = nullptr;
  if (cudaMallocFromPoolAsync(&part, part_bytes + 256, info->pool, stream) != cudaSuccess) return MIMO_ERR_CUDA;
  P.part_o = static_cast<float*>(part);
  P.part_ml = P.part_o + slots * kHeadDimV;
  P.item_counter = reinterpret_cast<unsigned long long*>(static_cast<char*>(part) + part_bytes);
  int st = MIMO_OK;
  if (tensor && cudaMemsetAsync(P.item_counter, 0, sizeof(unsigned long long), stream) != cudaSuccess)
    st = MIMO_ERR_CUDA;
  if (st == MIMO_OK) {
    if (tensor) {  // persistent: at most one CTA per SM, items from the shared counter
      const long long items = splits * P.qtiles * P.hkv * (long long)d->num_seqs;
      attn_decode_tc_kernel<<<(unsigned)std::min<long long>(items, info->sms), dtc::kThreads, dtc::kSmemBytes,
                              stream>>>(P);
    } else {
      dim3 grid((unsigned)(splits * P.qtiles), (unsigned)P.hkv, (unsigned)d->num_seqs);
      dec::attn_decode_partial_kernel<<<grid, dec::kThreads, dec::kSmemBytes, stream>>>(P);
    }
    if (cudaGetLastError() != cudaSuccess) st = MIMO_ERR_CUDA;
  }
  const long long warps = (long long)d->total_q * P.hq;
  // with one key split the tensor-core kernel writes the final rows itself (no partials to merge)
  if (st == MIMO_OK && !(tensor && splits == 1)) {
    dec::attn_decode_combine_kernel<<<(unsigned)((warps * 32 + dec::kThreads - 1) / dec::kThreads), dec::kThreads,
                                      0, stream>>>(P);
    if (cudaGetLastError() != cudaSuccess) st = MIMO_ERR_CUDA;
  }
  if (cudaFreeAsync(part, stream) != cudaSuccess) st = MIMO_ERR_CUDA;
  return st;
}

int launch_bwd(const void* q, const void* k, const void* v, const float* sink, const int32_t* cu,
               const mimo_attn_dims* d, int layer_kind, int window, double rope_base, float v_scale,
               const void* out, const float* lse, const void* dout, const float* dlse, float* dq, float* dk,
               float* dv, float* dsink, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MIMO_ERR_CUDA;
  DeviceInfo* info = device_info(dev);
  if (!info || !info->kernels_ready || !info->pool) return MIMO_ERR_CUDA;
  if (!bwd_attributes_ready(dev)) return MIMO_ERR_CUDA;
  bwd::BwdParams P;
  std::memset(&P, 0, sizeof P);
  P.q = static_cast<const uint16_t*>(q);
  P.k = static_cast<const uint16_t*>(k);
  P.v = static_cast<const uint16_t*>(v);
  P.sink = sink;
  P.cu_seqlens = cu;
  P.out = static_cast<const uint16_t*>(out);
  P.lse = lse;
  P.dout = static_cast<const uint16_t*>(dout);
  P.dlse = dlse;
  P.dq = dq;
  P.dk = dk;
  P.dv = dv;
  P.dsink = dsink;
  P.num_seqs = d->num_seqs;
  P.total_tokens = d->total_tokens;
  P.max_seqlen = d->max_seqlen;
  P.hq = d->num_q_heads;
  P.hkv = d->num_kv_heads;
  P.group = d->num_q_heads / d->num_kv_heads;
  P.window = (layer_kind == MIMO_LAYER_GLOBAL) ? -1 : window;
  P.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(kHeadDimQK)));
  P.v_scale = v_scale;
  for (int i = 0; i < kRopeDims / 2; ++i) P.theta[i] = std::pow(rope_base, -2.0 * i / kRopeDims);
  if (d->num_seqs > 65535 || d->num_q_heads > 65535) return MIMO_ERR_UNSUPPORTED;  // grid limits
  void* scratch = nullptr;
  const size_t n_d = (size_t)d->total_tokens * d->num_q_heads;
  if (cudaMallocFromPoolAsync(&scratch, n_d * sizeof(float), info->pool, stream) != cudaSuccess) return MIMO_ERR_CUDA;
  P.D = static_cast<float*>(scratch);
  int st = MIMO_OK;
  if (g_bwd_choice.load() != 1) {  // tensor cores: dq / dk / dv / dsink accumulate with atomics
    const size_t T = (size_t)d->total_tokens;
    CUtensorMap tq, tk, tv, to;
    // dq / dk / dv are zeroed by the prep kernel, dsink here
    if ((dsink && cudaMemsetAsync(dsink, 0, P.hq * 4, stream) != cudaSuccess) ||
        !encode_2d(&tq, q, (uint64_t)P.hq * kHeadDimQK, T) || !encode_2d(&tk, k, (uint64_t)P.hkv * kHeadDimQK, T) ||
        !encode_2d(&tv, v, (uint64_t)P.hkv * kHeadDimV, T) || !encode_2d(&to, dout, (uint64_t)P.hq * kHeadDimV, T)) {
      st = MIMO_ERR_CUDA;
    } else {
      bwdtc_prep_kernel<<<info->sms * 8, 256, 0, stream>>>(P);
      if (cudaGetLastError() != cudaSuccess) st = MIMO_ERR_CUDA;
      if (st == MIMO_OK && d->max_seqlen > 0) {
        // query heads per CTA: the most, up to kBwdHeadsPerCta, that divide the KV group
        int hpc = 1;
        for (int c = kBwdHeadsPerCta; c > 1; c /= 2)
          if (P.group % c == 0) {
            hpc = c;
            break;
          }
        dim3 grid((unsigned)((d->max_seqlen + 127) / 128), (unsigned)d->num_seqs, (unsigned)(d->num_q_heads / hpc));
        attn_bwd_tc_kernel<<<grid, bwdtc::kThreads, bwdtc::kSmemBytes, stream>>>(tq, tk, tv, to, P, hpc,
                                                                                 kDefaultWaitLimitNs);
        if (cudaGetLastError() != cudaSuccess) st = MIMO_ERR_CUDA;
      }
    }
    if (cudaFreeAsync(scratch, stream) != cudaSuccess) st = MIMO_ERR_CUDA;
    return st;
  }
  bwd::bwd_prep_kernel<<<info->sms * 8, bwd::kThreads, 0, stream>>>(P);
  if (cudaGetLastError() != cudaSuccess) st = MIMO_ERR_CUDA;
  if (st == MIMO_OK && d->max_seqlen > 0) {
    dim3 grid((unsigned)((d->max_seqlen + bwd::kRows - 1) / bwd::kRows), (unsigned)d->num_seqs, (unsigned)d->num_q_heads);
    bwd::bwd_main_kernel<<<grid, bwd::kThreads, bwd::kSmemBytes, stream>>>(P);
    if (cudaGetLastError() != cudaSuccess) st = MIMO_ERR_CUDA;
  }
  if (st == MIMO_OK) {
    const long long n = (long long)d->total_tokens * d->num_kv_heads * (kRopeDims / 2);
    if (n > 0) {
      bwd::bwd_finalize_kernel<<<(unsigned)((n + bwd::kThreads - 1) / bwd::kThreads), bwd::kThreads, 0, stream>>>(P);
      if (cudaGetLastError() != cudaSuccess) st = MIMO_ERR_CUDA;
    }
  }
  if (cudaFreeAsync(scratch, stream) != cudaSuccess) st = MIMO_ERR_CUDA;
  return st;
}
}  // namespace

extern "C" {

int mimo_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_indices,
                     const int32_t* kv_indptr, const int32_t* cu_q, const float* sink, const mimo_decode_dims* dims,
                     int layer_kind, int window, double rope_base, int rope_dims, float v_scale, void* out,
                     float* lse, void* stream) {
  int st = validate_decode(q, k_cache, v_cache, kv_indices, kv_indptr, cu_q, sink, dims, layer_kind, window,
                           rope_base, rope_dims, v_scale, out, lse);
  if (st != MIMO_OK) return st;
  if (dims->total_q == 0) return MIMO_OK;
  return launch_decode(q, k_cache, v_cache, kv_indices, kv_indptr, cu_q, sink, dims, layer_kind, window, rope_base,
                       v_scale, out, lse, static_cast<cudaStream_t>(stream));
}


int mimo_attn_fwd(const void* q, const void* k, const void* v, const float* sink, const int32_t* cu_seqlens,
                  const mimo_attn_dims* dims, int layer_kind, int window, double rope_base, int rope_dims,
                  float v_scale, void* out, float* lse, void* stream) {
  int st = validate(q, k, v, sink, cu_seqlens, dims, layer_kind, window, rope_base, rope_dims, v_scale, out, lse);
  if (st != MIMO_OK) return st;
  if (dims->total_tokens == 0) return MIMO_OK;
  FwdParams P;
  fill_params(P, sink, cu_seqlens, dims, layer_kind, window, rope_base, v_scale, out, lse);
  return launch(q, k, v, P, static_cast<cudaStream_t>(stream));
}

size_t mimo_attn_host_workspace_size(const mimo_attn_dims* d, int has_sink) {
  if (!d || d->num_seqs < 1 || d->total_tokens < 0 || d->num_q_heads < 1 || d->num_kv_heads < 1 ||
      d->head_dim_qk < 1 || d->head_dim_v < 1)
    return 0;
  const size_t T = d->total_tokens, hq = d->num_q_heads, hkv = d->num_kv_heads;
  size_t n = 0;
  n += align256(T * hq * d->head_dim_qk * 2);   // q
  n += align256(T * hkv * d->head_dim_qk * 2);  // k
  n += align256(T * hkv * d->head_dim_v * 2);   // v
  n += has_sink ? align256(hq * 4) : 0;         // sink
  n += align256((d->num_seqs + 1) * 4);         // cu_seqlens
  n += align256(T * hq * d->head_dim_v * 2);    // out
  n += align256(hq * T * 4);                    // lse
  return n;
}

int mimo_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, const float* sink_host,
                       const int32_t* cu_host, const mimo_attn_dims* d, int layer_kind, int window,
                       double rope_base, int rope_dims, float v_scale, void* out_host, float* lse_host,
                       void* workspace, size_t workspace_bytes, void* stream) {
  if (!d || !cu_host || !workspace) return MIMO_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return MIMO_ERR_INVALID_ARG;
  const size_t need = mimo_attn_host_workspace_size(d, sink_host != nullptr);
  if (need == 0 || workspace_bytes < need) return MIMO_ERR_INVALID_ARG;
  // cu_seqlens is in host memory here, so it is checked in full before any copy.
  if (cu_host[0] != 0 || cu_host[d->num_seqs] != d->total_tokens) return MIMO_ERR_INVALID_ARG;
  for (int b = 0; b < d->num_seqs; ++b) {
    const int64_t len = (int64_t)cu_host[b + 1] - cu_host[b];
    if (len < 0 || len > d->max_seqlen) return MIMO_ERR_INVALID_ARG;
  }
  const size_t T = d->total_tokens, hq = d->num_q_heads, hkv = d->num_kv_heads;
  const size_t bq = T * hq * d->head_dim_qk * 2, bk = T * hkv * d->head_dim_qk * 2, bv = T * hkv * d->head_dim_v * 2;
  const size_t bs = sink_host ? hq * 4 : 0, bc = (d->num_seqs + 1) * 4, bo = T * hq * d->head_dim_v * 2,
               bl = hq * T * 4;
  char* w = static_cast<char*>(workspace);
  char* dq = w;
  char* dk = dq + align256(bq);
  char* dv = dk + align256(bk);
  char* ds = dv + align256(bv);
  char* dc = ds + (sink_host ? align256(bs) : 0);
  char* dout = dc + align256(bc);
  char* dl = dout + align256(bo);
  int st = validate(T ? dq : nullptr, T ? dk : nullptr, T ? dv : nullptr, sink_host ? (const float*)ds : nullptr,
                    (const int32_t*)dc, d, layer_kind, window, rope_base, rope_dims, v_scale, T ? dout : nullptr,
                    T ? (const float*)dl : nullptr);
  if (st != MIMO_OK) return st;
  if (T > 0 && (!q_host || !k_host || !v_host || !out_host || !lse_host)) return MIMO_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  bool ok = true;
  if (T > 0) {
    ok = ok && cudaMemcpyAsync(dq, q_host, bq, cudaMemcpyHostToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(dk, k_host, bk, cudaMemcpyHostToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(dv, v_host, bv, cudaMemcpyHostToDevice, s) == cudaSuccess;
  }
  if (sink_host) ok = ok && cudaMemcpyAsync(ds, sink_host, bs, cudaMemcpyHostToDevice, s) == cudaSuccess;
  ok = ok && cudaMemcpyAsync(dc, cu_host, bc, cudaMemcpyHostToDevice, s) == cudaSuccess;
  if (!ok) return MIMO_ERR_CUDA;
  if (T > 0) {
    st = mimo_attn_fwd(dq, dk, dv, sink_host ? (const float*)ds : nullptr, (const int32_t*)dc, d, layer_kind,
                       window, rope_base, rope_dims, v_scale, dout, (float*)dl, stream);
    if (st != MIMO_OK) return st;
    ok = ok && cudaMemcpyAsync(out_host, dout, bo, cudaMemcpyDeviceToHost, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(lse_host, dl, bl, cudaMemcpyDeviceToHost, s) == cudaSuccess;
  }
  ok = ok && cudaStreamSynchronize(s) == cudaSuccess;
  return ok ? MIMO_OK : MIMO_ERR_CUDA;
}

int mimo_attn_check(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MIMO_ERR_CUDA;
  unsigned int e = 0;
  if (cudaMemcpyFromSymbol(&e, g_mimo_error, sizeof e) != cudaSuccess) return MIMO_ERR_CUDA;
  if (e) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_mimo_error, &zero, sizeof zero) != cudaSuccess) return MIMO_ERR_CUDA;
  }
  if (e & kErrTimeout) return MIMO_ERR_TIMEOUT;
  if (e & kErrRange) return MIMO_ERR_RANGE;
  if (e & kErrSeqlens) return MIMO_ERR_BAD_SEQLENS;
  return MIMO_OK;
}

int mimo_attn_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > 10000000000ull) return MIMO_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(limit_ns);
  if (cudaGetLastError() != cudaSuccess) return MIMO_ERR_CUDA;
  return mimo_attn_check(stream);
}

const char* mimo_attn_status_string(int status) {
  switch (status) {
    case MIMO_OK: return "ok";
    case MIMO_ERR_INVALID_ARG: return "invalid argument";
    case MIMO_ERR_UNSUPPORTED: return "unsupported configuration";
    case MIMO_ERR_CUDA: return "CUDA error";
    case MIMO_ERR_TIMEOUT: return "bounded wait timed out in a kernel";
    case MIMO_ERR_RANGE: return "rotated Q/K value outside the FP16 range";
    case MIMO_ERR_BAD_SEQLENS: return "cu_seqlens inconsistent with dims";
    case MIMO_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the no-alloc entry point holds";
    default: return "unknown status";
  }
}

int mimo_attn_profile_set_stride(int stride) {
  if (stride < 1) return MIMO_ERR_INVALID_ARG;
  ProfileState& st = profile_state();
  std::lock_guard<std::mutex> lock(st.mu);
  st.stride = stride;
  return MIMO_OK;
}

int mimo_attn_profile_start(void) {
  ProfileState& st = profile_state();
  std::lock_guard<std::mutex> lock(st.mu);
  st.enabled = true;
  st.launches = 0;
  for (auto& u : st.used) u = 0;
  return MIMO_OK;
}

int mimo_attn_profile_stop(int* launches, double* total_ms) {
  if (!launches || !total_ms) return MIMO_ERR_INVALID_ARG;
  ProfileState& st = profile_state();
  std::lock_guard<std::mutex> lock(st.mu);
  st.enabled = false;
  int n = 0;
  double ms = 0.0;
  for (int dev = 0; dev < 64; ++dev) {
    for (size_t i = 0; i < st.used[dev]; ++i) {
      auto& pr = st.pairs[dev][i];
      if (cudaEventSynchronize(pr.second) != cudaSuccess) return MIMO_ERR_CUDA;
      float e = 0.f;
      if (cudaEventElapsedTime(&e, pr.first, pr.second) != cudaSuccess) return MIMO_ERR_CUDA;
      ms += e;
      ++n;
    }
    st.used[dev] = 0;
  }
  *launches = n;
  *total_ms = ms;
  return MIMO_OK;
}

int mimo_attn_bwd(const void* q, const void* k, const void* v, const float* sink, const int32_t* cu_seqlens,
                  const mimo_attn_dims* dims, int layer_kind, int window, double rope_base, int rope_dims,
                  float v_scale, const void* out, const float* lse, const void* dout, const float* dlse, float* dq,
                  float* dk, float* dv, float* dsink, void* stream) {
  int st = validate(q, k, v, sink, cu_seqlens, dims, layer_kind, window, rope_base, rope_dims, v_scale, out, lse);
  if (st != MIMO_OK) return st;
  if ((sink != nullptr) != (dsink != nullptr)) return MIMO_ERR_INVALID_ARG;
  if (dims->total_tokens == 0) {
    if (dsink) cudaMemsetAsync(dsink, 0, sizeof(float) * dims->num_q_heads, static_cast<cudaStream_t>(stream));
    return MIMO_OK;
  }
  if (!dout || !dq || !dk || !dv || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return MIMO_ERR_INVALID_ARG;
  if (dlse && (reinterpret_cast<uintptr_t>(dlse) & 3u)) return MIMO_ERR_INVALID_ARG;
  return launch_bwd(q, k, v, sink, cu_seqlens, dims, layer_kind, window, rope_base, v_scale, out, lse, dout, dlse, dq,
                    dk, dv, dsink, static_cast<cudaStream_t>(stream));
}

int mimo_fp8_dequant_blockwise(const void* codes, const float* scale_inv, int64_t rows, int64_t cols, int block_rows,
                               int block_cols, void* out, void* stream) {
  if (rows < 0 || cols < 0 || block_rows < 1 || block_cols < 1) return MIMO_ERR_INVALID_ARG;
  if (cols % 16 != 0 || cols > 0x7FFFFFFFLL) return MIMO_ERR_UNSUPPORTED;
  if (rows == 0 || cols == 0) return MIMO_OK;
  if (!codes || !scale_inv || !out || !aligned16(codes) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(scale_inv) & 3u))
    return MIMO_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MIMO_ERR_CUDA;
  DeviceInfo* info = device_info(dev);
  if (!info) return MIMO_ERR_CUDA;
  const long long work = rows * (cols / 16);
  const unsigned grid = (unsigned)std::min<long long>((work + nb::kThreads - 1) / nb::kThreads, 8LL * info->sms);
  nb::fp8_dequant_kernel<<<grid, nb::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(codes), scale_inv, static_cast<uint16_t*>(out), rows, cols, block_rows, block_cols);
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}

int mimo_qkv_split(const void* fused, int64_t tokens, int num_q_heads, int num_kv_heads, void* q, void* k, void* v,
                   void* stream) {
  if (tokens < 0 || num_q_heads < 1 || num_kv_heads < 1 || num_q_heads % num_kv_heads != 0)
    return MIMO_ERR_INVALID_ARG;
  if (tokens == 0) return MIMO_OK;
  if (!fused || !q || !k || !v || !aligned16(fused) || !aligned16(q) || !aligned16(k) || !aligned16(v))
    return MIMO_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MIMO_ERR_CUDA;
  DeviceInfo* info = device_info(dev);
  if (!info) return MIMO_ERR_CUDA;
  const long long chunks = tokens * (long long)num_kv_heads * ((num_q_heads / num_kv_heads) * 24 + 40);
  const unsigned grid = (unsigned)std::min<long long>((chunks + nb::kThreads - 1) / nb::kThreads, 8LL * info->sms);
  nb::qkv_split_kernel<<<grid, nb::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(fused), static_cast<uint16_t*>(q), static_cast<uint16_t*>(k),
      static_cast<uint16_t*>(v), tokens, num_q_heads, num_kv_heads);
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}

int mimo_linear_proj(const void* x, const void* w, int64_t tokens, int64_t in_features, int64_t out_features,
                     void* y, void* stream) {
  if (tokens < 0 || in_features < 1 || out_features < 1) return MIMO_ERR_INVALID_ARG;
  if (in_features % 8 != 0 || out_features % 8 != 0) return MIMO_ERR_UNSUPPORTED;  // 16-byte rows
  if (tokens > INT32_MAX || in_features > INT32_MAX || out_features > INT32_MAX) return MIMO_ERR_UNSUPPORTED;
  if (tokens == 0) return MIMO_OK;
  if (!x || !w || !y || !aligned16(x) || !aligned16(w) || !aligned16(y)) return MIMO_ERR_INVALID_ARG;
  return gemm_bf16_nt(x, w, (int)tokens, (int)in_features, (int)out_features, y, static_cast<cudaStream_t>(stream));
}

int mimo_moe_route(const float* logits, const float* bias, int64_t tokens, int num_experts, int top_k, int normalize,
                   int32_t* ids, float* weights, void* stream) {
  if (tokens < 0 || num_experts < 32 || num_experts % 32 != 0 || top_k < 1 || top_k > 32 || top_k > num_experts)
    return MIMO_ERR_INVALID_ARG;
  if (num_experts > 256) return MIMO_ERR_UNSUPPORTED;
  if (tokens == 0) return MIMO_OK;
  if (!logits || !bias || !ids || !weights) return MIMO_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MIMO_ERR_CUDA;
  DeviceInfo* info = device_info(dev);
  if (!info) return MIMO_ERR_CUDA;
  const long long warps_per_cta = nb::kThreads / 32;
  if (top_k <= 16) {  // two tokens per warp
    const long long pairs = (tokens + 1) / 2;
    const unsigned grid = (unsigned)std::min<long long>((pairs + warps_per_cta - 1) / warps_per_cta, 16LL * info->sms);
    if (num_experts == 256)
      nb::route_pair_kernel<16, true><<<grid, nb::kThreads, nb::kRoutePairSmemBytes, static_cast<cudaStream_t>(stream)>>>(
          logits, bias, ids, weights, tokens, num_experts, top_k, normalize ? 1 : 0);
    else
      nb::route_pair_kernel<16, false><<<grid, nb::kThreads, nb::kRoutePairSmemBytes, static_cast<cudaStream_t>(stream)>>>(
          logits, bias, ids, weights, tokens, num_experts, top_k, normalize ? 1 : 0);
  } else {
    const unsigned grid =
        (unsigned)std::min<long long>((tokens + warps_per_cta - 1) / warps_per_cta, 16LL * info->sms);
    nb::route_kernel<8><<<grid, nb::kThreads, nb::kRouteSmemBytes, static_cast<cudaStream_t>(stream)>>>(
        logits, bias, ids, weights, tokens, num_experts, top_k, normalize ? 1 : 0);
  }
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}

int mimo_attn_version(void) { return (1 << 16) | 5; }

int mimo_attn_fwd_noalloc(const void* q, const void* k, const void* v, const float* sink,
                          const int32_t* cu_seqlens, const mimo_attn_dims* dims, int layer_kind, int window,
                          double rope_base, int rope_dims, float v_scale, void* out, float* lse, void* stream) {
  int st = validate(q, k, v, sink, cu_seqlens, dims, layer_kind, window, rope_base, rope_dims, v_scale, out, lse);
  if (st != MIMO_OK) return st;
  if (dims->total_tokens == 0) return MIMO_OK;
  FwdParams P;
  fill_params(P, sink, cu_seqlens, dims, layer_kind, window, rope_base, v_scale, out, lse);
  return launch_noalloc(q, k, v, P, static_cast<cudaStream_t>(stream));
}

size_t mimo_attn_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

int mimo_attn_set_bwd_kernel(int choice) {
  if (choice < 0 || choice > 2) return MIMO_ERR_INVALID_ARG;
  g_bwd_choice.store(choice);
  return MIMO_OK;
}

int mimo_attn_set_decode_kernel(int choice) {
  if (choice != MIMO_DECODE_AUTO && choice != MIMO_DECODE_CUDA_CORES && choice != MIMO_DECODE_TENSOR)
    return MIMO_ERR_INVALID_ARG;
  g_decode_choice.store(choice);
  return MIMO_OK;
}

int mimo_attn_set_kernel(int choice) {
  if (choice != MIMO_KERNEL_AUTO && choice != MIMO_KERNEL_SIMPLE && choice != MIMO_KERNEL_PIPELINED &&
      choice != MIMO_KERNEL_WINDOW && choice != MIMO_KERNEL_WINDOW_PACKED)
    return MIMO_ERR_INVALID_ARG;
  g_kernel_choice.store(choice);
  return MIMO_OK;
}

}  // extern "C"
