// tensormap_host.h -- host tensor-map encoder for the host build: records what the device model's
// tma_load_2d / tma_store_2d need (base, extents, row stride, box, element size).
#pragma once
namespace hemu {
CUresult host_encode_tiled(CUtensorMap* m, CUtensorMapDataType dt, cuuint32_t rank, void* base, const cuuint64_t* dims,
                           const cuuint64_t* strides, const cuuint32_t* box, const cuuint32_t*, CUtensorMapInterleave,
                           CUtensorMapSwizzle sw, CUtensorMapL2promotion, CUtensorMapFloatOOBfill) {
  if ((rank != 2 && rank != 3) || sw != CU_TENSOR_MAP_SWIZZLE_128B) return CUDA_ERROR_INVALID_VALUE;
  mimo::HostTmap t;
  t.base = static_cast<const uint8_t*>(base);
  t.inner = dims[0];
  t.rows = dims[1];
  t.stride = strides[0];
  t.box_inner = box[0];
  t.box_rows = box[1];
  t.elem = dt == CU_TENSOR_MAP_DATA_TYPE_UINT8 ? 1 : 2;
  if (rank == 3) {
    t.depth = dims[2];
    t.stride2 = strides[1];
    t.box_depth = box[2];
  }
  std::memset(m, 0, sizeof(*m));
  std::memcpy(m, &t, sizeof t);
  return CUDA_SUCCESS;
}
}  // namespace hemu
