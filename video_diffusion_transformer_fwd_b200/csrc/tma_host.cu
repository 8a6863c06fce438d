// Host helpers for TMA tensor maps: cuTensorMapEncodeTiled is fetched from
// the driver through the runtime, so the library has no link-time libcuda
// dependency and loads on machines without a GPU.
#include "common.cuh"
#include "sm100.cuh"

#include <cudaTypedefs.h>

#include <mutex>

namespace wan {

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

static int encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
                     uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return set_error(WAN_ECUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t gdim[2] = {inner, rows};
  cuuint64_t gstride[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dt, 2, const_cast<void *>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(WAN_ECUDA, "cuTensorMapEncodeTiled (2d) failed: %d", (int)r);
  return WAN_OK;
}

int encode_tmap_2d_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                        uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, inner, rows, row_stride_bytes, box_inner, box_rows);
}

int encode_tmap_2d_u8(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, rows, row_stride_bytes, box_inner, box_rows);
}

int encode_tmap_2d_f32(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                       uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, inner, rows, row_stride_bytes, box_inner, box_rows);
}

static int encode_3d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t rows,
                     uint64_t batches, uint64_t row_stride_bytes, uint64_t batch_stride_bytes,
                     uint32_t box_inner, uint32_t box_rows);

int encode_tmap_3d_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                        uint64_t batches, uint64_t row_stride_bytes, uint64_t batch_stride_bytes,
                        uint32_t box_inner, uint32_t box_rows) {
  return encode_3d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, inner, rows, batches, row_stride_bytes,
                   batch_stride_bytes, box_inner, box_rows);
}

int encode_tmap_3d_u8(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                      uint64_t batches, uint64_t row_stride_bytes, uint64_t batch_stride_bytes,
                      uint32_t box_inner, uint32_t box_rows) {
  return encode_3d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, rows, batches, row_stride_bytes,
                   batch_stride_bytes, box_inner, box_rows);
}

static int encode_3d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t rows,
                     uint64_t batches, uint64_t row_stride_bytes, uint64_t batch_stride_bytes,
                     uint32_t box_inner, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return set_error(WAN_ECUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t gdim[3] = {inner, rows, batches};
  cuuint64_t gstride[2] = {row_stride_bytes, batch_stride_bytes};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dt, 3, const_cast<void *>(base), gdim, gstride, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(WAN_ECUDA, "cuTensorMapEncodeTiled (3d) failed: %d", (int)r);
  return WAN_OK;
}

int sm_count() {
  static int counts[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!counts[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    counts[dev] = n;
  }
  return counts[dev];
}

}  // namespace wan
