// tma_host.cu -- cuTensorMapEncodeTiled through the runtime's driver entry
// point (no link-time dependency on libcuda).
#include "tma_host.h"

#include <mutex>

namespace fa {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                   void*, const cuuint64_t*, const cuuint64_t*,
                                   const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr,
                                cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Encoded maps of recent calls.  A map is a pure function of the encode
// arguments (address, extents, strides, box, type, swizzle), so an entry
// stays valid whatever happens to the memory it names; a repeated call with
// the same tensors skips the encode.
struct MapArgs {
  const void* base;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3];
  int dtype, swizzle;
  bool operator==(const MapArgs& o) const {
    return base == o.base && dims[0] == o.dims[0] && dims[1] == o.dims[1] &&
           dims[2] == o.dims[2] && strides[0] == o.strides[0] &&
           strides[1] == o.strides[1] && box[0] == o.box[0] && box[1] == o.box[1] &&
           box[2] == o.box[2] && dtype == o.dtype && swizzle == o.swizzle;
  }
};

constexpr int kMapCacheSlots = 64;
std::mutex g_map_mu;
MapArgs g_map_args[kMapCacheSlots];
CUtensorMap g_maps[kMapCacheSlots];
int g_map_used = 0, g_map_next = 0;

// Rank-3 tiled map with unit element strides, no interleave, 256-byte L2
// promotion and zero fill, from the cache or freshly encoded.
cudaError_t encode_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                      const cuuint64_t dims[3], const cuuint64_t strides[2],
                      const cuuint32_t box[3], CUtensorMapSwizzle swizzle) {
  MapArgs a;
  a.base = base;
  for (int i = 0; i < 3; ++i) a.dims[i] = dims[i], a.box[i] = box[i];
  a.strides[0] = strides[0];
  a.strides[1] = strides[1];
  a.dtype = int(dtype);
  a.swizzle = int(swizzle);
  {
    std::lock_guard<std::mutex> lock(g_map_mu);
    for (int i = 0; i < g_map_used; ++i)
      if (g_map_args[i] == a) {
        *map = g_maps[i];
        return cudaSuccess;
      }
  }
  EncodeTiledFn enc = get_encode();
  if (!enc) return cudaErrorNotSupported;
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> lock(g_map_mu);
  const int slot = g_map_next;  // round robin over the slots
  g_map_next = (g_map_next + 1) % kMapCacheSlots;
  if (g_map_used < kMapCacheSlots) ++g_map_used;
  g_map_args[slot] = a;
  g_maps[slot] = *map;
  return cudaSuccess;
}

}  // namespace

cudaError_t make_operand_map(CUtensorMap* map, const void* base,
                             const Problem& p, int S, int box_rows) {
  cuuint64_t dims[3], strides[2];
  const cuuint64_t esz = p.f8 ? 1 : 2;  // e4m3, or bf16 / fp16
  if (p.layout == FA_LAYOUT_BSH) {
    dims[0] = cuuint64_t(p.N) * p.D;
    dims[1] = cuuint64_t(S);
    dims[2] = cuuint64_t(p.B);
    strides[0] = dims[0] * esz;
    strides[1] = dims[0] * dims[1] * esz;
  } else {
    dims[0] = cuuint64_t(p.D);
    dims[1] = cuuint64_t(S);
    dims[2] = cuuint64_t(p.B) * p.N;
    strides[0] = dims[0] * esz;
    strides[1] = dims[0] * dims[1] * esz;
  }
  // 128-byte box rows: 64 16-bit or 128 8-bit columns
  const cuuint32_t box[3] = {cuuint32_t(128 / esz), cuuint32_t(box_rows), 1u};
  const CUtensorMapDataType dt = p.f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                      : (p.f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                               : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  return encode_3d(map, dt, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaError_t make_f32_rows_map(CUtensorMap* map, const void* base, int cols,
                              int rows, int64_t planes, int box_cols,
                              int box_rows) {
  const cuuint64_t dims[3] = {cuuint64_t(cols), cuuint64_t(rows), cuuint64_t(planes)};
  const cuuint64_t strides[2] = {cuuint64_t(cols) * 4, cuuint64_t(cols) * rows * 4};
  const cuuint32_t box[3] = {cuuint32_t(box_cols), cuuint32_t(box_rows), 1u};
  return encode_3d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace fa
