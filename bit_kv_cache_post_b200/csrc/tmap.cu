// Host-side tensor-map encoding shared by the kernels that load tiles with
// the TMA engine.  The driver's encoder is reached through the runtime's
// entry-point query, so the library links against the runtime only.
#include <cuda.h>

#include <cstring>

#include "wushkv_internal.cuh"

namespace wushkv {

EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

namespace {

// fp16 rows [rows][128] at `base`; box = 8 rows x 64 dims, 128-byte swizzle:
// 16-byte chunk j of box row i lands at chunk j ^ (i % 8) of that row.
bool make_rows_map(CUtensorMap* m, const void* base, uint64_t rows) {
  const EncodeTiledFn encode = tensor_map_encoder();
  if (!encode || rows == 0) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)WIN_BOX_ROWS};
  const cuuint32_t estr[2] = {1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

void make_window_maps(const DevCache& c, WindowMaps* m) {
  std::memset(m, 0, sizeof(*m));
  const uint64_t U = (uint64_t)c.units;
  const uint64_t lim = (uint64_t)1 << 31;   // box coordinates are 32-bit signed
  const uint64_t sink_rows = U * (uint64_t)c.sink, ring_rows = U * (uint64_t)c.ring_slots;
  m->has_sink = sink_rows > 0 && sink_rows < lim && make_rows_map(&m->sink_k, c.sink_k, sink_rows) &&
                make_rows_map(&m->sink_v, c.sink_v, sink_rows);
  m->has_ring = ring_rows > 0 && ring_rows < lim && make_rows_map(&m->ring_k, c.ring_k, ring_rows) &&
                make_rows_map(&m->ring_v, c.ring_v, ring_rows);
}

}  // namespace wushkv
