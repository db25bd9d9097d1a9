// Host side of TMA: 2-D tensor maps encoded through the driver entry point (fetched once through the
// runtime, so the library needs no link-time dependency on libcuda), cached per operand.
#include <cuda.h>

#include <map>
#include <mutex>
#include <tuple>

#include "tern_internal.cuh"

namespace tern {
namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(f);
  });
  return fn;
}

bool make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  // elements outside [0, inner) x [0, outer) read as zero
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

using Key = std::tuple<const void*, int, uint64_t, uint64_t, uint64_t, uint32_t, uint32_t, int>;

}  // namespace

bool tmap_2d(CUtensorMap* out, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
             uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  static std::mutex mu;
  static std::map<Key, CUtensorMap> maps;
  const Key key{base, (int)dt, inner, outer, row_stride_bytes, box_inner, box_outer, (int)sw};
  std::lock_guard<std::mutex> lock(mu);
  auto itr = maps.find(key);
  if (itr != maps.end()) {
    *out = itr->second;
    return true;
  }
  if (!make_map(out, dt, base, inner, outer, row_stride_bytes, box_inner, box_outer, sw)) return false;
  if (maps.size() > 4096) maps.clear();
  maps.emplace(key, *out);
  return true;
}

}  // namespace tern
