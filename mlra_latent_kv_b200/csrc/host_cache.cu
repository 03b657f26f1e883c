// Host-side caches of TMA descriptors and kernel attributes.
#include <cudaTypedefs.h>

#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "host_cache.h"

namespace mlra {
namespace {

std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
bool g_encode_tried = false;

using MapKey = std::tuple<int, uintptr_t, uint64_t, uint64_t, uint64_t, uint32_t, uint32_t>;
std::map<MapKey, CUtensorMap> g_maps;
std::map<std::pair<int, const void*>, int> g_smem;  // (device, function) -> limit set

bool encoder_locked() {
  if (!g_encode_tried) {
    g_encode_tried = true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return g_encode != nullptr;
}

bool encode(CUtensorMap* m, int rank, const void* base, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box, CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint32_t es[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename F>
bool cached(const MapKey& k, CUtensorMap* out, F make) {
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_maps.find(k);
  if (it != g_maps.end()) {
    *out = it->second;
    return true;
  }
  if (!encoder_locked()) return false;
  CUtensorMap m;
  if (!make(&m)) return false;
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps.emplace(k, m);
  *out = m;
  return true;
}

}  // namespace

bool tmap_2d(CUtensorMap* out, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows) {
  const MapKey k{2, reinterpret_cast<uintptr_t>(base), cols, rows, 0, box_cols, box_rows};
  return cached(k, out, [&](CUtensorMap* m) {
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    return encode(m, 2, base, dims, strides, box);
  });
}

bool tmap_2d_sw64(CUtensorMap* out, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                  uint32_t box_rows) {
  const MapKey k{4, reinterpret_cast<uintptr_t>(base), cols, rows, 0, box_cols, box_rows};
  return cached(k, out, [&](CUtensorMap* m) {
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    return encode(m, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B);
  });
}

bool tmap_3d_batch(CUtensorMap* out, const void* base, uint64_t K, uint64_t H, uint64_t B, uint32_t Bp) {
  const MapKey k{3, reinterpret_cast<uintptr_t>(base), K, H, B, 64, Bp};
  return cached(k, out, [&](CUtensorMap* m) {
    cuuint64_t dims[3] = {K, H, B};
    cuuint64_t strides[2] = {K * 2, H * K * 2};
    cuuint32_t box[3] = {64, 1, Bp};
    return encode(m, 3, base, dims, strides, box);
  });
}

cudaError_t ensure_smem(const void* func, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  int& cur = g_smem[{dev, func}];
  if (bytes <= cur) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) cur = bytes;
  return e;
}

void record_event(cudaEvent_t ev, cudaStream_t stream) {
  if (!ev) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, stream);
}

void host_cache_clear() {
  std::lock_guard<std::mutex> lock(g_mu);
  g_maps.clear();
  g_smem.clear();
}

}  // namespace mlra
