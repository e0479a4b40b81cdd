// pa_host.cu -- host helpers and the library's status / version entry points.
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <vector>

#include "pa_host.h"

namespace pa {

namespace {

std::mutex g_mu;
DeviceInfo g_devices[64];

struct SmemAttr {
  const void* func;
  int device;
  size_t bytes;
};
std::vector<SmemAttr> g_smem_attrs;

struct Occupancy {
  const void* func;
  int device;
  int threads;
  size_t smem;
  int per_sm;
};
std::vector<Occupancy> g_occupancy;

struct TmapEntry {
  const void* base;
  int elem_bytes;
  int rank;
  uint64_t dims[5];
  uint64_t strides[4];
  uint32_t box[5];
  bool ok;
  CUtensorMap map;
};
constexpr size_t kTmapCacheSize = 32;
std::vector<TmapEntry> g_tmaps;  // most recent last
size_t g_tmap_next = 0;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
bool g_encode_looked_up = false;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  if (!g_encode_looked_up) {
    g_encode_looked_up = true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  return g_encode;
}

}  // namespace

const DeviceInfo* current_device_info() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_devices[dev];
  if (d.device != dev) {
    int sms = 0, smem = 0, l2 = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess)
      return nullptr;
    d.num_sms = sms;
    d.max_smem_optin = smem;
    d.l2_bytes = l2;
    d.device = dev;
  }
  return &d;
}

bool ensure_smem_attr(const void* func, size_t bytes) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(g_mu);
  for (const SmemAttr& a : g_smem_attrs)
    if (a.func == func && a.device == dev && a.bytes >= bytes) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess)
    return false;
  for (SmemAttr& a : g_smem_attrs) {
    if (a.func == func && a.device == dev) {
      a.bytes = bytes;
      return true;
    }
  }
  g_smem_attrs.push_back({func, dev, bytes});
  return true;
}

int ctas_per_sm(const void* func, int threads, size_t smem) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(g_mu);
  for (const Occupancy& o : g_occupancy)
    if (o.func == func && o.device == dev && o.threads == threads && o.smem == smem)
      return o.per_sm;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem) != cudaSuccess)
    return 0;
  g_occupancy.push_back({func, dev, threads, smem, n});
  return n;
}

bool get_tensor_map(CUtensorMap* out, const void* base, const uint64_t dims[5],
                    const uint64_t strides[4], const uint32_t box[5], int elem_bytes,
                    int rank) {
  std::lock_guard<std::mutex> lock(g_mu);
  for (const TmapEntry& e : g_tmaps) {
    if (e.base == base && e.elem_bytes == elem_bytes && e.rank == rank &&
        std::memcmp(e.dims, dims, sizeof(e.dims)) == 0 &&
        std::memcmp(e.strides, strides, sizeof(e.strides)) == 0 &&
        std::memcmp(e.box, box, sizeof(e.box)) == 0) {
      if (e.ok) *out = e.map;
      return e.ok;
    }
  }
  TmapEntry e;
  e.base = base;
  e.elem_bytes = elem_bytes;
  e.rank = rank;
  std::memcpy(e.dims, dims, sizeof(e.dims));
  std::memcpy(e.strides, strides, sizeof(e.strides));
  std::memcpy(e.box, box, sizeof(e.box));
  e.ok = false;
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc != nullptr) {
    const cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
    cuuint64_t gdims[5];
    cuuint64_t gstr[4];
    cuuint32_t gbox[5];
    for (int i = 0; i < 5; ++i) {
      gdims[i] = dims[i];
      gbox[i] = box[i];
    }
    for (int i = 0; i < 4; ++i) gstr[i] = strides[i];
    const CUresult r = enc(&e.map,
                           elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                           : CU_TENSOR_MAP_DATA_TYPE_UINT16,
                           static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                           gdims, gstr, gbox, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    e.ok = (r == CUDA_SUCCESS);
  }
  if (g_tmaps.size() < kTmapCacheSize) {
    g_tmaps.push_back(e);
  } else {
    g_tmaps[g_tmap_next] = e;
    g_tmap_next = (g_tmap_next + 1) % kTmapCacheSize;
  }
  if (e.ok) *out = e.map;
  return e.ok;
}

}  // namespace pa

extern "C" const char* pa_status_string(pa_status status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_OUT_OF_BLOCKS: return "PA_ERR_OUT_OF_BLOCKS";
    case PA_ERR_NOT_FOUND: return "PA_ERR_NOT_FOUND";
    case PA_ERR_TOO_LARGE: return "PA_ERR_TOO_LARGE";
  }
  return "PA_ERR_UNKNOWN";
}

extern "C" int32_t pa_version(void) { return 200; }
