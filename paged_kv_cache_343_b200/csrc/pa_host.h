// pa_host.h -- host-side helpers shared by the library's entry points:
// per-device attributes, dynamic shared-memory opt-in, alignment checks and a
// small cache of TMA tensor descriptors keyed by pool address and shape.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <utility>

#include "../../include/pagedattn.h"

namespace pa {

struct DeviceInfo {
  int device = -1;
  int num_sms = 0;
  int max_smem_optin = 0;
  int l2_bytes = 0;
};

// Attributes of the current device (cached per device); nullptr on failure.
const DeviceInfo* current_device_info();

// Opts `func` into `bytes` of dynamic shared memory on the current device.
bool ensure_smem_attr(const void* func, size_t bytes);

// Resident CTAs per SM of `func` at this launch shape on the current device
// (cached); 0 on failure.
int ctas_per_sm(const void* func, int threads, size_t smem);

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// Tiled tensor map of `rank` (4 or 5) dimensions with 128-byte swizzle over
// `base`, elements of `elem_bytes` (1 or 2) bytes.  dims: innermost first;
// strides: bytes of dims 1..rank-1; box: elements per dim.  Returns false if
// the driver rejects it.
bool get_tensor_map(CUtensorMap* out, const void* base, const uint64_t dims[5],
                    const uint64_t strides[4], const uint32_t box[5], int elem_bytes = 2,
                    int rank = 5);

// Launches kernels with programmatic dependent launch on `stream`: the kernel
// may start while the previous kernel on the stream finishes and must call
// griddepcontrol.wait before it touches memory that kernel may write.
struct PdlLaunch {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr;
  PdlLaunch(cudaStream_t stream, dim3 grid, dim3 block, size_t smem = 0) {
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
  }
  template <typename... KArgs, typename... Args>
  cudaError_t operator()(void (*kernel)(KArgs...), Args&&... args) {
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  }
};

}  // namespace pa
