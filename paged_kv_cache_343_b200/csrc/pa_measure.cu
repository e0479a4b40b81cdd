// pa_measure.cu -- a read-only HBM stream, the ceiling the decode kernels are
// held against.  Decode reads each K/V byte once and writes almost nothing,
// and reading the growing cache is what limits it ("KV cache and
// PagedAttention: how vLLM uses GPU memory more efficiently", opening
// section), so its roofline is the rate at which this GPU can read, which a
// copy benchmark (half reads, half writes) does not show directly.
//
// Each thread streams 16-byte words with a grid-stride loop, so the loads in
// flight at any moment cover one contiguous window of the buffer (spreading
// each thread's loads over several windows measured slower), and folds them
// into an XOR; each CTA writes the XOR of everything it read, so nothing can
// be optimised away and the caller can check that every word was read
// exactly once (the XOR of the sink equals the XOR of the buffer).
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

constexpr int kStreamThreads = 512;

__device__ __forceinline__ uint32_t fold(const uint4 v) { return v.x ^ v.y ^ v.z ^ v.w; }

__global__ void __launch_bounds__(kStreamThreads)
    pa_stream_read_kernel(const uint4* __restrict__ buf, int64_t n16, uint32_t* __restrict__ sink) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  uint32_t acc = 0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += stride)
    acc ^= fold(__ldcs(buf + i));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ uint32_t s_warp[kStreamThreads / 32];
  if ((threadIdx.x & 31) == 0) s_warp[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
    for (int w = 0; w < kStreamThreads / 32; ++w) r ^= s_warp[w];
    sink[blockIdx.x] = r;
  }
}

}  // namespace pa

extern "C" pa_status pa_stream_read(const void* buf, int64_t bytes, uint32_t* sink,
                                    int32_t num_ctas, pa_stream_t stream) {
  if (bytes < 0 || bytes % 16 != 0 || num_ctas < 1 || num_ctas > 65535 || sink == nullptr ||
      !pa::aligned(sink, 4))
    return PA_ERR_INVALID_ARG;
  if (bytes > 0 && (buf == nullptr || !pa::aligned(buf, 16))) return PA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  pa::pa_stream_read_kernel<<<num_ctas, pa::kStreamThreads, 0, s>>>(
      static_cast<const uint4*>(buf), bytes / 16, sink);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
