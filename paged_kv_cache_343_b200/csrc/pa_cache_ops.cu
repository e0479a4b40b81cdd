// pa_cache_ops.cu -- the two cache-maintenance kernels of the hot path.
//
// reshape_and_cache ("How PagedAttention Works in vLLM to Maximize Memory
// Efficiency", "write_to_paged_cache: Direct In-Place Updates"): new K/V rows
// go straight into their pool slots, no staging buffer.  Slot s = block *
// block_size + offset; head h of the token lands at block * block_stride +
// offset * token_stride + h * head_stride (elements; head_dim contiguous).
// With the pool laid out [num_blocks, block_size, Hkv, D] that is
// s * Hkv * D + h * D: one contiguous row of Hkv * D words per token.
//
// copy_blocks ("PagedAttention", "How does copy-on-write work for parallel
// sampling?"): the copy step of copy-on-write, a whole physical block per
// (src, dst) pair and pool.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

constexpr int kRowThreads = 128;
constexpr int kCopyThreads = 256;
constexpr int kMaxCopyCaches = 128;  // pointers per copy_blocks launch (64 layers of K and V)

template <int VEC>
struct Vec;
template <>
struct Vec<8> {
  using T = uint4;
};
template <>
struct Vec<1> {
  using T = uint16_t;
};

// Where a pool's elements live (in elements): see pa_cache_strides.
struct PoolLayout {
  int64_t block_stride, token_stride, head_stride;
  int32_t block_size, head_dim;
  __device__ __forceinline__ int64_t slot_base(int64_t slot) const {
    return (slot / block_size) * block_stride + (slot % block_size) * token_stride;
  }
};

// One CTA per token (grid-stride); the block's threads split the K and V rows
// in VEC-element pieces, piece i of a row being head i / (D / VEC).
template <int VEC>
__global__ void __launch_bounds__(kRowThreads)
    pa_reshape_and_cache_kernel(const uint16_t* __restrict__ key,
                                const uint16_t* __restrict__ value, int64_t key_stride,
                                int64_t value_stride, uint16_t* __restrict__ key_cache,
                                uint16_t* __restrict__ value_cache, const PoolLayout lay,
                                const int32_t* __restrict__ slot_mapping, int32_t num_tokens,
                                int64_t num_slots, int32_t row_elems, int32_t* err) {
  using T = typename Vec<VEC>::T;
  const int32_t nvec = row_elems / VEC;
  const int32_t per_head = lay.head_dim / VEC;
  griddep_launch_dependents();
  griddep_wait();
  for (int64_t t = blockIdx.x; t < num_tokens; t += gridDim.x) {
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;  // padding token
    if (slot >= num_slots) {
      if (threadIdx.x == 0) flag_error(err, PA_DEVERR_BAD_SLOT);
      continue;
    }
    const int64_t base = lay.slot_base(slot);
    const T* ks = reinterpret_cast<const T*>(key + t * key_stride);
    const T* vs = reinterpret_cast<const T*>(value + t * value_stride);
    for (int32_t i = threadIdx.x; i < 2 * nvec; i += kRowThreads) {
      const bool is_v = i >= nvec;
      const int32_t j = is_v ? i - nvec : i;
      const int32_t h = j / per_head;
      const int64_t dst = base + h * lay.head_stride + (j - h * per_head) * VEC;
      *reinterpret_cast<T*>((is_v ? value_cache : key_cache) + dst) = (is_v ? vs : ks)[j];
    }
  }
}

// fp8 variant: each thread takes 8 elements (16 bytes in, 8 bytes out);
// code = e4m3(x / scale) with the quotient in fp32.
template <bool kBF16>
__global__ void __launch_bounds__(kRowThreads)
    pa_reshape_and_cache_fp8_kernel(const uint16_t* __restrict__ key,
                                    const uint16_t* __restrict__ value, int64_t key_stride,
                                    int64_t value_stride, uint8_t* __restrict__ key_cache,
                                    uint8_t* __restrict__ value_cache, const PoolLayout lay,
                                    const int32_t* __restrict__ slot_mapping, int32_t num_tokens,
                                    int64_t num_slots, int32_t row_elems,
                                    const float* __restrict__ k_scale,
                                    const float* __restrict__ v_scale, int32_t* err) {
  const int32_t nvec = row_elems / 8;
  const int32_t per_head = lay.head_dim / 8;
  griddep_launch_dependents();
  griddep_wait();
  const float ks = *k_scale, vs = *v_scale;
  for (int64_t t = blockIdx.x; t < num_tokens; t += gridDim.x) {
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (threadIdx.x == 0) flag_error(err, PA_DEVERR_BAD_SLOT);
      continue;
    }
    const int64_t base = lay.slot_base(slot);
    for (int32_t i = threadIdx.x; i < 2 * nvec; i += kRowThreads) {
      const bool is_v = i >= nvec;
      const int32_t j = is_v ? i - nvec : i;
      const int32_t h = j / per_head;
      const int64_t dst = base + h * lay.head_stride + (j - h * per_head) * 8;
      const uint4 x = reinterpret_cast<const uint4*>((is_v ? value + t * value_stride
                                                             : key + t * key_stride))[j];
      const float s = is_v ? vs : ks;
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
      uint16_t c[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float lo = __fdiv_rn(lo_to_float<kBF16>(w[q]), s);
        const float hi = __fdiv_rn(hi_to_float<kBF16>(w[q]), s);
        c[q] = pack_e4m3x2(lo, hi);
      }
      uint2 out;
      out.x = static_cast<uint32_t>(c[0]) | (static_cast<uint32_t>(c[1]) << 16);
      out.y = static_cast<uint32_t>(c[2]) | (static_cast<uint32_t>(c[3]) << 16);
      *reinterpret_cast<uint2*>((is_v ? value_cache : key_cache) + dst) = out;
    }
  }
}

struct CopyPtrs {
  uint8_t* p[kMaxCopyCaches];
};

// grid (num_pairs, num_caches): one CTA copies one block of one pool.
template <bool kVec16>
__global__ void __launch_bounds__(kCopyThreads)
    pa_copy_blocks_kernel(const CopyPtrs ptrs, const int32_t* __restrict__ mapping,
                          int32_t num_blocks, int64_t block_bytes, int32_t* err) {
  const int64_t pair = blockIdx.x;
  griddep_launch_dependents();
  griddep_wait();
  const int32_t src = mapping[2 * pair], dst = mapping[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) flag_error(err, PA_DEVERR_BAD_SLOT);
    return;
  }
  uint8_t* base = ptrs.p[blockIdx.y];
  if constexpr (kVec16) {
    const uint4* s = reinterpret_cast<const uint4*>(base + src * block_bytes);
    uint4* d = reinterpret_cast<uint4*>(base + dst * block_bytes);
    const int64_t n = block_bytes / 16;
    for (int64_t i = threadIdx.x; i < n; i += kCopyThreads) d[i] = s[i];
  } else {
    const uint8_t* s = base + src * block_bytes;
    uint8_t* d = base + dst * block_bytes;
    for (int64_t i = threadIdx.x; i < block_bytes; i += kCopyThreads) d[i] = s[i];
  }
}

// Strided pools: grid (num_pairs, num_caches), one CTA copies the
// block_size x Hkv rows of head_dim elements of one block of one pool in
// 16-byte pieces (row_bytes and all strides multiples of 16 bytes).
__global__ void __launch_bounds__(kCopyThreads)
    pa_copy_blocks_strided_kernel(const CopyPtrs ptrs, const int32_t* __restrict__ mapping,
                                  int32_t num_blocks, int64_t block_stride_b,
                                  int64_t token_stride_b, int64_t head_stride_b,
                                  int32_t block_size, int32_t num_kv_heads, int32_t row_bytes,
                                  int32_t* err) {
  const int64_t pair = blockIdx.x;
  griddep_launch_dependents();
  griddep_wait();
  const int32_t src = mapping[2 * pair], dst = mapping[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) flag_error(err, PA_DEVERR_BAD_SLOT);
    return;
  }
  uint8_t* base = ptrs.p[blockIdx.y];
  const uint8_t* s = base + src * block_stride_b;
  uint8_t* d = base + dst * block_stride_b;
  const int32_t per_row = row_bytes / 16;
  const int64_t n = static_cast<int64_t>(block_size) * num_kv_heads * per_row;
  for (int64_t i = threadIdx.x; i < n; i += kCopyThreads) {
    const int64_t r = i / per_row;  // row = token * Hkv + head
    const int64_t tok = r / num_kv_heads, h = r - tok * num_kv_heads;
    const int64_t off = tok * token_stride_b + h * head_stride_b + (i - r * per_row) * 16;
    *reinterpret_cast<uint4*>(d + off) = *reinterpret_cast<const uint4*>(s + off);
  }
}

}  // namespace pa

using namespace pa;

namespace {

pa_status reshape_impl(const void* key, const void* value, int64_t key_stride_t,
                       int64_t value_stride_t, void* key_cache, void* value_cache,
                       const pa_cache_strides* cs, const int32_t* slot_mapping,
                       int32_t num_tokens, int32_t num_blocks, int32_t block_size,
                       int32_t num_kv_heads, int32_t head_dim, pa_dtype dtype,
                       pa_kv_cache_dtype kv_cache_dtype, const float* k_scale,
                       const float* v_scale, int32_t* device_error_flag, pa_stream_t stream) {
  if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 ||
      head_dim <= 0)
    return PA_ERR_INVALID_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (kv_cache_dtype != PA_KV_AUTO && kv_cache_dtype != PA_KV_FP8_E4M3) return PA_ERR_UNSUPPORTED;
  if (cs->block_stride <= 0 || cs->token_stride <= 0 || cs->head_stride <= 0)
    return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  const int64_t row = static_cast<int64_t>(num_kv_heads) * head_dim;
  if (row > INT32_MAX || key_stride_t < row || value_stride_t < row) return PA_ERR_INVALID_ARG;
  PoolLayout lay;
  lay.block_stride = cs->block_stride;
  lay.token_stride = cs->token_stride;
  lay.head_stride = cs->head_stride;
  lay.block_size = block_size;
  lay.head_dim = head_dim;
  const int64_t num_slots = static_cast<int64_t>(num_blocks) * block_size;
  const int grid = num_tokens < (1 << 20) ? num_tokens : (1 << 20);
  PdlLaunch launch(reinterpret_cast<cudaStream_t>(stream), dim3(grid), dim3(kRowThreads));
  const uint16_t* k = static_cast<const uint16_t*>(key);
  const uint16_t* v = static_cast<const uint16_t*>(value);
  const int32_t re = static_cast<int32_t>(row);
  if (kv_cache_dtype == PA_KV_FP8_E4M3) {
    if (!key || !value || !key_cache || !value_cache || !slot_mapping || !k_scale || !v_scale)
      return PA_ERR_INVALID_ARG;
    // 16-byte row loads and 8-byte code stores
    if (head_dim % 8 != 0 || key_stride_t % 8 != 0 || value_stride_t % 8 != 0 ||
        cs->block_stride % 8 != 0 || cs->token_stride % 8 != 0 || cs->head_stride % 8 != 0 ||
        !aligned(key, 16) || !aligned(value, 16) || !aligned(key_cache, 8) ||
        !aligned(value_cache, 8) || !aligned(slot_mapping, 4) || !aligned(k_scale, 4) ||
        !aligned(v_scale, 4))
      return PA_ERR_INVALID_ARG;
    uint8_t* kc = static_cast<uint8_t*>(key_cache);
    uint8_t* vc = static_cast<uint8_t*>(value_cache);
    const cudaError_t e =
        dtype == PA_BF16
            ? launch(pa_reshape_and_cache_fp8_kernel<true>, k, v, key_stride_t, value_stride_t,
                     kc, vc, lay, slot_mapping, num_tokens, num_slots, re, k_scale, v_scale,
                     device_error_flag)
            : launch(pa_reshape_and_cache_fp8_kernel<false>, k, v, key_stride_t, value_stride_t,
                     kc, vc, lay, slot_mapping, num_tokens, num_slots, re, k_scale, v_scale,
                     device_error_flag);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  }
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned(key, 2) || !aligned(value, 2) || !aligned(key_cache, 2) ||
      !aligned(value_cache, 2) || !aligned(slot_mapping, 4))
    return PA_ERR_INVALID_ARG;
  const bool vec = aligned(key, 16) && aligned(value, 16) && aligned(key_cache, 16) &&
                   aligned(value_cache, 16) && key_stride_t % 8 == 0 &&
                   value_stride_t % 8 == 0 && head_dim % 8 == 0 && cs->block_stride % 8 == 0 &&
                   cs->token_stride % 8 == 0 && cs->head_stride % 8 == 0;
  uint16_t* kc = static_cast<uint16_t*>(key_cache);
  uint16_t* vc = static_cast<uint16_t*>(value_cache);
  const cudaError_t e =
      vec ? launch(pa_reshape_and_cache_kernel<8>, k, v, key_stride_t, value_stride_t, kc, vc,
                   lay, slot_mapping, num_tokens, num_slots, re, device_error_flag)
          : launch(pa_reshape_and_cache_kernel<1>, k, v, key_stride_t, value_stride_t, kc, vc,
                   lay, slot_mapping, num_tokens, num_slots, re, device_error_flag);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

extern "C" pa_status pa_reshape_and_cache(const void* key, const void* value,
                                          int64_t key_stride_t, int64_t value_stride_t,
                                          void* key_cache, void* value_cache,
                                          const int32_t* slot_mapping, int32_t num_tokens,
                                          int32_t num_blocks, int32_t block_size,
                                          int32_t num_kv_heads, int32_t head_dim,
                                          pa_dtype dtype, pa_kv_cache_dtype kv_cache_dtype,
                                          const float* k_scale, const float* v_scale,
                                          int32_t* device_error_flag, pa_stream_t stream) {
  const pa_cache_strides cs = {static_cast<int64_t>(block_size) * num_kv_heads * head_dim,
                               static_cast<int64_t>(num_kv_heads) * head_dim, head_dim};
  return reshape_impl(key, value, key_stride_t, value_stride_t, key_cache, value_cache, &cs,
                      slot_mapping, num_tokens, num_blocks, block_size, num_kv_heads, head_dim,
                      dtype, kv_cache_dtype, k_scale, v_scale, device_error_flag, stream);
}

extern "C" pa_status pa_reshape_and_cache_strided(
    const void* key, const void* value, int64_t key_stride_t, int64_t value_stride_t,
    void* key_cache, void* value_cache, const pa_cache_strides* cache_strides,
    const int32_t* slot_mapping, int32_t num_tokens, int32_t num_blocks, int32_t block_size,
    int32_t num_kv_heads, int32_t head_dim, pa_dtype dtype, pa_kv_cache_dtype kv_cache_dtype,
    const float* k_scale, const float* v_scale, int32_t* device_error_flag,
    pa_stream_t stream) {
  if (cache_strides == nullptr) return PA_ERR_INVALID_ARG;
  return reshape_impl(key, value, key_stride_t, value_stride_t, key_cache, value_cache,
                      cache_strides, slot_mapping, num_tokens, num_blocks, block_size,
                      num_kv_heads, head_dim, dtype, kv_cache_dtype, k_scale, v_scale,
                      device_error_flag, stream);
}

extern "C" pa_status pa_copy_blocks(void* const* key_caches, void* const* value_caches,
                                    int32_t num_layers, const int32_t* block_mapping,
                                    int32_t num_pairs, int32_t num_blocks, int64_t block_bytes,
                                    int32_t* device_error_flag, pa_stream_t stream) {
  if (num_layers < 0 || num_pairs < 0 || num_blocks <= 0 || block_bytes <= 0)
    return PA_ERR_INVALID_ARG;
  if (num_layers == 0 || num_pairs == 0) return PA_OK;
  if (!key_caches || !value_caches || !block_mapping || !aligned(block_mapping, 4))
    return PA_ERR_INVALID_ARG;
  bool vec = block_bytes % 16 == 0;
  for (int32_t l = 0; l < num_layers; ++l) {
    if (!key_caches[l] || !value_caches[l]) return PA_ERR_INVALID_ARG;
    vec = vec && aligned(key_caches[l], 16) && aligned(value_caches[l], 16);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int layers_per_launch = kMaxCopyCaches / 2;
  for (int32_t l0 = 0; l0 < num_layers; l0 += layers_per_launch) {
    const int32_t nl = num_layers - l0 < layers_per_launch ? num_layers - l0 : layers_per_launch;
    CopyPtrs ptrs;
    for (int32_t l = 0; l < nl; ++l) {
      ptrs.p[2 * l] = static_cast<uint8_t*>(key_caches[l0 + l]);
      ptrs.p[2 * l + 1] = static_cast<uint8_t*>(value_caches[l0 + l]);
    }
    PdlLaunch launch(s, dim3(num_pairs, 2 * nl), dim3(kCopyThreads));
    const cudaError_t e =
        vec ? launch(pa_copy_blocks_kernel<true>, ptrs, block_mapping, num_blocks, block_bytes,
                     device_error_flag)
            : launch(pa_copy_blocks_kernel<false>, ptrs, block_mapping, num_blocks, block_bytes,
                     device_error_flag);
    if (e != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

extern "C" pa_status pa_copy_blocks_strided(void* const* key_caches, void* const* value_caches,
                                            int32_t num_layers,
                                            const pa_cache_strides* cache_strides,
                                            const int32_t* block_mapping, int32_t num_pairs,
                                            int32_t num_blocks, int32_t block_size,
                                            int32_t num_kv_heads, int32_t head_dim,
                                            int32_t elem_bytes, int32_t* device_error_flag,
                                            pa_stream_t stream) {
  if (num_layers < 0 || num_pairs < 0 || num_blocks <= 0 || block_size <= 0 ||
      num_kv_heads <= 0 || head_dim <= 0 || (elem_bytes != 1 && elem_bytes != 2) ||
      cache_strides == nullptr)
    return PA_ERR_INVALID_ARG;
  const pa_cache_strides& cs = *cache_strides;
  if (cs.block_stride <= 0 || cs.token_stride <= 0 || cs.head_stride <= 0)
    return PA_ERR_INVALID_ARG;
  if (num_layers == 0 || num_pairs == 0) return PA_OK;
  if (!key_caches || !value_caches || !block_mapping || !aligned(block_mapping, 4))
    return PA_ERR_INVALID_ARG;
  const int64_t row_bytes = static_cast<int64_t>(head_dim) * elem_bytes;
  // whole 16-byte pieces: rows and every stride
  if (row_bytes % 16 != 0 || (cs.block_stride * elem_bytes) % 16 != 0 ||
      (cs.token_stride * elem_bytes) % 16 != 0 || (cs.head_stride * elem_bytes) % 16 != 0)
    return PA_ERR_INVALID_ARG;
  for (int32_t l = 0; l < num_layers; ++l) {
    if (!key_caches[l] || !value_caches[l] || !aligned(key_caches[l], 16) ||
        !aligned(value_caches[l], 16))
      return PA_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int layers_per_launch = kMaxCopyCaches / 2;
  for (int32_t l0 = 0; l0 < num_layers; l0 += layers_per_launch) {
    const int32_t nl = num_layers - l0 < layers_per_launch ? num_layers - l0 : layers_per_launch;
    CopyPtrs ptrs;
    for (int32_t l = 0; l < nl; ++l) {
      ptrs.p[2 * l] = static_cast<uint8_t*>(key_caches[l0 + l]);
      ptrs.p[2 * l + 1] = static_cast<uint8_t*>(value_caches[l0 + l]);
    }
    PdlLaunch launch(s, dim3(num_pairs, 2 * nl), dim3(kCopyThreads));
    const cudaError_t e = launch(pa_copy_blocks_strided_kernel, ptrs, block_mapping, num_blocks,
                                 cs.block_stride * elem_bytes, cs.token_stride * elem_bytes,
                                 cs.head_stride * elem_bytes, block_size, num_kv_heads,
                                 static_cast<int32_t>(row_bytes), device_error_flag);
    if (e != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}
