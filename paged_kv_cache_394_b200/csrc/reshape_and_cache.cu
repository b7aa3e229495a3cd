// reshape_and_cache.cu — scatter new tokens' K/V into their cache slots.
//
// Each cached token keeps one K and one V vector per kv head ([csdn]
// "内存困局的破局者：PagedAttention 是如何工作的？"); a sequence's cache grows a
// page at a time ([betteryeah] §2.2 "PagedAttention的分页机制").  Writing a new
// token is a pure copy into (block = slot / block_size, offset = slot %
// block_size), bit for bit.
//
// One thread moves one 16-byte chunk of K and the matching chunk of V, so a
// warp writes whole 256-byte rows (head_dim 128) with coalesced 16-byte
// stores.  The data type does not matter for a copy, so one kernel serves
// fp16 and bf16.
#include "common.cuh"
#include "host_common.h"

namespace pkv {

__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, int num_tokens,
    int num_kv_heads, int chunks_per_row, int block_size, int64_t num_slots, unsigned* err) {
  // Launched with programmatic serialisation: wait for the previous kernel
  // (the last step's decode reads the cache) before touching memory; the
  // decode kernel that usually follows may then start its prologue, and it
  // still waits for this grid to finish before reading the cache.
  grid_dependency_wait();
  trigger_dependents();
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * chunks_per_row;
  if (idx >= per_token * num_tokens) return;
  const int t = static_cast<int>(idx / per_token);
  const int64_t within = idx - t * per_token;  // (head, chunk) of this token
  const int64_t slot = slot_mapping[t];
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (within == 0) set_err(err, PKV_DEVERR_BAD_SLOT);
    return;
  }
  const int64_t block = slot / block_size;
  const int64_t offset = slot - block * block_size;
  const int head = static_cast<int>(within / chunks_per_row);
  const int chunk = static_cast<int>(within - static_cast<int64_t>(head) * chunks_per_row);
  const int64_t dst = ((block * num_kv_heads + head) * block_size + offset) * chunks_per_row + chunk;
  const int64_t src = static_cast<int64_t>(t) * per_token + within;
  k_cache[dst] = key[src];
  v_cache[dst] = value[src];
}

// E4M3 variant: the same scatter, quantising on the way in.  One thread reads
// 8 elements (16 bytes) of K and of V and writes 8 codes (8 bytes) of each,
// so a warp still stores whole rows.
template <class DT>
__device__ __forceinline__ uint2 quantize8(const uint4& raw, float scale) {
  float f[8];
  unpack8(raw, f, DT());
  uint32_t w[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      // IEEE float32 division, then E4M3 round-to-nearest-even, saturating
      const float2 x = make_float2(__fdiv_rn(f[4 * i + 2 * j], scale),
                                   __fdiv_rn(f[4 * i + 2 * j + 1], scale));
      const __nv_fp8x2_storage_t pair = __nv_cvt_float2_to_fp8x2(x, __NV_SATFINITE, __NV_E4M3);
      word |= static_cast<uint32_t>(pair) << (16 * j);
    }
    w[i] = word;
  }
  return make_uint2(w[0], w[1]);
}

template <class DT>
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, uint2* __restrict__ k_cache,
    uint2* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, int num_tokens,
    int num_kv_heads, int chunks_per_row, int block_size, int64_t num_slots,
    const float* __restrict__ k_scales, const float* __restrict__ v_scales, unsigned* err) {
  grid_dependency_wait();
  trigger_dependents();
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * chunks_per_row;
  if (idx >= per_token * num_tokens) return;
  const int t = static_cast<int>(idx / per_token);
  const int64_t within = idx - t * per_token;
  const int64_t slot = slot_mapping[t];
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (within == 0) set_err(err, PKV_DEVERR_BAD_SLOT);
    return;
  }
  const int64_t block = slot / block_size;
  const int64_t offset = slot - block * block_size;
  const int head = static_cast<int>(within / chunks_per_row);
  const int chunk = static_cast<int>(within - static_cast<int64_t>(head) * chunks_per_row);
  const int64_t dst = ((block * num_kv_heads + head) * block_size + offset) * chunks_per_row + chunk;
  const int64_t src = static_cast<int64_t>(t) * per_token + within;
  const float ks = k_scales[head], vs = v_scales[head];
  if (!(ks > 0.f && ks < INFINITY && vs > 0.f && vs < INFINITY)) {
    if (chunk == 0) set_err(err, PKV_DEVERR_BAD_SCALE);
    return;
  }
  k_cache[dst] = quantize8<DT>(key[src], ks);
  v_cache[dst] = quantize8<DT>(value[src], vs);
}

}  // namespace pkv

extern "C" pkv_status pkv_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                            void* v_cache, const int64_t* slot_mapping,
                                            int num_tokens, int num_kv_heads, int head_dim,
                                            int block_size, int num_blocks, pkv_dtype dtype,
                                            unsigned* dev_err, void* stream) {
  using namespace pkv;
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0 || !dtype_valid(dtype))
    return PKV_ERR_INVALID_ARG;
  if (!head_dim_supported(head_dim) || !block_size_supported(block_size))
    return PKV_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PKV_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_INVALID_ARG;
  const int chunks = head_dim / 8;
  const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * chunks;
  const int threads = 256;
  const int64_t grid = (total + threads - 1) / threads;
  if (grid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;
  return cuda_status(launch_after_previous(
      reshape_and_cache_kernel, dim3(static_cast<unsigned>(grid)), dim3(threads), stream,
      static_cast<const uint4*>(key), static_cast<const uint4*>(value),
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), slot_mapping, num_tokens,
      num_kv_heads, chunks, block_size, static_cast<int64_t>(num_blocks) * block_size, dev_err));
}

extern "C" pkv_status pkv_reshape_and_cache_fp8(const void* key, const void* value,
                                                void* k_cache, void* v_cache,
                                                const int64_t* slot_mapping, int num_tokens,
                                                int num_kv_heads, int head_dim, int block_size,
                                                int num_blocks, pkv_dtype dtype,
                                                const float* k_scales, const float* v_scales,
                                                unsigned* dev_err, void* stream) {
  using namespace pkv;
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0 || !dtype_valid(dtype))
    return PKV_ERR_INVALID_ARG;
  if (!head_dim_supported(head_dim) || !block_size_supported(block_size))
    return PKV_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PKV_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping || !k_scales || !v_scales)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_INVALID_ARG;
  const int chunks = head_dim / 8;
  const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * chunks;
  const int threads = 256;
  const int64_t grid = (total + threads - 1) / threads;
  if (grid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;
  auto kernel = dtype == PKV_FP16 ? reshape_and_cache_fp8_kernel<Fp16>
                                  : reshape_and_cache_fp8_kernel<Bf16>;
  return cuda_status(launch_after_previous(
      kernel, dim3(static_cast<unsigned>(grid)), dim3(threads), stream,
      static_cast<const uint4*>(key), static_cast<const uint4*>(value),
      static_cast<uint2*>(k_cache), static_cast<uint2*>(v_cache), slot_mapping, num_tokens,
      num_kv_heads, chunks, block_size, static_cast<int64_t>(num_blocks) * block_size, k_scales,
      v_scales, dev_err));
}
