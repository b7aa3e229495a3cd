// copy_blocks.cu — copy-on-write copy of whole physical blocks.
//
// Samples of one prompt share its blocks through their block tables; blocks
// are reference-counted and a block that several holders must modify is
// copied first ([cortexgrid] FAQ answer on parallel sampling).  The copy is of
// the whole block: every kv head, offset and dimension, for K and for V.
//
// Grid: (pair, K-or-V).  Each CTA streams one block (num_kv_heads *
// block_size * head_dim * 2 bytes, 32 KiB for 8 kv heads at block 16 / dim 128)
// with 16-byte loads, four in flight per thread before the stores.
#include "common.cuh"
#include "host_common.h"

namespace pkv {

__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* k_cache, uint4* v_cache,
                                                          const int64_t* __restrict__ mapping,
                                                          int64_t vecs_per_block,
                                                          int64_t num_blocks, unsigned* err) {
  const int pair = blockIdx.x;
  const int64_t src = mapping[2 * pair];
  const int64_t dst = mapping[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_err(err, PKV_DEVERR_BAD_PAIR);
    return;
  }
  uint4* cache = blockIdx.y == 0 ? k_cache : v_cache;
  const uint4* s = cache + src * vecs_per_block;
  uint4* d = cache + dst * vecs_per_block;
  constexpr int kBatch = 4;
  for (int64_t base = threadIdx.x; base < vecs_per_block; base += kBatch * blockDim.x) {
    uint4 v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t j = base + i * blockDim.x;
      if (j < vecs_per_block) v[i] = s[j];
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t j = base + i * blockDim.x;
      if (j < vecs_per_block) d[j] = v[i];
    }
  }
}

}  // namespace pkv

extern "C" pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                                      int num_pairs, int num_kv_heads, int head_dim,
                                      int block_size, int num_blocks, pkv_dtype dtype,
                                      unsigned* dev_err, void* stream) {
  using namespace pkv;
  if (num_pairs < 0 || num_kv_heads <= 0 || num_blocks <= 0 || !cache_dtype_valid(dtype))
    return PKV_ERR_INVALID_ARG;
  if (!head_dim_supported(head_dim) || !block_size_supported(block_size))
    return PKV_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PKV_OK;
  if (!k_cache || !v_cache || !block_mapping) return PKV_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return PKV_ERR_INVALID_ARG;
  // 16-byte vectors per block: 8 elements of a 16-bit cache, 16 of an E4M3 cache
  const int64_t vecs = static_cast<int64_t>(num_kv_heads) * block_size * head_dim *
                       cache_elem_bytes(dtype) / 16;
  dim3 grid(static_cast<unsigned>(num_pairs), 2);
  copy_blocks_kernel<<<grid, 256, 0, as_stream(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), block_mapping, vecs,
      num_blocks, dev_err);
  return cuda_status(cudaGetLastError());
}
