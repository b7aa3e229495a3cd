// paged_attn_prefill.cu — host side of chunked-prefill attention: validation,
// shape dispatch and the C entry point.  The kernel is in
// paged_prefill_kernels.cuh.
#include <math.h>

#include "host_common.h"
#include "paged_prefill_kernels.cuh"

namespace pkv {
namespace {

using PrefillFn = void (*)(const PrefillParams, const CUtensorMap, const CUtensorMap);

struct PrefillEntry {
  PrefillFn fn;
  int threads;
  size_t smem;
  int rows;
};

constexpr int kPrefillStages = 4;

template <int D, int BS, int G, class DT>
PrefillEntry make_prefill() {
  using Tr = PrefillTraits<D, BS, G, DT, kPrefillStages>;
  return PrefillEntry{paged_prefill_kernel<Tr>, Tr::THREADS, Tr::smem_bytes(), Tr::ROWS};
}

template <int D, int BS, class DT>
PrefillEntry prefill_group(int g) {
  switch (g) {
    case 1: return make_prefill<D, BS, 1, DT>();
    case 2: return make_prefill<D, BS, 2, DT>();
    case 4: return make_prefill<D, BS, 4, DT>();
    case 8: return make_prefill<D, BS, 8, DT>();
    default: return PrefillEntry{nullptr, 0, 0, 0};
  }
}

template <class DT>
PrefillEntry prefill_for(int d, int bs, int g) {
  if (d == 128 && bs == 16) return prefill_group<128, 16, DT>(g);
  if (d == 128 && bs == 32) return prefill_group<128, 32, DT>(g);
  if (d == 64 && bs == 16) return prefill_group<64, 16, DT>(g);
  if (d == 64 && bs == 32) return prefill_group<64, 32, DT>(g);
  return PrefillEntry{nullptr, 0, 0, 0};
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_paged_attn_prefill(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
    float scale, int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int max_context_len, int max_query_len, int num_blocks,
    pkv_dtype dtype, unsigned* dev_err, void* stream) {
  using namespace pkv;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 ||
      max_context_len < 0 || max_query_len < 0 || num_blocks <= 0 || !dtype_valid(dtype) ||
      num_heads % num_kv_heads != 0 || !isfinite(scale) || max_query_len > max_context_len)
    return PKV_ERR_INVALID_ARG;
  if (!head_dim_supported(head_dim) || !block_size_supported(block_size))
    return PKV_ERR_UNSUPPORTED;
  const int group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return PKV_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_context_len) >
      static_cast<long long>(max_blocks_per_seq) * block_size)
    return PKV_ERR_INVALID_ARG;
  if (num_seqs == 0 || max_query_len == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_INVALID_ARG;
  const PrefillEntry pe = dtype == PKV_FP16 ? prefill_for<Fp16>(head_dim, block_size, group)
                                            : prefill_for<Bf16>(head_dim, block_size, group);
  if (pe.fn == nullptr) return PKV_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(max_query_len) * group;
  const int q_tiles = static_cast<int>((rows + pe.rows - 1) / pe.rows);
  const long long grid = static_cast<long long>(num_seqs) * num_kv_heads * q_tiles;
  if (grid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;

  CUtensorMap kmap, vmap;
  pkv_status st =
      cache_tensor_map(&kmap, k_cache, num_blocks, num_kv_heads, block_size, head_dim, dtype);
  if (st != PKV_OK) return st;
  st = cache_tensor_map(&vmap, v_cache, num_blocks, num_kv_heads, block_size, head_dim, dtype);
  if (st != PKV_OK) return st;
  st = cuda_status(cudaFuncSetAttribute(reinterpret_cast<const void*>(pe.fn),
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(pe.smem)));
  if (st != PKV_OK) return st;

  PrefillParams p;
  p.out = out;
  p.q = q;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.query_start = query_start;
  p.qscale = scale * kLog2e;
  p.num_seqs = num_seqs;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_context_len = max_context_len;
  p.max_query_len = max_query_len;
  p.num_blocks = num_blocks;
  p.q_tiles = q_tiles;
  p.err = dev_err;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(pe.threads);
  cfg.dynamicSmemBytes = pe.smem;
  cfg.stream = as_stream(stream);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, pe.fn, p, kmap, vmap));
}
