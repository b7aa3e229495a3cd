// paged_attn_cascade.cu — the shared-prefix pass of cascade decode: shape
// dispatch and launch.  The kernels are the chunked-prefill kernels in prefix
// mode (paged_prefill_tc_kernels.cuh for head_dim 128,
// paged_prefill_kernels.cuh for 64); the entry points that run this pass and
// the decode of each member's own blocks are in paged_attn_decode.cu.
#include <cudaTypedefs.h>

#include "host_common.h"
#include "paged_prefill_kernels.cuh"
#include "paged_prefill_tc_kernels.cuh"

namespace pkv {
namespace {

using PrefixFn = void (*)(const PrefillParams, const CUtensorMap, const CUtensorMap);
using TcPrefixFn = void (*)(const PrefillParams, const CUtensorMap, const CUtensorMap,
                            const CUtensorMap);

struct PrefixEntry {
  PrefixFn fn;        // mma.sync kernel (head_dim 64), else null
  TcPrefixFn tc_fn;   // tcgen05 kernel (head_dim 128), else null
  int threads;
  size_t smem;
  int rows;           // query rows per CTA: (member, head) pairs
};

constexpr int kPrefixMmaStages = 4;

// head_dim 128: the tcgen05 kernel with one 128-row query tile per CTA
template <int BS, int G, class DT, bool FP8>
PrefixEntry make_tc_prefix() {
  using Tr = TcPrefillTraits<BS, G, DT, 1, true, FP8>;
  return PrefixEntry{nullptr, paged_prefill_tc_kernel<Tr>, Tr::THREADS, Tr::smem_bytes(),
                     Tr::ROWS};
}

// head_dim 64: the mma.sync kernel, 64 rows per CTA
template <int D, int BS, int G, class DT, bool FP8>
PrefixEntry make_mma_prefix() {
  using Tr = PrefillTraits<D, BS, G, DT, kPrefixMmaStages, true, FP8>;
  return PrefixEntry{paged_prefill_kernel<Tr>, nullptr, Tr::THREADS, Tr::smem_bytes(), Tr::ROWS};
}

// (The mma.sync kernel at head_dim 128 measured slower than the tcgen05 one as
// the prefix pass of the parallel-sampling batch on B200: 0.222 against 0.192
// ms per cascade decode.)
template <int D, int BS, int G, class DT, bool FP8>
PrefixEntry make_prefix() {
  if constexpr (D == 128) return make_tc_prefix<BS, G, DT, FP8>();
  else return make_mma_prefix<D, BS, G, DT, FP8>();
}

template <int D, int BS, class DT, bool FP8>
PrefixEntry prefix_group(int g) {
  switch (g) {
    case 1: return make_prefix<D, BS, 1, DT, FP8>();
    case 2: return make_prefix<D, BS, 2, DT, FP8>();
    case 4: return make_prefix<D, BS, 4, DT, FP8>();
    case 8: return make_prefix<D, BS, 8, DT, FP8>();
    default: return PrefixEntry{nullptr, nullptr, 0, 0, 0};
  }
}

template <class DT, bool FP8>
PrefixEntry prefix_for(int d, int bs, int g) {
  if (d == 128 && bs == 16) return prefix_group<128, 16, DT, FP8>(g);
  if (d == 128 && bs == 32) return prefix_group<128, 32, DT, FP8>(g);
  if (d == 64 && bs == 16) return prefix_group<64, 16, DT, FP8>(g);
  if (d == 64 && bs == 32) return prefix_group<64, 32, DT, FP8>(g);
  return PrefixEntry{nullptr, nullptr, 0, 0, 0};
}

}  // namespace

pkv_status launch_cascade_prefix(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* block_tables, const int32_t* context_lens,
                                 const CascadeGroups& groups, float scale, int num_seqs,
                                 int num_heads, int num_kv_heads, int head_dim, int block_size,
                                 int max_blocks_per_seq, int max_context_len, int num_blocks,
                                 pkv_dtype dtype, bool fp8, const float* k_scales,
                                 const float* v_scales, float* ws_out, float* ws_max,
                                 float* ws_sum, int max_parts, unsigned* dev_err,
                                 cudaStream_t stream) {
  const int group = num_heads / num_kv_heads;
  const bool f16 = dtype == PKV_FP16;
  const PrefixEntry pe = fp8 ? (f16 ? prefix_for<Fp16, true>(head_dim, block_size, group)
                                    : prefix_for<Bf16, true>(head_dim, block_size, group))
                             : (f16 ? prefix_for<Fp16, false>(head_dim, block_size, group)
                                    : prefix_for<Bf16, false>(head_dim, block_size, group));
  if (pe.fn == nullptr && pe.tc_fn == nullptr) return PKV_ERR_UNSUPPORTED;
  if (fp8 && (!k_scales || !v_scales)) return PKV_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(groups.max_group_size) * group;
  const int q_tiles = static_cast<int>((rows + pe.rows - 1) / pe.rows);
  const long long grid = static_cast<long long>(groups.num_groups) * num_kv_heads * q_tiles;
  if (grid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;
  if (grid == 0) return PKV_OK;
  CUtensorMap kmap, vmap, qmap;
  const pkv_dtype cdt = fp8 ? PKV_FP8_E4M3 : dtype;  // element type of the caches
  pkv_status st =
      cache_tensor_map(&kmap, k_cache, num_blocks, num_kv_heads, block_size, head_dim, cdt);
  if (st != PKV_OK) return st;
  st = cache_tensor_map(&vmap, v_cache, num_blocks, num_kv_heads, block_size, head_dim, cdt);
  if (st != PKV_OK) return st;
  if (pe.tc_fn != nullptr) {
    st = q_tensor_map(&qmap, q, num_seqs, num_heads, group, dtype);  // the members' queries
    if (st != PKV_OK) return st;
  }
  const void* fn = pe.tc_fn != nullptr ? reinterpret_cast<const void*>(pe.tc_fn)
                                       : reinterpret_cast<const void*>(pe.fn);
  st = cuda_status(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(pe.smem)));
  if (st != PKV_OK) return st;

  PrefillParams p = {};
  p.q = q;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.qscale = scale * kLog2e;
  p.num_seqs = groups.num_groups;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_context_len = max_context_len;
  p.max_query_len = groups.max_group_size;
  p.num_blocks = num_blocks;
  p.q_tiles = q_tiles;
  p.err = dev_err;
  p.k_scales = k_scales;
  p.v_scales = v_scales;
  p.group_start = groups.group_start;
  p.shared_blocks = groups.shared_blocks;
  p.max_shared_blocks = groups.max_shared_blocks;
  p.ws_out = ws_out;
  p.ws_max = ws_max;
  p.ws_sum = ws_sum;
  p.max_parts = max_parts;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(pe.threads);
  cfg.dynamicSmemBytes = pe.smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (pe.tc_fn != nullptr)
    return cuda_status(cudaLaunchKernelEx(&cfg, pe.tc_fn, p, qmap, kmap, vmap));
  return cuda_status(cudaLaunchKernelEx(&cfg, pe.fn, p, kmap, vmap));
}

}  // namespace pkv
