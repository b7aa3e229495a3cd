// paged_attn_prefill.cu — host side of chunked-prefill attention: validation,
// shape dispatch and the C entry point.  The kernel is in
// paged_prefill_kernels.cuh.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include <type_traits>

#include "host_common.h"
#include "paged_prefill_kernels.cuh"
#include "paged_prefill_tc_kernels.cuh"

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

template <int D, int BS, int G, class DT, bool FP8>
PrefillEntry make_prefill() {
  using Tr = PrefillTraits<D, BS, G, DT, kPrefillStages, false, FP8>;
  return PrefillEntry{paged_prefill_kernel<Tr>, Tr::THREADS, Tr::smem_bytes(), Tr::ROWS};
}

template <int D, int BS, class DT, bool FP8>
PrefillEntry prefill_group(int g) {
  switch (g) {
    case 1: return make_prefill<D, BS, 1, DT, FP8>();
    case 2: return make_prefill<D, BS, 2, DT, FP8>();
    case 4: return make_prefill<D, BS, 4, DT, FP8>();
    case 8: return make_prefill<D, BS, 8, DT, FP8>();
    default: return PrefillEntry{nullptr, 0, 0, 0};
  }
}

// (head_dim, block size, group) -> mma.sync kernel; fp8: the cache holds E4M3
// codes (head_dim 64)
template <class DT, bool FP8 = false>
PrefillEntry prefill_for(int d, int bs, int g) {
  if constexpr (!FP8) {
    if (d == 128 && bs == 16) return prefill_group<128, 16, DT, false>(g);
    if (d == 128 && bs == 32) return prefill_group<128, 32, DT, false>(g);
  }
  if (d == 64 && bs == 16) return prefill_group<64, 16, DT, FP8>(g);
  if (d == 64 && bs == 32) return prefill_group<64, 32, DT, FP8>(g);
  return PrefillEntry{nullptr, 0, 0, 0};
}

// ---- tcgen05 kernel (head_dim 128) -----------------------------------------------
using TcPrefillFn = void (*)(const PrefillParams, const CUtensorMap, const CUtensorMap,
                             const CUtensorMap);

struct TcEntry {
  TcPrefillFn fn;
  int threads;
  size_t smem;
  int rows;  // query rows per CTA
};

// Query tiles of 128 rows per CTA.  Two share every K/V tile, which halves the
// TMA traffic per FLOP (the per-SM TMA engine paces the one-tile kernel).
// Measured on B200 (kernel TFLOP/s, fp16, one tile -> two): 4 x 512 new tokens
// on 2048 cached 376 -> 482, 2048 on 8192 cached 419 -> 607, the LLaMA-7B
// prefill batch 350 -> 411.  bf16 (P split into hi + lo halves) gained once P
// moved to TMEM with two query tiles: the GQA prefill batch 388 -> 453.
#ifndef PKV_PREFILL_QUERY_TILES
#define PKV_PREFILL_QUERY_TILES 2
#endif
template <class DT>
constexpr int kTcQueryTiles = PKV_PREFILL_QUERY_TILES;

#ifndef PKV_PREFILL_NKEY
#define PKV_PREFILL_NKEY 64
#endif
template <int BS, int G, class DT, bool FP8>
TcEntry make_tc() {
  using Tr = TcPrefillTraits<BS, G, DT, kTcQueryTiles<DT>, false, FP8, FP8 ? 64 : PKV_PREFILL_NKEY>;
  return TcEntry{paged_prefill_tc_kernel<Tr>, Tr::THREADS, Tr::smem_bytes(), Tr::ROWS};
}

template <int BS, class DT, bool FP8>
TcEntry tc_group(int g) {
  switch (g) {
    case 1: return make_tc<BS, 1, DT, FP8>();
    case 2: return make_tc<BS, 2, DT, FP8>();
    case 4: return make_tc<BS, 4, DT, FP8>();
    case 8: return make_tc<BS, 8, DT, FP8>();
    default: return TcEntry{nullptr, 0, 0, 0};
  }
}

// (block size, group) -> tcgen05 kernel; fp8: the cache holds E4M3 codes
template <class DT, bool FP8 = false>
TcEntry tc_for(int bs, int g) {
  if (bs == 16) return tc_group<16, DT, FP8>(g);
  if (bs == 32) return tc_group<32, DT, FP8>(g);
  return TcEntry{nullptr, 0, 0, 0};
}

}  // namespace
}  // namespace pkv

namespace pkv {

pkv_status q_tensor_map(CUtensorMap* out, const void* q, int num_tokens, int num_heads, int group,
                        pkv_dtype dt) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  if (enc == nullptr) return cuda_status(cudaErrorNotSupported);
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(num_heads),
                        static_cast<cuuint64_t>(num_tokens)};
  cuuint64_t strides[2] = {128 * 2, static_cast<cuuint64_t>(num_heads) * 128 * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(128 / group)};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r =
      enc(out, dt == PKV_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
          3, const_cast<void*>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : cuda_status(cudaErrorInvalidValue);
}

}  // namespace pkv

namespace pkv {
namespace {

// Validates and launches prefill; fp8: the caches hold E4M3 codes with
// per-kv-head scales k_scales / v_scales.
pkv_status prefill_launch(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens,
                          const int32_t* query_start, float scale, int num_seqs, int num_tokens,
                          int num_heads, int num_kv_heads, int head_dim, int block_size,
                          int max_blocks_per_seq, int max_context_len, int max_query_len,
                          int num_blocks, pkv_dtype dtype, bool fp8, const float* k_scales,
                          const float* v_scales, unsigned* dev_err, void* stream) {
  if (num_seqs < 0 || num_tokens < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
      max_blocks_per_seq <= 0 ||
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
  if (fp8 && (!k_scales || !v_scales)) return PKV_ERR_INVALID_ARG;
  if (num_seqs == 0 || max_query_len == 0 || num_tokens == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_INVALID_ARG;
  const bool use_tc = head_dim == 128;
  const PrefillEntry pe =
      use_tc ? PrefillEntry{nullptr, 0, 0, 0}
      : fp8  ? (dtype == PKV_FP16 ? prefill_for<Fp16, true>(head_dim, block_size, group)
                                  : prefill_for<Bf16, true>(head_dim, block_size, group))
      : dtype == PKV_FP16 ? prefill_for<Fp16>(head_dim, block_size, group)
                          : prefill_for<Bf16>(head_dim, block_size, group);
  const TcEntry te = !use_tc ? TcEntry{nullptr, 0, 0, 0}
                     : fp8 ? (dtype == PKV_FP16 ? tc_for<Fp16, true>(block_size, group)
                                                : tc_for<Bf16, true>(block_size, group))
                     : dtype == PKV_FP16 ? tc_for<Fp16>(block_size, group)
                                         : tc_for<Bf16>(block_size, group);
  if (pe.fn == nullptr && te.fn == nullptr) return PKV_ERR_UNSUPPORTED;
  const int tile_rows = use_tc ? te.rows : pe.rows;
  const long long rows = static_cast<long long>(max_query_len) * group;
  const int q_tiles = static_cast<int>((rows + tile_rows - 1) / tile_rows);
  const long long grid = static_cast<long long>(num_seqs) * num_kv_heads * q_tiles;
  if (grid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;

  CUtensorMap kmap, vmap, qmap;
  const pkv_dtype cdt = fp8 ? PKV_FP8_E4M3 : dtype;  // element type of the caches
  pkv_status st =
      cache_tensor_map(&kmap, k_cache, num_blocks, num_kv_heads, block_size, head_dim, cdt);
  if (st != PKV_OK) return st;
  st = cache_tensor_map(&vmap, v_cache, num_blocks, num_kv_heads, block_size, head_dim, cdt);
  if (st != PKV_OK) return st;
  if (use_tc) {
    st = q_tensor_map(&qmap, q, num_tokens, num_heads, group, dtype);
    if (st != PKV_OK) return st;
  }
  const void* fn = use_tc ? reinterpret_cast<const void*>(te.fn)
                          : reinterpret_cast<const void*>(pe.fn);
  const size_t smem = use_tc ? te.smem : pe.smem;
  st = cuda_status(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(smem)));
  if (st != PKV_OK) return st;

  PrefillParams p = {};
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
  p.k_scales = k_scales;
  p.v_scales = v_scales;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(use_tc ? te.threads : pe.threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = as_stream(stream);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (use_tc) return cuda_status(cudaLaunchKernelEx(&cfg, te.fn, p, qmap, kmap, vmap));
  return cuda_status(cudaLaunchKernelEx(&cfg, pe.fn, p, kmap, vmap));
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_paged_attn_prefill(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
    float scale, int num_seqs, int num_tokens, int num_heads, int num_kv_heads, int head_dim,
    int block_size, int max_blocks_per_seq, int max_context_len, int max_query_len,
    int num_blocks, pkv_dtype dtype, unsigned* dev_err, void* stream) {
  return pkv::prefill_launch(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                             scale, num_seqs, num_tokens, num_heads, num_kv_heads, head_dim,
                             block_size, max_blocks_per_seq, max_context_len, max_query_len,
                             num_blocks, dtype, false, nullptr, nullptr, dev_err, stream);
}

extern "C" pkv_status pkv_paged_attn_prefill_fp8(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
    float scale, const float* k_scales, const float* v_scales, int num_seqs, int num_tokens,
    int num_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
    int max_context_len, int max_query_len, int num_blocks, pkv_dtype dtype, unsigned* dev_err,
    void* stream) {
  return pkv::prefill_launch(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                             scale, num_seqs, num_tokens, num_heads, num_kv_heads, head_dim,
                             block_size, max_blocks_per_seq, max_context_len, max_query_len,
                             num_blocks, dtype, true, k_scales, v_scales, dev_err, stream);
}
