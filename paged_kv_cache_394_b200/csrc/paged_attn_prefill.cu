// paged_attn_prefill.cu — host side of chunked-prefill attention: validation,
// shape dispatch and the C entry point.  The kernel is in
// paged_prefill_kernels.cuh.
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <mutex>
#include <type_traits>
#include <vector>

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

// Planned prefill: the work items and merge entries of pkv_prefill_plan on
// the device, and the workspace for the pieces' partials.
struct PrefillPlanArgs {
  const int32_t* work;
  int num_items;
  const int32_t* merges;
  int num_merges;
  void* workspace;
  size_t workspace_bytes;
};

// Rows of a planned unit: the tcgen05 kernel's query rows per CTA.
constexpr int kPlanRows = PKV_PREFILL_QUERY_TILES * 128;

struct PlanWorkspace {
  size_t out_off, max_off, sum_off, total;
};

// [num_merges][H_kv][kPlanRows][kMaxPieces] partial rows: o (128 floats), m, l
PlanWorkspace plan_workspace(int num_merges, int num_kv_heads) {
  const size_t n = static_cast<size_t>(num_merges) * num_kv_heads * kPlanRows * kMaxPieces;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  PlanWorkspace w;
  w.out_off = 0;
  w.max_off = up(n * 128 * sizeof(float));
  w.sum_off = w.max_off + up(n * sizeof(float));
  w.total = w.sum_off + up(n * sizeof(float));
  return w;
}

// Validates and launches prefill; fp8: the caches hold E4M3 codes with
// per-kv-head scales k_scales / v_scales.
pkv_status prefill_launch(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens,
                          const int32_t* query_start, float scale, int num_seqs, int num_tokens,
                          int num_heads, int num_kv_heads, int head_dim, int block_size,
                          int max_blocks_per_seq, int max_context_len, int max_query_len,
                          int num_blocks, pkv_dtype dtype, bool fp8, const float* k_scales,
                          const float* v_scales, unsigned* dev_err, void* stream,
                          const PrefillPlanArgs* plan = nullptr) {
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
  if (plan != nullptr) {
    // the plan's units are the tcgen05 kernel's (head_dim 128); its pieces
    // write partials into the workspace that the merge kernel combines
    if (!use_tc) return PKV_ERR_UNSUPPORTED;
    if (plan->work == nullptr || plan->num_items < 0 || plan->num_merges < 0 ||
        (plan->num_merges > 0 && plan->merges == nullptr))
      return PKV_ERR_INVALID_ARG;
    if (plan->num_merges > 0) {
      const PlanWorkspace pw = plan_workspace(plan->num_merges, num_kv_heads);
      if (plan->workspace == nullptr || plan->workspace_bytes < pw.total)
        return PKV_ERR_WORKSPACE;
      if (!aligned16(plan->workspace)) return PKV_ERR_INVALID_ARG;
    }
  }
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
  const long long grid =
      static_cast<long long>(plan ? plan->num_items : num_seqs * static_cast<long long>(q_tiles)) *
      num_kv_heads;
  if (grid > 0x7fffffffLL ||
      (plan && static_cast<long long>(plan->num_merges) * num_kv_heads * (kPlanRows / 8) >
                   0x7fffffffLL))
    return PKV_ERR_UNSUPPORTED;
  if (plan && tile_rows != kPlanRows) return PKV_ERR_UNSUPPORTED;
  if (grid == 0) return PKV_OK;

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
  if (plan != nullptr) {
    p.work = plan->work;
    p.merges = plan->merges;
    p.num_merges = plan->num_merges;
    p.unit_rows = kPlanRows;
    if (plan->num_merges > 0) {
      const PlanWorkspace pw = plan_workspace(plan->num_merges, num_kv_heads);
      unsigned char* ws = static_cast<unsigned char*>(plan->workspace);
      p.ws_out = reinterpret_cast<float*>(ws + pw.out_off);
      p.ws_max = reinterpret_cast<float*>(ws + pw.max_off);
      p.ws_sum = reinterpret_cast<float*>(ws + pw.sum_off);
    }
  }

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
  if (!use_tc) return cuda_status(cudaLaunchKernelEx(&cfg, pe.fn, p, kmap, vmap));
  st = cuda_status(cudaLaunchKernelEx(&cfg, te.fn, p, qmap, kmap, vmap));
  if (st != PKV_OK || plan == nullptr || plan->num_merges == 0) return st;
  cudaLaunchConfig_t mcfg = cfg;
  mcfg.gridDim = dim3(static_cast<unsigned>(plan->num_merges * num_kv_heads * (kPlanRows / 8)));
  mcfg.blockDim = dim3(256);
  mcfg.dynamicSmemBytes = 0;
  return cuda_status(dtype == PKV_FP16
                         ? cudaLaunchKernelEx(&mcfg, paged_prefill_merge_kernel<Fp16>, p)
                         : cudaLaunchKernelEx(&mcfg, paged_prefill_merge_kernel<Bf16>, p));
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

// ---------------------------------------------------------------------------
// Planned prefill.  A (sequence, query tile) unit of the tcgen05 kernel reads
// every key its rows see; in a batch of few sequences the units of the
// longest history outlast the rest and the launch ends on them.  The planner
// cuts such units' keys into pieces (history tiles that every row sees, then
// the rest with the causal edge), one CTA each, and a merge kernel combines
// the pieces' partials as split-K decode does.  Not in the pages: a
// scheduling choice for B200.
// ---------------------------------------------------------------------------
namespace pkv {
namespace {

// Per-CTA fixed cost (Q load, pipeline fill, epilogue) in query-tile x
// 64-key tiles, the unit of the cost model.
constexpr int kPlanCtaOverhead = 4;
// A unit is cut only when its CTA would cost more than this many SM shares
// of the batch.  Measured on B200 (kernel TFLOP/s, whole launch, unit cut at
// 1x the share -> uncut): the LLaMA-7B prefill batch (longest unit 1.1x its
// share) 572 -> 661, the GQA batch (1.3x) 570 -> 650; where the longest
// units are 2-5x their share, cutting them paid (uncut -> cut): one sequence
// of 256 new tokens on 4000 cached 216 -> 430, histories of 8192, 100, 50
// and 0 tokens (2.0x) 510 -> 750.
constexpr double kPlanCutShares = 1.5;

struct PlanUnit {
  int seq, tile, nq, cost, hist_tiles;
};

struct PlanPiece {
  int seq, tile, kb, ke, piece, merge, pieces, cost;
};

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_prefill_plan(const int32_t* query_start, const int32_t* context_lens,
                                       int num_seqs, int num_heads, int num_kv_heads,
                                       int head_dim, int num_sms, int32_t* work,
                                       int work_capacity, int* num_items, int32_t* merges,
                                       int merge_capacity, int* num_merges,
                                       size_t* workspace_bytes) {
  using namespace pkv;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      num_sms <= 0 || work_capacity < 0 || merge_capacity < 0 || num_items == nullptr ||
      num_merges == nullptr || (num_seqs > 0 && (query_start == nullptr || context_lens == nullptr)))
    return PKV_ERR_INVALID_ARG;
  if (head_dim != 128) return PKV_ERR_UNSUPPORTED;
  const int group = num_heads / num_kv_heads;
  constexpr int NKEY = 64, M = 128, QT = kPlanRows / M;
  // ---- units and their cost: key tiles summed over the unit's query tiles
  std::vector<PlanUnit> units;
  long long total = 0;
  for (int s = 0; s < num_seqs; ++s) {
    const long long ql = static_cast<long long>(query_start[s + 1]) - query_start[s];
    if (ql <= 0) continue;
    const long long hist = std::max<long long>(0, static_cast<long long>(context_lens[s]) - ql);
    const long long rows = ql * group;
    for (long long t = 0; t * kPlanRows < rows; ++t) {
      long long cost = 0;
      int nq = 0;
      for (int q = 0; q < QT; ++q) {
        const long long r0 = t * kPlanRows + q * M;
        if (r0 >= rows) break;
        const long long last = (std::min(rows, r0 + M) - 1) / group;
        cost += (hist + last + 1 + NKEY - 1) / NKEY;
        ++nq;
      }
      if (cost > 0x3fffffff || t > 0x7fffffff) return PKV_ERR_UNSUPPORTED;
      units.push_back(PlanUnit{s, static_cast<int>(t), nq, static_cast<int>(cost),
                               static_cast<int>(std::min<long long>(hist / NKEY, 0x3fffffff))});
      total += (cost + kPlanCtaOverhead) * num_kv_heads;
    }
  }
  // ---- cut every unit whose CTA would cost more than kPlanCutShares SM
  // shares of the batch into pieces of about one share (at most kMaxPieces,
  // each history piece at least one key tile)
  const double share = static_cast<double>(total) / num_sms;
  std::vector<PlanPiece> pieces;
  int n_merge = 0;
  for (const PlanUnit& u : units) {
    const double c = u.cost + kPlanCtaOverhead;
    int n = 1;
    if (c > kPlanCutShares * share)
      n = std::min<int>(kMaxPieces, static_cast<int>(std::ceil(c / share)));
    // history tiles for the first n - 1 pieces: balance them with the last
    long long k = 0;
    if (n > 1) {
      k = std::min<long long>(u.hist_tiles,
                              static_cast<long long>(static_cast<double>(u.cost) * (n - 1) /
                                                     (static_cast<double>(n) * u.nq)));
      if (k < n - 1) n = static_cast<int>(k) + 1;
      if (n > 1) k = std::min<long long>(k, u.hist_tiles);
    }
    if (n <= 1) {
      pieces.push_back(PlanPiece{u.seq, u.tile, 0, -1, 0, 0, 1, u.cost + kPlanCtaOverhead});
      continue;
    }
    const int merge = n_merge++;
    long long kb = 0;
    for (int i = 0; i < n - 1; ++i) {
      const long long tiles = k / (n - 1) + (i < k % (n - 1) ? 1 : 0);
      pieces.push_back(PlanPiece{u.seq, u.tile, static_cast<int>(kb * NKEY),
                                 static_cast<int>((kb + tiles) * NKEY), i, merge, n,
                                 static_cast<int>(tiles * u.nq + kPlanCtaOverhead)});
      kb += tiles;
    }
    pieces.push_back(PlanPiece{u.seq, u.tile, static_cast<int>(kb * NKEY), -1, n - 1, merge, n,
                               static_cast<int>(u.cost - kb * u.nq + kPlanCtaOverhead)});
  }
  if (pieces.size() > 0x7fffffffULL) return PKV_ERR_UNSUPPORTED;
  // ---- longest first; ties in (sequence, tile, piece) order
  std::stable_sort(pieces.begin(), pieces.end(),
                   [](const PlanPiece& a, const PlanPiece& b) { return a.cost > b.cost; });
  *num_items = static_cast<int>(pieces.size());
  *num_merges = n_merge;
  if (workspace_bytes != nullptr)
    *workspace_bytes = n_merge > 0 ? plan_workspace(n_merge, num_kv_heads).total : 0;
  if (work != nullptr) {
    if (work_capacity < static_cast<long long>(pieces.size())) return PKV_ERR_INVALID_ARG;
    for (size_t i = 0; i < pieces.size(); ++i) {
      const PlanPiece& q = pieces[i];
      int32_t* it = work + i * kPlanItemInts;
      const int32_t v[kPlanItemInts] = {q.seq, q.tile, q.kb, q.ke, q.piece, q.merge, q.pieces, 0};
      std::copy(v, v + kPlanItemInts, it);
    }
  }
  if (merges != nullptr) {
    if (merge_capacity < n_merge) return PKV_ERR_INVALID_ARG;
    for (const PlanPiece& q : pieces)
      if (q.pieces > 1 && q.piece == 0) {
        int32_t* m = merges + 4 * static_cast<size_t>(q.merge);
        m[0] = q.seq;
        m[1] = q.tile;
        m[2] = q.pieces;
        m[3] = 0;
      }
  }
  return PKV_OK;
}

extern "C" pkv_status pkv_paged_attn_prefill_planned(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
    const int32_t* work, int num_items, const int32_t* merges, int num_merges, float scale,
    int num_seqs, int num_tokens, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int max_context_len, int max_query_len, int num_blocks,
    pkv_dtype dtype, void* workspace, size_t workspace_bytes, unsigned* dev_err, void* stream) {
  const pkv::PrefillPlanArgs plan{work, num_items, merges, num_merges, workspace,
                                  workspace_bytes};
  return pkv::prefill_launch(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                             scale, num_seqs, num_tokens, num_heads, num_kv_heads, head_dim,
                             block_size, max_blocks_per_seq, max_context_len, max_query_len,
                             num_blocks, dtype, false, nullptr, nullptr, dev_err, stream, &plan);
}

extern "C" pkv_status pkv_paged_attn_prefill_fp8_planned(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
    const int32_t* work, int num_items, const int32_t* merges, int num_merges, float scale,
    const float* k_scales, const float* v_scales, int num_seqs, int num_tokens, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int max_context_len,
    int max_query_len, int num_blocks, pkv_dtype dtype, void* workspace, size_t workspace_bytes,
    unsigned* dev_err, void* stream) {
  const pkv::PrefillPlanArgs plan{work, num_items, merges, num_merges, workspace,
                                  workspace_bytes};
  return pkv::prefill_launch(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                             scale, num_seqs, num_tokens, num_heads, num_kv_heads, head_dim,
                             block_size, max_blocks_per_seq, max_context_len, max_query_len,
                             num_blocks, dtype, true, k_scales, v_scales, dev_err, stream, &plan);
}
