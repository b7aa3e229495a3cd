// paged_attn_decode.cu — host side of PagedAttention decode: shape dispatch,
// partition choice, workspace layout, TMA tensor maps and the C entry points.
// The kernels are in paged_attn_kernels.cuh.
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <type_traits>
#include <vector>

#include "host_common.h"
#include "paged_attn_kernels.cuh"

namespace pkv {

// ---------------------------------------------------------------------------
// Host side: shape dispatch, partition choice, workspace layout, launch.
// ---------------------------------------------------------------------------

// E4M3 cache at head_dim 128: every group size runs on the tensor-core
// kernel, with this many stages per warp.  Measured on B200 (decode kernel
// GB/s): with 2 stages (32 KiB of ring, about five CTAs per SM) it reads
// LLaMA-7B shapes at 5667 (G = 1; the CUDA-core kernel: 5087), GQA chat at
// 5135 (G = 4), long contexts at 6203; with 3 stages 5549 / 4964 / 6162;
// with 6 stages 4396 / 3457 / 4207.  Later, with sequences longest first and
// the lazy reference max (LLaMA-7B / GQA chat / long contexts): 4 warps x 2
// stages 6241 / 5585 / 6360; 4 x 3: 6013 / 5473 / 6314; 8 x 2: 5485 / 4528 /
// 5208; 8 x 3: 5582 / 4492 / 5099; 2 x 4: 5905 / 5382 / 6228.
constexpr int kFp8MmaStages = 2;

// Warps per CTA and ring stages per warp for a (head_dim, block_size): about
// 96 KiB of ring per CTA so two CTAs fit on an SM, 2..4 stages per warp.
// An 8-bit cache moves half the bytes per block for about the same
// instructions per token, so per-warp latency, not the ring, limits it: its
// CTAs keep 2 stages per warp (32 KiB of ring) and about six fit on an SM.
// Measured on B200 for LLaMA-7B shapes (D = 128, bs 16, G = 1): 2 stages x 4
// warps 5050 GB/s, 3 x 4: 4832, 3 x 8: 4762, 6 x 4 (two CTAs per SM): 3500.
template <int D, int BS, int KB = 2>
struct LaunchShape {
  static constexpr int W = 4;
  static constexpr int STAGE = 2 * BS * D * KB;
  static constexpr int NS = KB == 1 ? 2 : cmax(2, cmin(4, (96 * 1024) / (W * STAGE)));
};

using KernelFn = void (*)(const DecodeParams);

struct KernelEntry {
  KernelFn fn;
  int threads;
  size_t smem_fixed;  // bytes before the block-table slice
};

template <int D, int BS, int G, class DT, class KV = DT>
KernelEntry make_entry() {
  using LS = LaunchShape<D, BS, static_cast<int>(sizeof(typename KV::T))>;
  using Tr = DecodeTraits<D, BS, G, DT, LS::W, LS::NS, KV>;
  return KernelEntry{paged_decode_kernel<Tr>, Tr::THREADS, Tr::smem_bytes(0)};
}

// Built with PKV_DECODE_GQA_CUDA_CORES=1 (python -m paged_kv_cache_394_b200.build
// --define PKV_DECODE_GQA_CUDA_CORES=1), 16-bit caches run every group size on
// the CUDA-core kernel: the comparison that shows what the tensor cores buy
// for grouped-query decode.  The default build uses them for G >= 2.
#ifndef PKV_DECODE_GQA_CUDA_CORES
#define PKV_DECODE_GQA_CUDA_CORES 0
#endif

template <int D, int BS, class DT>
KernelEntry entry_for_group(int g) {
#if PKV_DECODE_GQA_CUDA_CORES
  switch (g) {
    case 1: return make_entry<D, BS, 1, DT>();
    case 2: return make_entry<D, BS, 2, DT>();
    case 4: return make_entry<D, BS, 4, DT>();
    case 8: return make_entry<D, BS, 8, DT>();
    default: return KernelEntry{nullptr, 0, 0};
  }
#else
  // one query head per kv head: the CUDA-core kernel (G >= 2 uses the tensor cores)
  return g == 1 ? make_entry<D, BS, 1, DT>() : KernelEntry{nullptr, 0, 0};
#endif
}

template <class DT>
KernelEntry entry_for(int d, int bs, int g) {
  if (d == 128 && bs == 16) return entry_for_group<128, 16, DT>(g);
  if (d == 128 && bs == 32) return entry_for_group<128, 32, DT>(g);
  if (d == 64 && bs == 16) return entry_for_group<64, 16, DT>(g);
  if (d == 64 && bs == 32) return entry_for_group<64, 32, DT>(g);
  return KernelEntry{nullptr, 0, 0};
}

KernelEntry decode_entry(int d, int bs, int g, pkv_dtype dt) {
  return dt == PKV_FP16 ? entry_for<Fp16>(d, bs, g) : entry_for<Bf16>(d, bs, g);
}

// E4M3 cache on the CUDA cores at head_dim 64 (the codes widen to fp32 in
// registers; q and out keep their 16-bit type).
template <int D, int BS, class DT>
KernelEntry fp8_entry_for_group(int g) {
  switch (g) {
    case 1: return make_entry<D, BS, 1, DT, Fp8E4M3>();
    case 2: return make_entry<D, BS, 2, DT, Fp8E4M3>();
    case 4: return make_entry<D, BS, 4, DT, Fp8E4M3>();
    case 8: return make_entry<D, BS, 8, DT, Fp8E4M3>();
    default: return KernelEntry{nullptr, 0, 0};
  }
}

template <class DT>
KernelEntry fp8_entry_for(int d, int bs, int g) {
  if (d == 64 && bs == 16) return fp8_entry_for_group<64, 16, DT>(g);
  if (d == 64 && bs == 32) return fp8_entry_for_group<64, 32, DT>(g);
  return KernelEntry{nullptr, 0, 0};
}

KernelEntry fp8_decode_entry(int d, int bs, int g, pkv_dtype dt) {
  return dt == PKV_FP16 ? fp8_entry_for<Fp16>(d, bs, g) : fp8_entry_for<Bf16>(d, bs, g);
}

// ---- tensor-core kernel dispatch -------------------------------------------
using MmaKernelFn = void (*)(const DecodeParams, const CUtensorMap, const CUtensorMap);

struct MmaEntry {
  MmaKernelFn fn;
  int threads;
  size_t smem_fixed;
};

// 4 warps with 2 stages each: 64 KiB of ring per CTA at D = 128 (three CTAs
// per SM; the E4M3 form, 32 KiB).  Measured on B200 with 16-bit caches
// (decode kernel GB/s, 3 stages -> 2): GQA chat 6173 -> 6282, parallel-sampling
// prefix sharing (logical bytes, from L2) 9128 -> 11305.  Per-warp latency,
// not the ring depth, limits these kernels once K/V hit in L2.
template <int D, int KB = 2>
struct MmaShape {
  static constexpr int W = 4;
  static constexpr int STAGE = 2 * (D * KB / 128) * 16 * 128;
  static constexpr int NS = KB == 1 ? kFp8MmaStages : 2;
};

template <int D, int BS, int G, class DT, class KV = DT>
MmaEntry make_mma_entry() {
  using MS = MmaShape<D, static_cast<int>(sizeof(typename KV::T))>;
  using Tr = MmaTraits<D, BS, G, DT, MS::W, MS::NS, KV>;
  return MmaEntry{paged_decode_mma_kernel<Tr>, Tr::THREADS, Tr::smem_bytes(0)};
}

template <int D, int BS, class DT>
MmaEntry mma_for_group(int g) {
  switch (g) {
    case 2: return make_mma_entry<D, BS, 2, DT>();
    case 4: return make_mma_entry<D, BS, 4, DT>();
    case 8: return make_mma_entry<D, BS, 8, DT>();
    default: return MmaEntry{nullptr, 0, 0};
  }
}

template <class DT>
MmaEntry mma_for(int d, int bs, int g) {
  if (d == 128 && bs == 16) return mma_for_group<128, 16, DT>(g);
  if (d == 128 && bs == 32) return mma_for_group<128, 32, DT>(g);
  if (d == 64 && bs == 16) return mma_for_group<64, 16, DT>(g);
  if (d == 64 && bs == 32) return mma_for_group<64, 32, DT>(g);
  return MmaEntry{nullptr, 0, 0};
}

MmaEntry mma_entry(int d, int bs, int g, pkv_dtype dt) {
  return dt == PKV_FP16 ? mma_for<Fp16>(d, bs, g) : mma_for<Bf16>(d, bs, g);
}

// E4M3 cache on the tensor cores: head_dim 128 (a row is one 128-byte box).
template <int BS, class DT>
MmaEntry fp8_mma_for_group(int g) {
  switch (g) {
    case 1: return make_mma_entry<128, BS, 1, DT, Fp8E4M3>();
    case 2: return make_mma_entry<128, BS, 2, DT, Fp8E4M3>();
    case 4: return make_mma_entry<128, BS, 4, DT, Fp8E4M3>();
    case 8: return make_mma_entry<128, BS, 8, DT, Fp8E4M3>();
    default: return MmaEntry{nullptr, 0, 0};
  }
}

MmaEntry fp8_mma_entry(int d, int bs, int g, pkv_dtype dt) {
  if (d != 128) return MmaEntry{nullptr, 0, 0};
  if (bs == 16) return dt == PKV_FP16 ? fp8_mma_for_group<16, Fp16>(g) : fp8_mma_for_group<16, Bf16>(g);
  if (bs == 32) return dt == PKV_FP16 ? fp8_mma_for_group<32, Fp16>(g) : fp8_mma_for_group<32, Bf16>(g);
  return MmaEntry{nullptr, 0, 0};
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Tensor map over a cache viewed as rows of head_dim elements
// ([num_blocks * num_kv_heads * block_size, head_dim]); boxes of 16 rows x 128
// bytes with the 128-byte swizzle, or of 16 whole rows unswizzled for E4M3
// rows of 64 codes.  Encoded maps are cached per thread, keyed by everything
// they depend on.
pkv_status cache_tensor_map(CUtensorMap* out, const void* base, int num_blocks, int hkv, int bs,
                            int d, pkv_dtype dt) {
  struct Slot {
    const void* base;
    int num_blocks, hkv, bs, d, dt;
    CUtensorMap map;
  };
  thread_local Slot slots[4] = {};
  thread_local int next = 0;
  for (const Slot& sl : slots) {
    if (sl.base == base && sl.num_blocks == num_blocks && sl.hkv == hkv && sl.bs == bs &&
        sl.d == d && sl.dt == dt) {
      *out = sl.map;
      return PKV_OK;
    }
  }
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return cuda_status(cudaErrorNotSupported);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d),
                        static_cast<cuuint64_t>(num_blocks) * hkv * bs};
  // 16 rows x 128 bytes: 64 16-bit elements or 128 E4M3 codes; E4M3 rows
  // of 64 codes: 16 whole rows, unswizzled
  const int eb = cache_elem_bytes(dt);
  const bool narrow = d * eb < 128;
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * eb};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(narrow ? d : 128 / eb), 16};
  cuuint32_t estr[2] = {1, 1};
  Slot& sl = slots[next];
  next = (next + 1) % 4;
  const CUresult r =
      enc(&sl.map,
          dt == PKV_FP16   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
          : dt == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                           : CU_TENSOR_MAP_DATA_TYPE_UINT8,
          2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          narrow ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    sl.base = nullptr;
    return cuda_status(cudaErrorInvalidValue);
  }
  sl.base = base;
  sl.num_blocks = num_blocks;
  sl.hkv = hkv;
  sl.bs = bs;
  sl.d = d;
  sl.dt = dt;
  *out = sl.map;
  return PKV_OK;
}

KernelFn reduce_entry(int d, pkv_dtype dt) {
  if (d == 128) return dt == PKV_FP16 ? paged_decode_reduce_kernel<128, Fp16>
                                      : paged_decode_reduce_kernel<128, Bf16>;
  return dt == PKV_FP16 ? paged_decode_reduce_kernel<64, Fp16>
                        : paged_decode_reduce_kernel<64, Bf16>;
}

// The decode kernels' bound on a warp's wait for its own loads, and the
// testing switch that withholds one load (pkv_testing_decode_wait).
std::atomic<uint64_t> g_wait_ns{kWaitTimeoutNs};
std::atomic<int> g_withhold_first_load{0};

constexpr int kMaxPartitionBlocks = 4096;  // block-table slice kept in shared memory
constexpr int kSlots = 2 * 148;            // resident decode CTAs: two per SM, 148 SMs

// Partition size in tokens, at most `cap` when chosen.  With enough
// (sequence, kv head) units to fill the GPU and contexts of at most `cap`
// tokens, one pass (no reduce) is fastest.  Otherwise contexts are cut so
// there are about four CTAs per resident slot, in partitions of 256..cap
// tokens.  Measured on B200 with the sequences taken longest first (decode
// kernel GB/s, partition 512 / 1024 / 2048): GQA chat 5972 / 6310 / 6447, its
// E4M3 form 4632 / 5209 / 5522 (a CTA's start-up is not amortised over short
// partitions).  The cap is the most a partition may hold before its CTA, which
// gets only its share of the bandwidth while the GPU is full, outlasts the
// launch: 4096 tokens for 16-bit caches (GQA chat, contexts up to 4096: 6519
// -> 6769 GB/s kernel, 6468 -> 6742 per step without the reduce) and 2048 for
// E4M3 ones, which are read twice as fast (4096 there gained 5612 -> 5916 on
// back-to-back launches, whose next launch hides the tail, but lost 5475 ->
// 5071 per step, behind the cache write).
constexpr int kAutoPartitionCap16 = 4096;
constexpr int kAutoPartitionCap8 = 2048;
int choose_partition(int num_seqs, int num_kv_heads, int block_size, int max_context_len,
                     int requested, int cap) {
  if (requested > 0) return requested;
  const int whole =
      std::max(block_size, (max_context_len + block_size - 1) / block_size * block_size);
  const long long units = std::max(1LL, static_cast<long long>(num_seqs) * num_kv_heads);
  if (units >= kSlots && max_context_len <= cap) return whole;
  const long long parts = std::max(1LL, (4LL * kSlots + units - 1) / units);
  const long long want = (max_context_len + parts - 1) / parts;
  int part = 256;
  while (part < want && part < cap) part <<= 1;
  return std::min(whole, part);
}

struct WorkspaceLayout {
  size_t out_off, max_off, sum_off, total;
};

WorkspaceLayout workspace_layout(int num_seqs, int num_heads, int head_dim, int max_parts) {
  WorkspaceLayout w{0, 0, 0, 0};
  if (max_parts <= 1) return w;
  const size_t n = static_cast<size_t>(num_seqs) * num_heads * max_parts;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  w.out_off = 0;
  w.max_off = up(n * head_dim * sizeof(float));
  w.sum_off = w.max_off + up(n * sizeof(float));
  w.total = w.sum_off + up(n * sizeof(float));
  return w;
}

// A work item packs its partition and its sequence's partition count into
// 16 bits each.
constexpr int kMaxPlannedParts = 0xffff;

int parts_for(int max_context_len, int block_size, int partition) {
  const int nblk = (max_context_len + block_size - 1) / block_size;
  const int pb = partition / block_size;
  return std::max(1, (nblk + pb - 1) / pb);
}

}  // namespace pkv

extern "C" int pkv_paged_attn_partition_size(int num_seqs, int num_kv_heads, int block_size,
                                             int max_context_len, int requested) {
  if (block_size <= 0) return 0;
  return pkv::choose_partition(num_seqs, num_kv_heads, block_size, max_context_len, requested,
                               pkv::kAutoPartitionCap16);
}

extern "C" int pkv_paged_attn_partition_size_fp8(int num_seqs, int num_kv_heads, int block_size,
                                                 int max_context_len, int requested) {
  if (block_size <= 0) return 0;
  return pkv::choose_partition(num_seqs, num_kv_heads, block_size, max_context_len, requested,
                               pkv::kAutoPartitionCap8);
}

extern "C" size_t pkv_paged_attn_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                                 int head_dim, int block_size,
                                                 int max_context_len, int partition_size) {
  using namespace pkv;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_context_len < 0 || partition_size < 0)
    return 0;
  // the E4M3 rule's partitions are never longer, so its count covers both
  const int part = choose_partition(num_seqs, num_kv_heads, block_size, max_context_len,
                                    partition_size, kAutoPartitionCap8);
  if (part % block_size != 0) return 0;
  const int max_parts = parts_for(max_context_len, block_size, part);
  return workspace_layout(num_seqs, num_heads, head_dim, max_parts).total;
}

namespace pkv {

// Shared body of the 16-bit and the E4M3 decode entry points.  With fp8 the
// caches hold E4M3 codes and every value of kv head h is code * k_scales[h]
// (keys) or code * v_scales[h] (values): the K scale folds into the q
// pre-scale, the V scale into the output numerator.
pkv_status decode_launch(void* out, const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_tables, const int32_t* context_lens, float scale,
                         int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                         int block_size, int max_blocks_per_seq, int max_context_len,
                         int num_blocks, pkv_dtype dtype, int partition_size, void* workspace,
                         size_t workspace_bytes, unsigned* dev_err, void* stream, bool fp8,
                         const float* k_scales, const float* v_scales,
                         const CascadeGroups* cascade = nullptr,
                         const int32_t* seq_order = nullptr, bool after_prefix = false,
                         const int32_t* work = nullptr, int num_work = 0) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 ||
      max_context_len < 0 || num_blocks <= 0 || partition_size < 0 || !dtype_valid(dtype) ||
      num_heads % num_kv_heads != 0 || !isfinite(scale))
    return PKV_ERR_INVALID_ARG;
  if (!head_dim_supported(head_dim) || !block_size_supported(block_size))
    return PKV_ERR_UNSUPPORTED;
  const int group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return PKV_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_context_len) >
      static_cast<long long>(max_blocks_per_seq) * block_size)
    return PKV_ERR_INVALID_ARG;
  if (partition_size % block_size != 0) return PKV_ERR_INVALID_ARG;
  if (num_seqs == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens ||
      (fp8 && (!k_scales || !v_scales)))
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_INVALID_ARG;
  // a work list holds at least one item per sequence, for the partition size
  // it was planned with
  if (work != nullptr && (partition_size == 0 || num_work < num_seqs ||
                          (reinterpret_cast<uintptr_t>(work) & 7u) != 0))
    return PKV_ERR_INVALID_ARG;

  const int part = choose_partition(num_seqs, num_kv_heads, block_size, max_context_len,
                                    partition_size,
                                    fp8 ? kAutoPartitionCap8 : kAutoPartitionCap16);
  const int part_blocks = part / block_size;
  if (part_blocks > kMaxPartitionBlocks) return PKV_ERR_UNSUPPORTED;
  // cascade decode: workspace slot 0 holds the prefix pass's partial and the
  // kernel's partitions start at slot 1
  const int grid_parts = parts_for(max_context_len, block_size, part);
  const int max_parts = grid_parts + (cascade ? 1 : 0);
  const WorkspaceLayout wl = workspace_layout(num_seqs, num_heads, head_dim, max_parts);
  if (wl.total > 0) {
    if (workspace == nullptr || workspace_bytes < wl.total) return PKV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return PKV_ERR_INVALID_ARG;
  }
  if (work != nullptr && grid_parts > kMaxPlannedParts) return PKV_ERR_UNSUPPORTED;
  const long long grid = static_cast<long long>(work ? num_work : num_seqs) * num_kv_heads *
                         (work ? 1 : grid_parts);
  if (grid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;

  // 16-bit: G >= 2 on the tensor cores, G = 1 on the CUDA cores;
  // E4M3: every G on the tensor cores at head_dim 128, on the CUDA cores at 64
  const bool use_mma = fp8 ? head_dim == 128 : group >= 2 && !PKV_DECODE_GQA_CUDA_CORES;
  const KernelEntry ke = use_mma ? KernelEntry{nullptr, 0, 0}
                         : fp8   ? fp8_decode_entry(head_dim, block_size, group, dtype)
                                 : decode_entry(head_dim, block_size, group, dtype);
  const MmaEntry me = !use_mma ? MmaEntry{nullptr, 0, 0}
                      : fp8    ? fp8_mma_entry(head_dim, block_size, group, dtype)
                               : mma_entry(head_dim, block_size, group, dtype);
  if (ke.fn == nullptr && me.fn == nullptr) return PKV_ERR_UNSUPPORTED;
  const size_t smem = (use_mma ? me.smem_fixed : ke.smem_fixed) + static_cast<size_t>(part_blocks) * 4;
  const void* kernel_ptr = use_mma ? reinterpret_cast<const void*>(me.fn)
                                   : reinterpret_cast<const void*>(ke.fn);
  pkv_status st = cuda_status(cudaFuncSetAttribute(
      kernel_ptr, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
  if (st != PKV_OK) return st;
  CUtensorMap kmap, vmap;
  if (use_mma) {
    const pkv_dtype cdt = fp8 ? PKV_FP8_E4M3 : dtype;
    st = cache_tensor_map(&kmap, k_cache, num_blocks, num_kv_heads, block_size, head_dim, cdt);
    if (st != PKV_OK) return st;
    st = cache_tensor_map(&vmap, v_cache, num_blocks, num_kv_heads, block_size, head_dim, cdt);
    if (st != PKV_OK) return st;
  }

  DecodeParams p;
  p.out = out;
  p.q = q;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.qscale = scale * kLog2e;
  p.k_scales = k_scales;
  p.v_scales = v_scales;
  p.num_seqs = num_seqs;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_context_len = max_context_len;
  p.num_blocks = num_blocks;
  p.block_size = block_size;
  p.part_blocks = part_blocks;
  p.max_parts = max_parts;
  p.grid_parts = grid_parts;
  p.group_start = cascade ? cascade->group_start : nullptr;
  p.shared_blocks = cascade ? cascade->shared_blocks : nullptr;
  p.num_groups = cascade ? cascade->num_groups : 0;
  p.max_shared_blocks = cascade ? cascade->max_shared_blocks : 0;
  p.seq_order = cascade ? nullptr : seq_order;  // cascade groups stay together
  p.independent_of_prior = after_prefix ? 1 : 0;
  p.work = reinterpret_cast<const int2*>(work);
  p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  p.withhold_first_load = g_withhold_first_load.load(std::memory_order_relaxed);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.ws_out = wl.total ? reinterpret_cast<float*>(ws + wl.out_off) : nullptr;
  p.ws_max = wl.total ? reinterpret_cast<float*>(ws + wl.max_off) : nullptr;
  p.ws_sum = wl.total ? reinterpret_cast<float*>(ws + wl.sum_off) : nullptr;
  p.err = dev_err;

  // Both kernels are launched with programmatic stream serialization: each
  // may begin its prologue while the previous kernel drains, and waits in
  // griddepcontrol.wait before touching memory that kernel wrote.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(use_mma ? me.threads : ke.threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = as_stream(stream);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  st = use_mma ? cuda_status(cudaLaunchKernelEx(&cfg, me.fn, p, kmap, vmap))
               : cuda_status(cudaLaunchKernelEx(&cfg, ke.fn, p));
  if (st != PKV_OK || max_parts <= 1) return st;

  const long long warps = static_cast<long long>(num_seqs) * num_heads;
  cudaLaunchConfig_t rcfg = cfg;
  rcfg.gridDim = dim3(static_cast<unsigned>((warps + 3) / 4));
  rcfg.blockDim = dim3(128);
  rcfg.dynamicSmemBytes = 0;
  // after a prefix pass the decode kernel did not wait for it, so the merge
  // must wait for both in plain stream order
  if (after_prefix) rcfg.numAttrs = 0;
  return cuda_status(cudaLaunchKernelEx(&rcfg, reduce_entry(head_dim, dtype), p));
}

}  // namespace pkv

extern "C" pkv_status pkv_testing_decode_wait(uint64_t wait_ns, int withhold_first_load) {
  if (wait_ns == 0 || wait_ns > pkv::kWaitTimeoutNs) return PKV_ERR_INVALID_ARG;
  pkv::g_wait_ns.store(wait_ns, std::memory_order_relaxed);
  pkv::g_withhold_first_load.store(withhold_first_load != 0 ? 1 : 0, std::memory_order_relaxed);
  return PKV_OK;
}

extern "C" pkv_status pkv_paged_attn_decode(void* out, const void* q, const void* k_cache,
                                            const void* v_cache, const int32_t* block_tables,
                                            const int32_t* context_lens, float scale,
                                            int num_seqs, int num_heads, int num_kv_heads,
                                            int head_dim, int block_size, int max_blocks_per_seq,
                                            int max_context_len, int num_blocks, pkv_dtype dtype,
                                            int partition_size, void* workspace,
                                            size_t workspace_bytes, unsigned* dev_err,
                                            void* stream) {
  return pkv::decode_launch(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                            num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                            max_blocks_per_seq, max_context_len, num_blocks, dtype,
                            partition_size, workspace, workspace_bytes, dev_err, stream, false,
                            nullptr, nullptr);
}

extern "C" pkv_status pkv_paged_attn_decode_fp8(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, float scale,
    const float* k_scales, const float* v_scales, int num_seqs, int num_heads, int num_kv_heads,
    int head_dim, int block_size,
    int max_blocks_per_seq, int max_context_len, int num_blocks, pkv_dtype dtype,
    int partition_size, void* workspace, size_t workspace_bytes, unsigned* dev_err,
    void* stream) {
  return pkv::decode_launch(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                            num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                            max_blocks_per_seq, max_context_len, num_blocks, dtype,
                            partition_size, workspace, workspace_bytes, dev_err, stream, true,
                            k_scales, v_scales);
}

extern "C" pkv_status pkv_paged_attn_decode_ordered(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* seq_order,
    float scale, int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int max_context_len, int num_blocks, pkv_dtype dtype,
    int partition_size, void* workspace, size_t workspace_bytes, unsigned* dev_err,
    void* stream) {
  if (num_seqs > 0 && seq_order == nullptr) return PKV_ERR_INVALID_ARG;
  return pkv::decode_launch(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                            num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                            max_blocks_per_seq, max_context_len, num_blocks, dtype,
                            partition_size, workspace, workspace_bytes, dev_err, stream, false,
                            nullptr, nullptr, nullptr, seq_order);
}

extern "C" pkv_status pkv_paged_attn_decode_fp8_ordered(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* seq_order,
    float scale, const float* k_scales, const float* v_scales, int num_seqs, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int max_context_len,
    int num_blocks, pkv_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes,
    unsigned* dev_err, void* stream) {
  if (num_seqs > 0 && seq_order == nullptr) return PKV_ERR_INVALID_ARG;
  return pkv::decode_launch(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                            num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                            max_blocks_per_seq, max_context_len, num_blocks, dtype,
                            partition_size, workspace, workspace_bytes, dev_err, stream, true,
                            k_scales, v_scales, nullptr, seq_order);
}

// Longest-first order of the sequences, in buckets of kOrderBucket tokens
// (index order within a bucket): a counting sort over the bucket numbers.
extern "C" pkv_status pkv_decode_order(const int32_t* context_lens, int num_seqs,
                                       int32_t* order) {
  constexpr int kOrderBucket = 256;
  constexpr int kOrderMaxBucket = 4095;  // contexts of 1 Mi tokens or more share one bucket
  if (num_seqs < 0 || (num_seqs > 0 && (context_lens == nullptr || order == nullptr)))
    return PKV_ERR_INVALID_ARG;
  auto bucket = [&](int i) {
    return std::min(std::max(context_lens[i], 0) / kOrderBucket, kOrderMaxBucket);
  };
  int top = 0;
  for (int i = 0; i < num_seqs; ++i) top = std::max(top, bucket(i));
  // position k = top - bucket: the longest sequences first
  std::vector<int> start(static_cast<size_t>(top) + 2, 0);
  for (int i = 0; i < num_seqs; ++i) ++start[top - bucket(i) + 1];
  for (int k = 1; k <= top + 1; ++k) start[k] += start[k - 1];
  for (int i = 0; i < num_seqs; ++i) order[start[top - bucket(i)]++] = i;
  return PKV_OK;
}

// Work list of (sequence, partition) items, longest first in buckets of
// kOrderBucket tokens of the item's own length (index order within a
// bucket): a counting sort, as for pkv_decode_order.
extern "C" pkv_status pkv_decode_plan(const int32_t* context_lens, int num_seqs, int block_size,
                                      int partition_size, int32_t* work, int capacity,
                                      int* num_items) {
  constexpr int kOrderBucket = 256;
  if (num_seqs < 0 || block_size <= 0 || partition_size <= 0 ||
      partition_size % block_size != 0 || capacity < 0 || num_items == nullptr ||
      (num_seqs > 0 && context_lens == nullptr))
    return PKV_ERR_INVALID_ARG;
  const int pb = partition_size / block_size;
  auto parts = [&](int i) {
    const long long nblk = (std::max(context_lens[i], 0) + 0LL + block_size - 1) / block_size;
    return std::max(1LL, (nblk + pb - 1) / pb);
  };
  long long n = 0;
  for (int i = 0; i < num_seqs; ++i) {
    const long long np = parts(i);
    if (np > pkv::kMaxPlannedParts) return PKV_ERR_UNSUPPORTED;
    n += np;
  }
  if (n > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;
  *num_items = static_cast<int>(n);
  if (work == nullptr) return PKV_OK;  // size query
  if (capacity < n) return PKV_ERR_INVALID_ARG;
  // tokens of item (i, j): the partition's share of the context
  auto bucket = [&](int i, int j) {
    const long long len = std::max(context_lens[i], 0);
    const long long rest = len - static_cast<long long>(j) * partition_size;
    return static_cast<int>(std::min<long long>(rest, partition_size) / kOrderBucket);
  };
  const int top = partition_size / kOrderBucket;
  std::vector<long long> start(static_cast<size_t>(top) + 2, 0);
  for (int i = 0; i < num_seqs; ++i)
    for (int j = 0, np = static_cast<int>(parts(i)); j < np; ++j) ++start[top - bucket(i, j) + 1];
  for (int k = 1; k <= top + 1; ++k) start[k] += start[k - 1];
  for (int i = 0; i < num_seqs; ++i) {
    const int np = static_cast<int>(parts(i));
    for (int j = 0; j < np; ++j) {
      const long long at = start[top - bucket(i, j)]++;
      work[2 * at] = i;
      work[2 * at + 1] = j | (np << 16);
    }
  }
  return PKV_OK;
}

extern "C" pkv_status pkv_paged_attn_decode_planned(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* work, int num_items,
    float scale, int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int max_context_len, int num_blocks, pkv_dtype dtype,
    int partition_size, void* workspace, size_t workspace_bytes, unsigned* dev_err,
    void* stream) {
  if (num_seqs > 0 && work == nullptr) return PKV_ERR_INVALID_ARG;
  return pkv::decode_launch(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                            num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                            max_blocks_per_seq, max_context_len, num_blocks, dtype,
                            partition_size, workspace, workspace_bytes, dev_err, stream, false,
                            nullptr, nullptr, nullptr, nullptr, false, work, num_items);
}

extern "C" pkv_status pkv_paged_attn_decode_fp8_planned(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* work, int num_items,
    float scale, const float* k_scales, const float* v_scales, int num_seqs, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int max_context_len,
    int num_blocks, pkv_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes,
    unsigned* dev_err, void* stream) {
  if (num_seqs > 0 && work == nullptr) return PKV_ERR_INVALID_ARG;
  return pkv::decode_launch(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                            num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                            max_blocks_per_seq, max_context_len, num_blocks, dtype,
                            partition_size, workspace, workspace_bytes, dev_err, stream, true,
                            k_scales, v_scales, nullptr, nullptr, false, work, num_items);
}

// ---------------------------------------------------------------------------
// Cascade decode for sequences that share a cached prefix.
//
// Parallel samples of one prompt share the prompt's blocks through their
// block tables ([cortexgrid] FAQ on parallel sampling; [csdn] "分页式KV缓存":
// common prompts point at the same pages).  Plain decode reads those blocks
// once per sample; the samples of a prompt run at about the same time, so the
// repeats come from L2, and L2 bandwidth then bounds the step.  Here the
// shared blocks are read once per group: a chunked-prefill kernel in prefix
// mode (tcgen05 at head_dim 128, mma.sync at 64) attends every member's query
// rows to them together (slot 0 of the split-K workspace), the decode kernel
// covers each member's own blocks (slots 1..), and the reduce merges the
// partials.  The result is that of plain decode, over 16-bit or E4M3 caches.
// ---------------------------------------------------------------------------
extern "C" size_t pkv_paged_attn_cascade_workspace_bytes(int num_seqs, int num_heads,
                                                         int num_kv_heads, int head_dim,
                                                         int block_size, int max_context_len,
                                                         int partition_size) {
  using namespace pkv;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_context_len < 0 || partition_size < 0)
    return 0;
  const int part = choose_partition(num_seqs, num_kv_heads, block_size, max_context_len,
                                    partition_size, kAutoPartitionCap8);
  if (part % block_size != 0) return 0;
  return workspace_layout(num_seqs, num_heads, head_dim,
                          1 + parts_for(max_context_len, block_size, part))
      .total;
}

namespace pkv {
namespace {

// Shared body of the 16-bit and the E4M3 cascade entry points.
pkv_status cascade_launch(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens,
                          const int32_t* group_start, const int32_t* shared_blocks, float scale,
                          int num_seqs, int num_groups, int max_group_size, int max_shared_blocks,
                          int num_heads, int num_kv_heads, int head_dim, int block_size,
                          int max_blocks_per_seq, int max_context_len, int num_blocks,
                          pkv_dtype dtype, int partition_size, void* workspace,
                          size_t workspace_bytes, unsigned* dev_err, void* stream, bool fp8,
                          const float* k_scales, const float* v_scales) {
  if (num_seqs < 0 || num_groups < 0 || max_group_size < 0 || max_shared_blocks < 0 ||
      num_kv_heads <= 0 || block_size <= 0 ||
      static_cast<long long>(max_shared_blocks) * block_size > max_context_len ||
      (num_seqs > 0 && (num_groups == 0 || max_group_size == 0)))
    return PKV_ERR_INVALID_ARG;
  if (!head_dim_supported(head_dim)) return PKV_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PKV_OK;
  if (!group_start || !shared_blocks || !workspace || (fp8 && (!k_scales || !v_scales)))
    return PKV_ERR_INVALID_ARG;
  const CascadeGroups groups{group_start, shared_blocks, num_groups, max_group_size,
                             max_shared_blocks};
  // validate everything (and the workspace) before the first launch
  const size_t need = pkv_paged_attn_cascade_workspace_bytes(
      num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len, partition_size);
  if (workspace_bytes < need || !aligned16(workspace)) return PKV_ERR_WORKSPACE;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !dtype_valid(dtype) ||
      num_heads <= 0 || num_heads % num_kv_heads != 0 || !isfinite(scale) ||
      partition_size < 0 || partition_size % block_size != 0 || max_blocks_per_seq <= 0 ||
      num_blocks <= 0 ||
      static_cast<long long>(max_context_len) >
          static_cast<long long>(max_blocks_per_seq) * block_size ||
      !aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_INVALID_ARG;
  const int group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return PKV_ERR_UNSUPPORTED;
  if (!block_size_supported(block_size)) return PKV_ERR_UNSUPPORTED;
  const int part = choose_partition(num_seqs, num_kv_heads, block_size, max_context_len,
                                    partition_size,
                                    fp8 ? kAutoPartitionCap8 : kAutoPartitionCap16);
  if (part / block_size > kMaxPartitionBlocks) return PKV_ERR_UNSUPPORTED;
  const int max_parts = 1 + parts_for(max_context_len, block_size, part);
  if (static_cast<long long>(num_seqs) * num_kv_heads * max_parts > 0x7fffffffLL)
    return PKV_ERR_UNSUPPORTED;
  const WorkspaceLayout wl = workspace_layout(num_seqs, num_heads, head_dim, max_parts);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  // The prefix pass goes first; each of its CTAs waits for the cache writes
  // before it lets the next grid start, so the suffix decode, which reads
  // nothing the prefix pass writes, starts without waiting for it and fills
  // the SMs the prefix pass frees; the merge waits for both in stream order.
  // Measured on B200 (parallel-sampling batch, one cascade decode): 0.192 ms
  // with the suffix waiting for the prefix pass, 0.178 ms without.
  if (max_shared_blocks > 0) {
    const pkv_status st = launch_cascade_prefix(
        q, k_cache, v_cache, block_tables, context_lens, groups, scale, num_seqs, num_heads,
        num_kv_heads, head_dim, block_size, max_blocks_per_seq, max_context_len, num_blocks,
        dtype, fp8, k_scales, v_scales, reinterpret_cast<float*>(ws + wl.out_off),
        reinterpret_cast<float*>(ws + wl.max_off), reinterpret_cast<float*>(ws + wl.sum_off),
        max_parts, dev_err, as_stream(stream));
    if (st != PKV_OK) return st;
  }
  return decode_launch(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_seqs,
                       num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                       max_context_len, num_blocks, dtype, partition_size, workspace,
                       workspace_bytes, dev_err, stream, fp8, k_scales, v_scales, &groups,
                       nullptr, max_shared_blocks > 0);
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_paged_attn_decode_cascade(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* group_start,
    const int32_t* shared_blocks, float scale, int num_seqs, int num_groups, int max_group_size,
    int max_shared_blocks, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int max_context_len, int num_blocks, pkv_dtype dtype,
    int partition_size, void* workspace, size_t workspace_bytes, unsigned* dev_err,
    void* stream) {
  return pkv::cascade_launch(out, q, k_cache, v_cache, block_tables, context_lens, group_start,
                             shared_blocks, scale, num_seqs, num_groups, max_group_size,
                             max_shared_blocks, num_heads, num_kv_heads, head_dim, block_size,
                             max_blocks_per_seq, max_context_len, num_blocks, dtype,
                             partition_size, workspace, workspace_bytes, dev_err, stream, false,
                             nullptr, nullptr);
}

extern "C" pkv_status pkv_paged_attn_decode_cascade_fp8(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* group_start,
    const int32_t* shared_blocks, float scale, const float* k_scales, const float* v_scales,
    int num_seqs, int num_groups, int max_group_size, int max_shared_blocks, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int max_context_len,
    int num_blocks, pkv_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes,
    unsigned* dev_err, void* stream) {
  return pkv::cascade_launch(out, q, k_cache, v_cache, block_tables, context_lens, group_start,
                             shared_blocks, scale, num_seqs, num_groups, max_group_size,
                             max_shared_blocks, num_heads, num_kv_heads, head_dim, block_size,
                             max_blocks_per_seq, max_context_len, num_blocks, dtype,
                             partition_size, workspace, workspace_bytes, dev_err, stream, true,
                             k_scales, v_scales);
}

// ---------------------------------------------------------------------------
// Decode whose split-K scratch lives in a fixed device array.
//
// For callers that cannot allocate device memory: a plugin loaded into a host
// application that owns every device allocation and hands out none, or a
// serving loop that must not call cudaMalloc once it is running, because
// cudaMalloc can synchronise the device and stall every stream in flight.
// The caller still passes all inputs and outputs; only the scratch is fixed.
// ---------------------------------------------------------------------------

// The split-K scratch of pkv_paged_attn_decode_static_ws.  Every GPU on which
// this library is loaded keeps these PKV_STATIC_WORKSPACE_BYTES (once per
// CUDA context that loads it) until the process exits.  In host code this
// name is only a stand-in for the device symbol, never a device address: the
// kernels get the address that cudaGetSymbolAddress returns in the current
// context.
static __device__ __align__(256) unsigned char pkv_static_workspace[PKV_STATIC_WORKSPACE_BYTES];


namespace pkv {
namespace {
// The array exists once per CUDA context: every context that loads the
// library (the device's primary context, one rebuilt after cudaDeviceReset,
// or a context the application made current through the driver API) holds
// its own copy at its own address.  So the address is cached per context,
// keyed by the driver's context id, which is unique for the life of the
// process (a context rebuilt after a reset gets a new one).
using CtxGetCurrentFn = CUresult(CUDAAPI*)(CUcontext*);
using CtxGetIdFn = CUresult(CUDAAPI*)(CUcontext, unsigned long long*);

struct ContextFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

// cuCtxGetCurrent and cuCtxGetId through the runtime's driver entry point
// (no -lcuda).
const ContextFns& context_fns() {
  static ContextFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &ptr, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<CtxGetCurrentFn>(ptr);
    ptr = nullptr;
    q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<CtxGetIdFn>(ptr);
  });
  return f;
}

struct StaticWsEntry {
  unsigned long long ctx_id;
  void* addr;
};
constexpr int kStaticWsEntries = 64;
StaticWsEntry g_static_ws[kStaticWsEntries] = {};
int g_static_ws_next = 0;
std::mutex g_static_ws_mutex;

// Device address of pkv_static_workspace in the context current on this
// thread, looked up (cudaGetSymbolAddress) the first time a context is seen
// and cached under its id.
pkv_status static_workspace_address(void** addr) {
  const ContextFns& f = context_fns();
  if (f.get_current == nullptr || f.get_id == nullptr) return cuda_status(cudaErrorNotSupported);
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS) return cuda_status(cudaErrorDeviceUninitialized);
  if (ctx == nullptr) {
    // The runtime has not made a context current on this thread yet: the
    // lookup initialises the current device's primary context.
    void* p = nullptr;
    const pkv_status st = cuda_status(cudaGetSymbolAddress(&p, pkv_static_workspace));
    if (st != PKV_OK) return st;
    if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
      return cuda_status(cudaErrorDeviceUninitialized);
  }
  unsigned long long id = 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return cuda_status(cudaErrorDeviceUninitialized);
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  for (const StaticWsEntry& e : g_static_ws) {
    if (e.addr != nullptr && e.ctx_id == id) {
      *addr = e.addr;
      return PKV_OK;
    }
  }
  void* p = nullptr;
  const pkv_status st = cuda_status(cudaGetSymbolAddress(&p, pkv_static_workspace));
  if (st != PKV_OK) return st;
  g_static_ws[g_static_ws_next] = StaticWsEntry{id, p};
  g_static_ws_next = (g_static_ws_next + 1) % kStaticWsEntries;
  *addr = p;
  return PKV_OK;
}
}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_paged_attn_decode_static_ws(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, float scale, int num_seqs,
    int num_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
    int max_context_len, int num_blocks, pkv_dtype dtype, int partition_size, unsigned* dev_err,
    void* stream) {
  using namespace pkv;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || block_size <= 0 ||
      max_context_len < 0 || partition_size < 0)
    return PKV_ERR_INVALID_ARG;
  const size_t need = pkv_paged_attn_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim,
                                                     block_size, max_context_len, partition_size);
  if (need > PKV_STATIC_WORKSPACE_BYTES) return PKV_ERR_WORKSPACE;
  void* ws = nullptr;
  const pkv_status st = static_workspace_address(&ws);
  if (st != PKV_OK) return st;
  return pkv_paged_attn_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                               num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                               max_blocks_per_seq, max_context_len, num_blocks, dtype,
                               partition_size, ws, PKV_STATIC_WORKSPACE_BYTES, dev_err, stream);
}
