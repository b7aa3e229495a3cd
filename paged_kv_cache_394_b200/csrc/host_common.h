// host_common.h — host-side helpers shared by the pagedkv entry points.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "pagedkv.h"

namespace pkv {

// Records `e` as the calling thread's last CUDA error and maps it to a status.
pkv_status cuda_status(cudaError_t e);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool head_dim_supported(int d) { return d == 64 || d == 128; }
inline bool block_size_supported(int bs) { return bs == 16 || bs == 32; }
inline bool dtype_valid(int dt) { return dt == PKV_FP16 || dt == PKV_BF16; }
// Element types a cache may hold: the 16-bit ones, or E4M3 codes.
inline bool cache_dtype_valid(int dt) { return dtype_valid(dt) || dt == PKV_FP8_E4M3; }
inline int cache_elem_bytes(int dt) { return dt == PKV_FP8_E4M3 ? 1 : 2; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Launches `kernel` with programmatic stream serialisation: its CTAs may be
// scheduled while the previous kernel in the stream drains, so the kernel
// must call griddepcontrol.wait before it touches memory that kernel uses.
template <class... KArgs, class... Args>
cudaError_t launch_after_previous(void (*kernel)(KArgs...), dim3 grid, dim3 block, void* stream,
                                  Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = as_stream(stream);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// 2-D TMA tensor map over a cache viewed as [num_blocks * hkv * bs, d] rows
// (cached per thread): boxes of 16 rows x 128 bytes (64 16-bit elements or 128
// E4M3 codes) with the 128-byte swizzle; E4M3 rows of 64 codes come as boxes of
// 16 whole rows, unswizzled.
pkv_status cache_tensor_map(CUtensorMap* out, const void* base, int num_blocks, int hkv, int bs,
                            int d, pkv_dtype dt);

// 3-D TMA tensor map over q [T, H, 128] (16-bit): boxes of (128/group tokens)
// x (group heads) x 64 dims, i.e. a 128-row query tile ordered (token, head),
// with the 128-byte swizzle.
pkv_status q_tensor_map(CUtensorMap* out, const void* q, int num_tokens, int num_heads, int group,
                        pkv_dtype dt);

// Groups of cascade decode (device arrays): group g is sequences
// group_start[g] .. group_start[g+1]-1, sharing their first shared_blocks[g]
// blocks.
struct CascadeGroups {
  const int32_t* group_start;
  const int32_t* shared_blocks;
  int num_groups;
  int max_group_size;
  int max_shared_blocks;
};

// The shared-prefix pass of cascade decode: writes each member's prefix
// partial (m, l, unnormalised o) into slot 0 of its rows of the split-K
// workspace (max_parts slots per (sequence, head)).  head_dim 128 runs the
// tcgen05 kernel, 64 the mma.sync kernel; fp8: the caches hold E4M3 codes with
// per-kv-head scales k_scales / v_scales (the V scale goes into o).
pkv_status launch_cascade_prefix(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* block_tables, const int32_t* context_lens,
                                 const CascadeGroups& groups, float scale, int num_seqs,
                                 int num_heads, int num_kv_heads, int head_dim, int block_size,
                                 int max_blocks_per_seq, int max_context_len, int num_blocks,
                                 pkv_dtype dtype, bool fp8, const float* k_scales,
                                 const float* v_scales, float* ws_out, float* ws_max,
                                 float* ws_sum, int max_parts, unsigned* dev_err,
                                 cudaStream_t stream);

}  // namespace pkv
