// host_common.h — host-side helpers shared by the pagedkv entry points.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

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

// 2-D TMA tensor map over a cache viewed as [num_blocks * hkv * bs, d] rows,
// boxes of 16 rows x 64 elements with the 128-byte swizzle (cached per thread).
pkv_status cache_tensor_map(CUtensorMap* out, const void* base, int num_blocks, int hkv, int bs,
                            int d, pkv_dtype dt);

}  // namespace pkv
