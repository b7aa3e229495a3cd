// decode_step.cu — one decode step driven from host buffers.
//
// Copies the step's inputs (q, the new tokens' K/V and slots, the copy-on-
// write pairs, block tables, context lengths) from host memory into a
// caller-provided device staging buffer, runs copy_blocks, reshape_and_cache
// and paged_attn_decode on the device-resident caches, and copies the output
// back — all enqueued on one stream.  One cudaMemcpyAsync per buffer.
#include <cuda_runtime.h>

#include "host_common.h"

namespace pkv {
namespace {

struct StagingLayout {
  size_t q, key, value, slots, pairs, tables, lens, out, total;
};

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

StagingLayout staging_layout(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                             int max_blocks_per_seq, int num_new_tokens, int num_pairs) {
  StagingLayout l{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += up256(bytes);
    return at;
  };
  const size_t qo = static_cast<size_t>(num_seqs) * num_heads * head_dim * 2;
  const size_t kv = static_cast<size_t>(num_new_tokens) * num_kv_heads * head_dim * 2;
  l.q = take(qo);
  l.key = take(kv);
  l.value = take(kv);
  l.slots = take(static_cast<size_t>(num_new_tokens) * 8);
  l.pairs = take(static_cast<size_t>(num_pairs) * 16);
  l.tables = take(static_cast<size_t>(num_seqs) * max_blocks_per_seq * 4);
  l.lens = take(static_cast<size_t>(num_seqs) * 4);
  l.out = take(qo);
  l.total = off;
  return l;
}

}  // namespace
}  // namespace pkv

extern "C" size_t pkv_decode_step_staging_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                                int head_dim, int max_blocks_per_seq,
                                                int num_new_tokens, int num_pairs) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_blocks_per_seq <= 0 || num_new_tokens < 0 || num_pairs < 0)
    return 0;
  return pkv::staging_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                             num_new_tokens, num_pairs)
      .total;
}

extern "C" pkv_status pkv_decode_step_host(
    void* out_host, const void* q_host, const void* key_host, const void* value_host,
    const int64_t* slot_mapping_host, int num_new_tokens, const int64_t* block_mapping_host,
    int num_pairs, const int32_t* block_tables_host, const int32_t* context_lens_host,
    void* k_cache, void* v_cache, float scale, int num_seqs, int num_heads, int num_kv_heads,
    int head_dim, int block_size, int max_blocks_per_seq, int max_context_len, int num_blocks,
    pkv_dtype dtype, int partition_size, void* staging, size_t staging_bytes, void* workspace,
    size_t workspace_bytes, unsigned* dev_err, void* stream) {
  using namespace pkv;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 ||
      num_new_tokens < 0 || num_pairs < 0 || !dtype_valid(dtype))
    return PKV_ERR_INVALID_ARG;
  if (!head_dim_supported(head_dim) || !block_size_supported(block_size))
    return PKV_ERR_UNSUPPORTED;
  if (num_seqs > 0 && (!out_host || !q_host || !block_tables_host || !context_lens_host))
    return PKV_ERR_INVALID_ARG;
  if (num_new_tokens > 0 && (!key_host || !value_host || !slot_mapping_host))
    return PKV_ERR_INVALID_ARG;
  if (num_pairs > 0 && !block_mapping_host) return PKV_ERR_INVALID_ARG;
  if (!staging || !aligned16(staging)) return PKV_ERR_INVALID_ARG;
  const StagingLayout l = staging_layout(num_seqs, num_heads, num_kv_heads, head_dim,
                                         max_blocks_per_seq, num_new_tokens, num_pairs);
  if (staging_bytes < l.total) return PKV_ERR_WORKSPACE;

  cudaStream_t s = as_stream(stream);
  unsigned char* st = static_cast<unsigned char*>(staging);
  const size_t qo = static_cast<size_t>(num_seqs) * num_heads * head_dim * 2;
  const size_t kv = static_cast<size_t>(num_new_tokens) * num_kv_heads * head_dim * 2;
  struct Copy {
    size_t dst;
    const void* src;
    size_t bytes;
  } copies[] = {
      {l.q, q_host, qo},
      {l.key, key_host, kv},
      {l.value, value_host, kv},
      {l.slots, slot_mapping_host, static_cast<size_t>(num_new_tokens) * 8},
      {l.pairs, block_mapping_host, static_cast<size_t>(num_pairs) * 16},
      {l.tables, block_tables_host, static_cast<size_t>(num_seqs) * max_blocks_per_seq * 4},
      {l.lens, context_lens_host, static_cast<size_t>(num_seqs) * 4},
  };
  for (const Copy& c : copies) {
    if (c.bytes == 0) continue;
    pkv_status r =
        cuda_status(cudaMemcpyAsync(st + c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, s));
    if (r != PKV_OK) return r;
  }
  pkv_status r = pkv_copy_blocks(k_cache, v_cache, reinterpret_cast<const int64_t*>(st + l.pairs),
                                 num_pairs, num_kv_heads, head_dim, block_size, num_blocks, dtype,
                                 dev_err, stream);
  if (r != PKV_OK) return r;
  r = pkv_reshape_and_cache(st + l.key, st + l.value, k_cache, v_cache,
                            reinterpret_cast<const int64_t*>(st + l.slots), num_new_tokens,
                            num_kv_heads, head_dim, block_size, num_blocks, dtype, dev_err, stream);
  if (r != PKV_OK) return r;
  r = pkv_paged_attn_decode(st + l.out, st + l.q, k_cache, v_cache,
                            reinterpret_cast<const int32_t*>(st + l.tables),
                            reinterpret_cast<const int32_t*>(st + l.lens), scale, num_seqs,
                            num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                            max_context_len, num_blocks, dtype, partition_size, workspace,
                            workspace_bytes, dev_err, stream);
  if (r != PKV_OK) return r;
  if (qo == 0) return PKV_OK;
  return cuda_status(cudaMemcpyAsync(out_host, st + l.out, qo, cudaMemcpyDeviceToHost, s));
}
