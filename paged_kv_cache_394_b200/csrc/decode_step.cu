// decode_step.cu — one decode step driven from host buffers.
//
// Copies the step's inputs (q, the new tokens' K/V and slots, the copy-on-
// write pairs, block tables, context lengths) from host memory into a
// caller-provided device staging buffer, runs copy_blocks, reshape_and_cache
// and paged_attn_decode on the device-resident caches, and copies the output
// back — all enqueued on one stream.  One cudaMemcpyAsync per buffer.
//
// The pipeline (pkv_decode_pipeline_*) runs consecutive steps the same way
// but overlapped across three streams: step i+1's inputs cross the host link
// on an upload stream while step i computes on the caller's stream, and step
// i's output returns on a download stream while step i+1 computes.  Two
// staging areas alternate between steps; events order each area's reuse.
#include <cuda_runtime.h>

#include <algorithm>
#include <new>

#include "host_common.h"

namespace pkv {
namespace step {

struct StagingLayout {
  size_t q, key, value, slots, pairs, tables, lens, work, out, total;
};

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t work_items(int num_seqs, int max_blocks_per_seq) {
  return static_cast<size_t>(num_seqs) * max_blocks_per_seq;
}

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
  // pipeline: the step's work list (pkv_decode_plan), at most one item per
  // block of each sequence (an empty sequence has one item and no block)
  l.work = take(work_items(num_seqs, max_blocks_per_seq) * 8);
  l.out = take(qo);
  l.total = off;
  return l;
}

}  // namespace step
}  // namespace pkv

extern "C" size_t pkv_decode_step_staging_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                                int head_dim, int max_blocks_per_seq,
                                                int num_new_tokens, int num_pairs) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_blocks_per_seq <= 0 || num_new_tokens < 0 || num_pairs < 0)
    return 0;
  return pkv::step::staging_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq,
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
  using namespace pkv::step;
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

// ---------------------------------------------------------------------------
// Pipelined host-buffer steps.
// ---------------------------------------------------------------------------
struct pkv_decode_pipeline {
  int num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq;
  int max_new_tokens, max_pairs;
  pkv_dtype dtype;
  unsigned char* staging[2];  // two areas of `layout.total` bytes
  pkv::step::StagingLayout layout;  // offsets inside one area, sized for the maxima
  int32_t* work_host;         // pinned [2][work_items][2]: each area's work list
  cudaStream_t compute, up, down;
  cudaEvent_t ev_up[2], ev_comp[2], ev_down[2];
  long long steps;
};

namespace pkv {
namespace step {
size_t pipeline_area_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                           int max_blocks_per_seq, int max_new_tokens, int max_pairs) {
  return up256(staging_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                              max_new_tokens, max_pairs)
                   .total);
}

void pipeline_release(pkv_decode_pipeline* pl) {
  if (pl->up) cudaStreamSynchronize(pl->up);
  if (pl->down) cudaStreamSynchronize(pl->down);
  for (int b = 0; b < 2; ++b) {
    if (pl->ev_up[b]) cudaEventDestroy(pl->ev_up[b]);
    if (pl->ev_comp[b]) cudaEventDestroy(pl->ev_comp[b]);
    if (pl->ev_down[b]) cudaEventDestroy(pl->ev_down[b]);
  }
  if (pl->up) cudaStreamDestroy(pl->up);
  if (pl->down) cudaStreamDestroy(pl->down);
  if (pl->work_host) cudaFreeHost(pl->work_host);
}
}  // namespace step
}  // namespace pkv

extern "C" size_t pkv_decode_pipeline_staging_bytes(int num_seqs, int num_heads,
                                                    int num_kv_heads, int head_dim,
                                                    int max_blocks_per_seq, int max_new_tokens,
                                                    int max_pairs) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_blocks_per_seq <= 0 || max_new_tokens < 0 || max_pairs < 0)
    return 0;
  return 2 * pkv::step::pipeline_area_bytes(num_seqs, num_heads, num_kv_heads, head_dim,
                                      max_blocks_per_seq, max_new_tokens, max_pairs);
}

extern "C" pkv_status pkv_decode_pipeline_create(
    pkv_decode_pipeline** out, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
    int block_size, int max_blocks_per_seq, int max_new_tokens, int max_pairs, pkv_dtype dtype,
    void* staging, size_t staging_bytes, void* stream) {
  using namespace pkv;
  using namespace pkv::step;
  if (out == nullptr) return PKV_ERR_INVALID_ARG;
  *out = nullptr;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 ||
      max_new_tokens < 0 || max_pairs < 0 || !dtype_valid(dtype) ||
      num_heads % num_kv_heads != 0)
    return PKV_ERR_INVALID_ARG;
  if (!head_dim_supported(head_dim) || !block_size_supported(block_size))
    return PKV_ERR_UNSUPPORTED;
  if (staging == nullptr || !aligned16(staging)) return PKV_ERR_INVALID_ARG;
  const size_t area = pipeline_area_bytes(num_seqs, num_heads, num_kv_heads, head_dim,
                                          max_blocks_per_seq, max_new_tokens, max_pairs);
  if (staging_bytes < 2 * area) return PKV_ERR_WORKSPACE;
  pkv_decode_pipeline* pl = new (std::nothrow) pkv_decode_pipeline();
  if (pl == nullptr) return PKV_ERR_INVALID_ARG;
  pl->num_seqs = num_seqs;
  pl->num_heads = num_heads;
  pl->num_kv_heads = num_kv_heads;
  pl->head_dim = head_dim;
  pl->block_size = block_size;
  pl->max_blocks_per_seq = max_blocks_per_seq;
  pl->max_new_tokens = max_new_tokens;
  pl->max_pairs = max_pairs;
  pl->dtype = dtype;
  pl->staging[0] = static_cast<unsigned char*>(staging);
  pl->staging[1] = pl->staging[0] + area;
  pl->layout = staging_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                              max_new_tokens, max_pairs);
  pl->compute = as_stream(stream);
  // pinned host memory for the per-step work list (no device memory is allocated)
  pkv_status st = cuda_status(cudaHostAlloc(
      reinterpret_cast<void**>(&pl->work_host),
      2 * std::max<size_t>(work_items(num_seqs, max_blocks_per_seq), 1) * 8,
      cudaHostAllocDefault));
  if (st == PKV_OK) st = cuda_status(cudaStreamCreateWithFlags(&pl->up, cudaStreamNonBlocking));
  if (st == PKV_OK) st = cuda_status(cudaStreamCreateWithFlags(&pl->down, cudaStreamNonBlocking));
  for (int b = 0; b < 2 && st == PKV_OK; ++b) {
    st = cuda_status(cudaEventCreateWithFlags(&pl->ev_up[b], cudaEventDisableTiming));
    if (st == PKV_OK)
      st = cuda_status(cudaEventCreateWithFlags(&pl->ev_comp[b], cudaEventDisableTiming));
    if (st == PKV_OK)
      st = cuda_status(cudaEventCreateWithFlags(&pl->ev_down[b], cudaEventDisableTiming));
  }
  if (st != PKV_OK) {
    pipeline_release(pl);
    delete pl;
    return st;
  }
  *out = pl;
  return PKV_OK;
}

extern "C" pkv_status pkv_decode_pipeline_step(
    pkv_decode_pipeline* pl, void* out_host, const void* q_host, const void* key_host,
    const void* value_host, const int64_t* slot_mapping_host, int num_new_tokens,
    const int64_t* block_mapping_host, int num_pairs, const int32_t* block_tables_host,
    const int32_t* context_lens_host, void* k_cache, void* v_cache, float scale,
    int max_context_len, int num_blocks, int partition_size, void* workspace,
    size_t workspace_bytes, unsigned* dev_err) {
  using namespace pkv;
  using namespace pkv::step;
  if (pl == nullptr || num_new_tokens < 0 || num_pairs < 0 ||
      num_new_tokens > pl->max_new_tokens || num_pairs > pl->max_pairs)
    return PKV_ERR_INVALID_ARG;
  const int S = pl->num_seqs, H = pl->num_heads, HKV = pl->num_kv_heads, D = pl->head_dim;
  if (S > 0 && (!out_host || !q_host || !block_tables_host || !context_lens_host))
    return PKV_ERR_INVALID_ARG;
  if (num_new_tokens > 0 && (!key_host || !value_host || !slot_mapping_host))
    return PKV_ERR_INVALID_ARG;
  if (num_pairs > 0 && !block_mapping_host) return PKV_ERR_INVALID_ARG;
  const int b = static_cast<int>(pl->steps & 1);
  unsigned char* st = pl->staging[b];
  const StagingLayout& l = pl->layout;
  // the work list (the partitions that exist, longest first), planned on the
  // host from this step's lengths into the area's pinned buffer once step
  // i-2 has uploaded it
  if (max_context_len < 0 || partition_size < 0) return PKV_ERR_INVALID_ARG;
  const size_t cap = std::max<size_t>(work_items(S, pl->max_blocks_per_seq), 1);
  int32_t* work_host = pl->work_host + static_cast<size_t>(b) * cap * 2;
  const int part =
      pkv_paged_attn_partition_size(S, HKV, pl->block_size, max_context_len, partition_size);
  int items = 0;
  pkv_status r = cuda_status(cudaEventSynchronize(pl->ev_up[b]));
  if (r != PKV_OK) return r;
  if (S > 0) {
    r = pkv_decode_plan(context_lens_host, S, pl->block_size, part, work_host,
                        static_cast<int>(std::min<size_t>(cap, 0x7fffffff)), &items);
    if (r != PKV_OK) return r;
  }
  const size_t qo = static_cast<size_t>(S) * H * D * 2;
  const size_t kv = static_cast<size_t>(num_new_tokens) * HKV * D * 2;
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
      {l.tables, block_tables_host, static_cast<size_t>(S) * pl->max_blocks_per_seq * 4},
      {l.lens, context_lens_host, static_cast<size_t>(S) * 4},
      {l.work, work_host, static_cast<size_t>(items) * 8},
  };
  // upload: once step i-2 has finished reading this area's inputs
  r = cuda_status(cudaStreamWaitEvent(pl->up, pl->ev_comp[b], 0));
  for (const Copy& c : copies) {
    if (r != PKV_OK) return r;
    if (c.bytes == 0) continue;
    r = cuda_status(cudaMemcpyAsync(st + c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, pl->up));
  }
  if (r == PKV_OK) r = cuda_status(cudaEventRecord(pl->ev_up[b], pl->up));
  // compute: once the inputs are in and step i-2's output has left this area
  if (r == PKV_OK) r = cuda_status(cudaStreamWaitEvent(pl->compute, pl->ev_up[b], 0));
  if (r == PKV_OK) r = cuda_status(cudaStreamWaitEvent(pl->compute, pl->ev_down[b], 0));
  if (r != PKV_OK) return r;
  void* cs = pl->compute;
  r = pkv_copy_blocks(k_cache, v_cache, reinterpret_cast<const int64_t*>(st + l.pairs), num_pairs,
                      HKV, D, pl->block_size, num_blocks, pl->dtype, dev_err, cs);
  if (r == PKV_OK)
    r = pkv_reshape_and_cache(st + l.key, st + l.value, k_cache, v_cache,
                              reinterpret_cast<const int64_t*>(st + l.slots), num_new_tokens, HKV,
                              D, pl->block_size, num_blocks, pl->dtype, dev_err, cs);
  if (r == PKV_OK)
    r = pkv_paged_attn_decode_planned(st + l.out, st + l.q, k_cache, v_cache,
                                      reinterpret_cast<const int32_t*>(st + l.tables),
                                      reinterpret_cast<const int32_t*>(st + l.lens),
                                      reinterpret_cast<const int32_t*>(st + l.work), items,
                                      scale, S, H, HKV, D, pl->block_size,
                                      pl->max_blocks_per_seq, max_context_len, num_blocks,
                                      pl->dtype, part, workspace, workspace_bytes, dev_err, cs);
  if (r == PKV_OK) r = cuda_status(cudaEventRecord(pl->ev_comp[b], pl->compute));
  // download: once this step's output is written
  if (r == PKV_OK) r = cuda_status(cudaStreamWaitEvent(pl->down, pl->ev_comp[b], 0));
  if (r == PKV_OK && qo > 0)
    r = cuda_status(cudaMemcpyAsync(out_host, st + l.out, qo, cudaMemcpyDeviceToHost, pl->down));
  if (r == PKV_OK) r = cuda_status(cudaEventRecord(pl->ev_down[b], pl->down));
  if (r == PKV_OK) ++pl->steps;
  return r;
}

extern "C" pkv_status pkv_decode_pipeline_join(pkv_decode_pipeline* pl, void* stream) {
  using namespace pkv;
  if (pl == nullptr) return PKV_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  pkv_status r = cuda_status(cudaStreamWaitEvent(s, pl->ev_down[0], 0));
  if (r == PKV_OK) r = cuda_status(cudaStreamWaitEvent(s, pl->ev_down[1], 0));
  return r;
}

extern "C" pkv_status pkv_decode_pipeline_sync(pkv_decode_pipeline* pl) {
  using namespace pkv;
  if (pl == nullptr) return PKV_ERR_INVALID_ARG;
  pkv_status r = cuda_status(cudaEventSynchronize(pl->ev_down[0]));
  if (r == PKV_OK) r = cuda_status(cudaEventSynchronize(pl->ev_down[1]));
  return r;
}

extern "C" void pkv_decode_pipeline_destroy(pkv_decode_pipeline* pl) {
  if (pl == nullptr) return;
  pkv::step::pipeline_release(pl);
  delete pl;
}
