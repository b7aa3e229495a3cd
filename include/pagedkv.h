/*
 * pagedkv.h — C ABI of libpagedkv.so: PagedAttention decode on NVIDIA B200
 * (sm_100a), the cache-write scatter, the copy-on-write block copy, and a
 * host-side block allocator with prefix caching; beyond the decode path,
 * chunked-prefill attention, cascade decode over shared prefixes, and an
 * 8-bit (E4M3) cache.
 *
 * Sources cited by page title and section:
 *   [csdn]       devpress.csdn.net, "vLLM镜像深度优化：PagedAttention助力大模型推理效率飞跃"
 *   [cortexgrid] aidocs.cortexgrid.cn/docs/0a2c4066ef83, vLLM explainer with an FAQ
 *   [betteryeah] betteryeah.com, "vLLM是什么？完整解析高性能LLM推理引擎的技术原理与部署实践"
 *
 * The KV cache is cut into fixed-size blocks (pages) of block_size tokens that
 * sit anywhere in a physical pool; a per-sequence block table maps logical
 * block j of sequence i to a physical block ([csdn] "分页式KV缓存"; [betteryeah]
 * §2.2; [cortexgrid] FAQ on block tables).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Layouts are row-major.  The caches are
 *        k_cache, v_cache : [num_blocks, num_kv_heads, block_size, head_dim]
 *    so one (block, kv head) is one contiguous run of block_size*head_dim
 *    elements.  Elements are 16-bit (PKV_FP16 or PKV_BF16), or 1-byte E4M3
 *    codes for the *_fp8 entry points (and copy_blocks with PKV_FP8_E4M3).
 *  - A slot is physical_block * block_size + offset (int64); a negative slot
 *    marks a padding token.
 *  - Ownership: the caller owns every buffer.  The library never allocates or
 *    frees device memory; scratch for split-K decode ("workspace") and for the
 *    host-buffer step ("staging") is passed in by the caller (except for
 *    pkv_paged_attn_decode_static_ws, whose scratch is a fixed array inside
 *    the library).
 *  - Execution: device work is enqueued asynchronously on `stream` (a
 *    cudaStream_t passed as void*; NULL is the legacy default stream).  No
 *    entry point synchronizes, with one exception: pkv_decode_step_host
 *    given pageable (not page-locked) host buffers, whose copies the CUDA
 *    runtime performs synchronously.  All device pointers must belong to the
 *    device that is current on the calling thread.
 *  - Host-side validation happens before anything is enqueued: a bad scalar or
 *    a null / misaligned pointer returns PKV_ERR_INVALID_ARG, a valid but
 *    unbuilt shape returns PKV_ERR_UNSUPPORTED, a launch failure returns
 *    PKV_ERR_CUDA (pkv_last_cuda_error() gives the CUDA error code).
 *  - Device-side index errors (values the host cannot see because they live
 *    in device memory) never fault: the kernel skips the offending access and
 *    ORs a PKV_DEVERR_* bit into *dev_err when dev_err is not NULL.  Read the
 *    word after the stream has synchronized; outputs are then unreliable.
 *  - Alignment: every tensor pointer (16-bit or E4M3) must be 16-byte aligned.
 *  - Supported shapes: head_dim in {64, 128}, block_size in {16, 32},
 *    num_heads / num_kv_heads in {1, 2, 4, 8}, q/out dtype fp16 or bf16,
 *    for every entry point and cache type.
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = 1,   /* bad scalar, null or misaligned pointer      */
  PKV_ERR_UNSUPPORTED = 2,   /* shape / dtype combination not built         */
  PKV_ERR_WORKSPACE = 3,     /* workspace or staging buffer too small       */
  PKV_ERR_CUDA = 4,          /* a CUDA runtime call failed                  */
  PKV_ERR_OUT_OF_BLOCKS = 5  /* allocator: the free list is empty           */
} pkv_status;

/* PKV_FP8_E4M3 is a cache element type only (copy_blocks, and the caches of
 * the *_fp8 entry points); queries and outputs are always 16-bit. */
typedef enum { PKV_FP16 = 0, PKV_BF16 = 1, PKV_FP8_E4M3 = 2 } pkv_dtype;

/* Bits ORed into *dev_err by the kernels. */
#define PKV_DEVERR_BAD_BLOCK 1u   /* decode: table entry outside [0, num_blocks)          */
#define PKV_DEVERR_BAD_SLOT 2u    /* reshape_and_cache: slot >= num_blocks * block_size   */
#define PKV_DEVERR_BAD_PAIR 4u    /* copy_blocks: src or dst outside [0, num_blocks)      */
#define PKV_DEVERR_BAD_CONTEXT 8u /* decode: context_len < 0, > max_context_len, or more
                                     blocks than max_blocks_per_seq                        */
#define PKV_DEVERR_TIMEOUT 16u    /* decode: a bounded wait for an async copy gave up      */
#define PKV_DEVERR_BAD_SCALE 32u  /* *_fp8: a scale that is not finite and > 0            */
#define PKV_DEVERR_BAD_ORDER 64u  /* *_ordered, *_planned: an entry outside [0, num_seqs),
                                     or a work item that disagrees with the lengths */

/* Library version string, e.g. "pagedkv 0.1.0 sm_100a". */
const char* pkv_version(void);
/* Static English description of a status code. */
const char* pkv_status_string(int status);
/* cudaError_t of the most recent PKV_ERR_CUDA on the calling thread (0 if none). */
int pkv_last_cuda_error(void);

/*
 * pkv_reshape_and_cache — write the K and V vectors of new tokens into their
 * cache slots ([csdn] "内存困局的破局者": the cache keeps K and V per token;
 * [betteryeah] §2.2: pages are filled as a sequence grows).
 *
 *   key, value    device, [num_tokens, num_kv_heads, head_dim], 16-bit
 *   k_cache, v_cache  device caches (layout above), written in place
 *   slot_mapping  device int64 [num_tokens]; token t goes to
 *                 block = slot / block_size, offset = slot % block_size;
 *                 slot < 0 skips the token; slot >= num_blocks*block_size sets
 *                 PKV_DEVERR_BAD_SLOT and skips it.
 * Bit-exact copy.  Two tokens with the same slot leave one of them (which
 * one is unspecified).  num_tokens == 0 is a no-op.
 */
pkv_status pkv_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                 void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                 int num_kv_heads, int head_dim, int block_size,
                                 int num_blocks, pkv_dtype dtype, unsigned* dev_err,
                                 void* stream);

/*
 * pkv_copy_blocks — copy-on-write block copy ([cortexgrid] FAQ on parallel
 * sampling: shared blocks are reference-counted and copied when several
 * holders must modify them).
 *
 *   block_mapping  device int64 [num_pairs, 2] of (src, dst) physical blocks.
 *                  For each pair the whole K block and the whole V block (all
 *                  kv heads, offsets and dims) of src are copied to dst.
 * Preconditions (what the allocator produces): dst values are distinct and no
 * dst is also a src in the same call; otherwise the result is unspecified.
 * A pair with an index outside [0, num_blocks) sets PKV_DEVERR_BAD_PAIR and
 * is skipped.  Bit-exact.  num_pairs == 0 is a no-op.  dtype is the cache's
 * element type: PKV_FP16, PKV_BF16 or PKV_FP8_E4M3 (1-byte codes).
 */
pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                           int num_pairs, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, pkv_dtype dtype, unsigned* dev_err, void* stream);

/*
 * Split-K (partitioned) decode.  For long contexts the context of each
 * sequence is cut into partitions of partition_size tokens; each partition
 * produces a (max logit, exp-sum, unnormalised output) triple in the
 * workspace and a second kernel merges them.  pkv_paged_attn_partition_size
 * returns the partition size `pkv_paged_attn_decode` will use (16-bit caches),
 * pkv_paged_attn_partition_size_fp8 the one `pkv_paged_attn_decode_fp8` will:
 *   requested > 0  -> requested (must be a multiple of block_size);
 *   requested == 0 -> chosen from the shape, at most 4096 tokens (E4M3: 2048,
 *                     since a 1-byte cache is read twice as fast and a long
 *                     partition's CTA would outlast the launch); a value >=
 *                     max_context_len means single pass (no workspace needed).
 */
int pkv_paged_attn_partition_size(int num_seqs, int num_kv_heads, int block_size,
                                  int max_context_len, int requested);
int pkv_paged_attn_partition_size_fp8(int num_seqs, int num_kv_heads, int block_size,
                                      int max_context_len, int requested);

/* Workspace bytes pkv_paged_attn_decode and pkv_paged_attn_decode_fp8 need
 * for these arguments (the larger of the two; 0 when both run single-pass).
 * Returns 0 too for invalid arguments. */
size_t pkv_paged_attn_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                      int head_dim, int block_size, int max_context_len,
                                      int partition_size);

/*
 * pkv_paged_attn_decode — attention of each sequence's one new query token
 * over its paged KV cache.  The kernel assembles each sequence's keys and
 * values from the block table across non-contiguous blocks ([csdn]
 * "分页式KV缓存"; [betteryeah] §2.4), so the result equals
 *     out[i, h, :] = softmax(scale * q[i, h, :] . K_i^T) . V_i
 * over the context_lens[i] cached tokens of sequence i, where query head h
 * reads kv head h / (num_heads / num_kv_heads).  fp32 accumulation, output
 * rounded to the input dtype (round to nearest even).
 *
 *   out            device [num_seqs, num_heads, head_dim], written
 *   q              device [num_seqs, num_heads, head_dim]
 *   block_tables   device int32 [num_seqs, max_blocks_per_seq]; entries at or
 *                  beyond ceil(context_len / block_size) are never read
 *   context_lens   device int32 [num_seqs]; 0 gives an all-zero output row
 *   max_context_len  an upper bound of context_lens (sizes the launch)
 *   partition_size 0 = choose; else force this partition size (see above)
 *   workspace      device, >= pkv_paged_attn_workspace_bytes(...) bytes,
 *                  16-byte aligned; may be NULL when that is 0.  Its contents
 *                  need no initialisation and are scratch afterwards.
 * A table entry outside [0, num_blocks) sets PKV_DEVERR_BAD_BLOCK and that
 * block is left out.  num_seqs == 0 is a no-op.
 */
pkv_status pkv_paged_attn_decode(void* out, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, float scale, int num_seqs,
                                 int num_heads, int num_kv_heads, int head_dim,
                                 int block_size, int max_blocks_per_seq, int max_context_len,
                                 int num_blocks, pkv_dtype dtype, int partition_size,
                                 void* workspace, size_t workspace_bytes, unsigned* dev_err,
                                 void* stream);

/*
 * pkv_paged_attn_prefill — chunked-prefill attention over the paged cache.
 * Sequence i appends q_len_i = query_start[i+1] - query_start[i] tokens in
 * this step; their K/V must already be in the cache (pkv_reshape_and_cache),
 * so the sequence caches context_lens[i] tokens and its j-th new token sits at
 * position p = context_lens[i] - q_len_i + j.  That token's query attends
 * causally to tokens 0..p, gathered through the block table as in decode
 * ([csdn] "分页式KV缓存"; [betteryeah] §2.2, §2.4):
 *     out[t, h, :] = softmax(scale * q[t, h, :] . K[0..p]^T) . V[0..p]
 * with query head h reading kv head h / (num_heads / num_kv_heads).  fp32
 * accumulation on the tensor cores (tcgen05 with TMEM accumulators for
 * head_dim 128, mma.sync for 64); output rounded to nearest even.
 *
 *   q, out        device [T, num_heads, head_dim] with T = query_start[num_seqs]:
 *                 the queries of all sequences, packed in order
 *   num_tokens    T (the extent of q and out)
 *   query_start   device int32 [num_seqs + 1], non-decreasing, starting at 0
 *   max_query_len an upper bound of q_len_i (sizes the launch); <= max_context_len
 * A sequence whose q_len is negative, above its context length or above
 * max_query_len, or whose context length is out of range, sets
 * PKV_DEVERR_BAD_CONTEXT and its rows are left unwritten.  A table entry
 * outside [0, num_blocks) sets PKV_DEVERR_BAD_BLOCK.  No workspace is needed.
 */
pkv_status pkv_paged_attn_prefill(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, const int32_t* query_start,
                                  float scale, int num_seqs, int num_tokens, int num_heads,
                                  int num_kv_heads,
                                  int head_dim, int block_size, int max_blocks_per_seq,
                                  int max_context_len, int max_query_len, int num_blocks,
                                  pkv_dtype dtype, unsigned* dev_err, void* stream);

/*
 * Sequence order for decode.  A decode grid takes its (sequence, kv head,
 * partition) CTAs in order; with a few waves of CTAs of very different
 * lengths, a long sequence that starts last leaves the GPU partly idle at the
 * end.  pkv_decode_order (host only) writes into order[num_seqs] the
 * sequences longest first, by context length in buckets of 256 tokens, index
 * order within a bucket (so sequences of about the same length, such as the
 * samples of one prompt that share its blocks, stay adjacent and share L2).
 * context_lens and order are host arrays.
 *
 * pkv_paged_attn_decode_ordered / pkv_paged_attn_decode_fp8_ordered are
 * pkv_paged_attn_decode / pkv_paged_attn_decode_fp8 with the CTAs taken in
 * the order of seq_order (device int32 [num_seqs], a permutation of
 * 0..num_seqs-1, e.g. pkv_decode_order's); results are identical.  An entry
 * outside [0, num_seqs) sets PKV_DEVERR_BAD_ORDER and that entry's CTAs do
 * nothing; a repeated entry leaves the missing sequences' outputs unwritten.
 * The pages do not order sequences; this is a scheduling choice for B200.
 */
pkv_status pkv_decode_order(const int32_t* context_lens, int num_seqs, int32_t* order);
pkv_status pkv_paged_attn_decode_ordered(void* out, const void* q, const void* k_cache,
                                         const void* v_cache, const int32_t* block_tables,
                                         const int32_t* context_lens, const int32_t* seq_order,
                                         float scale, int num_seqs, int num_heads,
                                         int num_kv_heads, int head_dim, int block_size,
                                         int max_blocks_per_seq, int max_context_len,
                                         int num_blocks, pkv_dtype dtype, int partition_size,
                                         void* workspace, size_t workspace_bytes,
                                         unsigned* dev_err, void* stream);
pkv_status pkv_paged_attn_decode_fp8_ordered(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* seq_order,
    float scale, const float* k_scales, const float* v_scales, int num_seqs, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int max_context_len,
    int num_blocks, pkv_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes,
    unsigned* dev_err, void* stream);

/*
 * Planned decode.  A split-K decode grid holds max-context / partition CTAs
 * for every (sequence, kv head), and those past a shorter sequence's end
 * find no tokens and exit.  When the caller knows the context lengths on the
 * host (the scheduler that owns the block tables does), pkv_decode_plan lists
 * only the (sequence, partition) items that exist, and the planned decode
 * launches one CTA per item and kv head.  Results are identical to
 * pkv_paged_attn_decode with the same partition_size.  Not in the pages: a
 * scheduling choice for B200.
 *
 * pkv_decode_plan (host only): context_lens is a host int32 [num_seqs];
 * partition_size > 0 and a multiple of block_size (e.g. what
 * pkv_paged_attn_partition_size or _fp8 returns for the batch).  Writes the
 * item count, sum over sequences of max(1, ceil(ceil(len / block_size) /
 * (partition_size / block_size))), into *num_items and, when work is not
 * NULL, the items into work (host int32 [capacity][2]; capacity below the
 * count is PKV_ERR_INVALID_ARG): item i is (sequence, partition | count << 16)
 * where count is the sequence's partition count.  Items come longest first
 * by their own token count, in buckets of 256 tokens, in (sequence,
 * partition) order within a bucket.  A sequence of more than 65535
 * partitions is PKV_ERR_UNSUPPORTED.  With work == NULL it only counts.
 *
 * pkv_paged_attn_decode_planned / pkv_paged_attn_decode_fp8_planned take the
 * arguments of pkv_paged_attn_decode / _fp8 and the plan's items: work is the
 * device copy (8-byte aligned) of pkv_decode_plan's output for these
 * context lengths, num_items its count (at least num_seqs), partition_size
 * the one it was planned with (0 is PKV_ERR_INVALID_ARG).  Workspace as for
 * pkv_paged_attn_decode with that partition_size.  An item whose sequence is
 * outside [0, num_seqs), or whose partition count disagrees with the
 * sequence's context length on the device, sets PKV_DEVERR_BAD_ORDER (the
 * sequence's output is then not to be trusted: a list planned from other
 * lengths may lack partitions); a list that leaves a sequence out leaves its
 * output unwritten.
 */
pkv_status pkv_decode_plan(const int32_t* context_lens, int num_seqs, int block_size,
                           int partition_size, int32_t* work, int capacity, int* num_items);
pkv_status pkv_paged_attn_decode_planned(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* work, int num_items,
    float scale, int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int max_context_len, int num_blocks, pkv_dtype dtype,
    int partition_size, void* workspace, size_t workspace_bytes, unsigned* dev_err, void* stream);
pkv_status pkv_paged_attn_decode_fp8_planned(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* work, int num_items,
    float scale, const float* k_scales, const float* v_scales, int num_seqs, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int max_context_len,
    int num_blocks, pkv_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes,
    unsigned* dev_err, void* stream);

/*
 * pkv_testing_decode_wait — for tests of failure detection; not for serving.
 * Every wait of a decode kernel on its own loads is bounded: a warp that waits
 * longer than wait_ns (2 s by default) gives up, ORs PKV_DEVERR_TIMEOUT into
 * *dev_err, waits (bounded by 2 s) for its loads still in flight, and lets the
 * kernel finish, so the CUDA context stays usable.  This call sets wait_ns
 * for later decode launches from any thread (0 < wait_ns <= 2e9, else
 * PKV_ERR_INVALID_ARG).  With withhold_first_load non-zero, the first CTA of
 * every later decode launch skips its first load, so that a wait runs out
 * and the path above runs; its outputs are then not meaningful.  Restore
 * with (2000000000, 0).
 */
pkv_status pkv_testing_decode_wait(uint64_t wait_ns, int withhold_first_load);

/*
 * pkv_paged_attn_decode_static_ws — pkv_paged_attn_decode without a caller
 * workspace.  No counterpart in the source pages: it exists for callers that
 * cannot allocate device memory, such as a plugin inside a host application
 * that owns all device allocations, or a serving loop that must not call
 * cudaMalloc after start-up (cudaMalloc can synchronise the device).
 *
 * Arguments and results are those of pkv_paged_attn_decode; only the split-K
 * scratch differs.  It is a fixed array of PKV_STATIC_WORKSPACE_BYTES inside
 * the library, which every GPU that loads the library holds until the process
 * exits.  This entry point allocates and frees nothing.
 *  - If the call would need more scratch than that (see
 *    pkv_paged_attn_workspace_bytes), it returns PKV_ERR_WORKSPACE and
 *    enqueues nothing.  16 MiB holds, e.g., 8 sequences x 40 heads x 64
 *    partitions of head_dim 128.
 *  - The array exists once per CUDA context that loads the library: the
 *    device's primary context, a primary context rebuilt after
 *    cudaDeviceReset, or a context the application created and made current
 *    through the driver API each hold their own copy, at their own address.
 *    The first call made with a context current looks the address up in that
 *    context (cudaGetSymbolAddress) and caches it under the context's id;
 *    later calls in the same context only read the cache.  Make the first
 *    call in each context before any stream capture.
 *  - All calls in a context share the one array, and it keeps whatever the
 *    last call left there.  Nothing in it needs to start at zero: every value
 *    a call reads back was written earlier in the same call.  Calls that
 *    overlap on the GPU (different streams, or different host threads without
 *    ordering between them) race on the array; serialise them.
 */
#define PKV_STATIC_WORKSPACE_BYTES ((size_t)16 << 20)
pkv_status pkv_paged_attn_decode_static_ws(void* out, const void* q, const void* k_cache,
                                           const void* v_cache, const int32_t* block_tables,
                                           const int32_t* context_lens, float scale,
                                           int num_seqs, int num_heads, int num_kv_heads,
                                           int head_dim, int block_size, int max_blocks_per_seq,
                                           int max_context_len, int num_blocks, pkv_dtype dtype,
                                           int partition_size, unsigned* dev_err, void* stream);

/*
 * pkv_paged_attn_decode_cascade — pkv_paged_attn_decode for sequences that
 * share a cached prefix, such as the parallel samples of one prompt
 * ([cortexgrid] FAQ on parallel sampling; [csdn] "分页式KV缓存": sequences
 * with a common prompt point at the same first pages).  The result is that
 * of pkv_paged_attn_decode on the same arguments; only the work differs: the
 * shared blocks are read once per group instead of once per sequence.
 *
 *   group_start    device int32 [num_groups + 1], non-decreasing, 0 first and
 *                  num_seqs last: group g is sequences group_start[g] ..
 *                  group_start[g+1] - 1 (so members are consecutive)
 *   shared_blocks  device int32 [num_groups]: the first shared_blocks[g]
 *                  entries of every member's table row are the same physical
 *                  blocks (whole blocks only: a partly filled last prompt
 *                  block is per member after copy-on-write), and every member
 *                  caches at least shared_blocks[g] * block_size tokens
 *   max_group_size, max_shared_blocks  upper bounds (size the launch);
 *                  max_shared_blocks * block_size <= max_context_len.  With
 *                  max_shared_blocks = 0 the shared-prefix pass is skipped
 *   workspace      >= pkv_paged_attn_cascade_workspace_bytes(...) bytes
 * The group's table entries are read from its first member.  A member whose
 * context is shorter than its group's shared tokens sets
 * PKV_DEVERR_BAD_CONTEXT, and so does a shared_blocks[g] above
 * max_shared_blocks: both passes then treat the group as sharing only
 * max_shared_blocks blocks.  head_dim 64 or 128; 16-bit caches (E4M3:
 * pkv_paged_attn_decode_cascade_fp8).  Other arguments and errors as in
 * pkv_paged_attn_decode.
 */
size_t pkv_paged_attn_cascade_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                              int head_dim, int block_size,
                                              int max_context_len, int partition_size);
pkv_status pkv_paged_attn_decode_cascade(void* out, const void* q, const void* k_cache,
                                         const void* v_cache, const int32_t* block_tables,
                                         const int32_t* context_lens,
                                         const int32_t* group_start,
                                         const int32_t* shared_blocks, float scale,
                                         int num_seqs, int num_groups, int max_group_size,
                                         int max_shared_blocks, int num_heads,
                                         int num_kv_heads, int head_dim, int block_size,
                                         int max_blocks_per_seq, int max_context_len,
                                         int num_blocks, pkv_dtype dtype, int partition_size,
                                         void* workspace, size_t workspace_bytes,
                                         unsigned* dev_err, void* stream);

/*
 * 8-bit (E4M3) cache.  The pages name quantised inference as a way to fit
 * larger models and batches into the memory ([csdn] "量化模型优先考虑边缘场景";
 * [betteryeah] §4.2 "启用量化推理") without fixing a format; this library stores
 * the cache as OCP FP8 E4M3 codes (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits, subnormals, no infinities, 0x7F/0xFF NaN, largest finite
 * 448) with one float scale per kv head and cache:
 *     code = E4M3(x / scale[h]),   value = decode(code) * scale[h].
 * Each cache element is one byte; the layout is that of the 16-bit caches.
 * k_scales, v_scales: device float32 [num_kv_heads] (the same value in every
 * entry gives one scale per cache).  They live in device memory so a captured
 * graph can pick up new scales; a scale that is not finite and > 0 sets
 * PKV_DEVERR_BAD_SCALE (the write then skips that head's elements; decode
 * output is unreliable).
 *
 * pkv_reshape_and_cache_fp8 — pkv_reshape_and_cache that quantises on the way
 * in.  key/value are 16-bit of type `dtype` ([num_tokens, num_kv_heads,
 * head_dim]); k_cache/v_cache hold codes.  Each element of kv head h is
 * widened to float32, divided by k_scales[h] (keys) or v_scales[h] (values)
 * in IEEE float32 (round to nearest), and rounded to E4M3 by
 * round-to-nearest-even; magnitudes that round above 448 become +-448, NaN
 * becomes a NaN code.  Slots behave as in pkv_reshape_and_cache.  Null
 * scale pointers give PKV_ERR_INVALID_ARG.
 */
pkv_status pkv_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache,
                                     void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int num_blocks, pkv_dtype dtype, const float* k_scales,
                                     const float* v_scales, unsigned* dev_err, void* stream);

/*
 * pkv_paged_attn_decode_fp8 — pkv_paged_attn_decode over E4M3 caches:
 *     out[i, h, :] = softmax(scale * q[i, h, :] . K~^T) . V~,
 *     K~ = decode(k_cache codes) * k_scales[g],  V~ = decode(v_cache codes) * v_scales[g]
 * with g the kv head of query head h.  q and out are 16-bit of type `dtype`;
 * every other argument, the workspace (same size as
 * pkv_paged_attn_workspace_bytes gives) and the error behaviour are those of
 * pkv_paged_attn_decode.  fp32 accumulation; head_dim 128 runs on the tensor
 * cores (mma.sync with the codes widened exactly to fp16; bf16 queries are
 * rounded to fp16 there, magnitudes above 65504 saturating), head_dim 64 on
 * the CUDA cores in fp32.  Null scale pointers give PKV_ERR_INVALID_ARG.
 */
pkv_status pkv_paged_attn_decode_fp8(void* out, const void* q, const void* k_cache,
                                     const void* v_cache, const int32_t* block_tables,
                                     const int32_t* context_lens, float scale,
                                     const float* k_scales, const float* v_scales,
                                     int num_seqs, int num_heads,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int max_blocks_per_seq, int max_context_len,
                                     int num_blocks, pkv_dtype dtype, int partition_size,
                                     void* workspace, size_t workspace_bytes,
                                     unsigned* dev_err, void* stream);

/*
 * pkv_paged_attn_prefill_fp8 — pkv_paged_attn_prefill over E4M3 caches:
 *     out[t, h, :] = softmax(scale * q[t, h, :] . K~[0..p]^T) . V~[0..p]
 * with K~ and V~ decoded as for pkv_paged_attn_decode_fp8 (codes times the kv
 * head's k_scales / v_scales entry).  The kernel stages each tile's codes by
 * TMA and widens them exactly to fp16 before the tensor cores read them
 * (tcgen05 at head_dim 128, mma.sync at 64); bf16 queries are rounded to fp16
 * there, magnitudes above 65504 saturating.  The K scale folds into the logit
 * scale and the V scale into the final normalisation.  Every other argument
 * and the error behaviour are those of pkv_paged_attn_prefill; null scale
 * pointers give PKV_ERR_INVALID_ARG and a scale that is not finite and > 0
 * sets PKV_DEVERR_BAD_SCALE.
 */
pkv_status pkv_paged_attn_prefill_fp8(void* out, const void* q, const void* k_cache,
                                      const void* v_cache, const int32_t* block_tables,
                                      const int32_t* context_lens, const int32_t* query_start,
                                      float scale, const float* k_scales, const float* v_scales,
                                      int num_seqs, int num_tokens, int num_heads,
                                      int num_kv_heads, int head_dim, int block_size,
                                      int max_blocks_per_seq, int max_context_len,
                                      int max_query_len, int num_blocks, pkv_dtype dtype,
                                      unsigned* dev_err, void* stream);

/*
 * Planned prefill (head_dim 128).  The tcgen05 prefill gives each (sequence,
 * query tile of 256 rows) unit one CTA per kv head, which reads every key its
 * rows see; in a batch of few sequences of very different histories the
 * units of the longest one outlast the rest and the launch ends on them.
 * pkv_prefill_plan (host only) cuts each unit whose CTA would cost more than
 * 1.5 SM shares of the batch into up to 4 pieces of about one share: whole
 * 64-key tiles of history, which every row of the unit sees, then the rest
 * of its keys with the causal edge.  The planned prefill runs one CTA per
 * item (a whole unit or a piece, most expensive first); the pieces of a
 * unit write partials (m, l,
 * unnormalised o in fp32) to the workspace and a merge kernel combines them
 * as the split-K decode reduce does.  The result is that of
 * pkv_paged_attn_prefill up to the rounding of that merge.  Not in the
 * pages: a scheduling choice for B200.
 *
 * pkv_prefill_plan: query_start (host int32 [num_seqs + 1]) and context_lens
 * (host int32 [num_seqs]) as the prefill will see them; num_sms the SMs the
 * launch spreads over (148 on B200; <= 0 is PKV_ERR_INVALID_ARG).  Writes
 * the item count to *num_items, the merge-entry count to *num_merges and,
 * if workspace_bytes is not NULL, the workspace the planned prefill needs.
 * work (host int32 [work_capacity][8]) and merges (host int32
 * [merge_capacity][4]) may be NULL to count only; a capacity below the count
 * is PKV_ERR_INVALID_ARG.  head_dim other than 128 is PKV_ERR_UNSUPPORTED.
 *
 * pkv_paged_attn_prefill_planned / pkv_paged_attn_prefill_fp8_planned take
 * the arguments of pkv_paged_attn_prefill / _fp8, the device copies of the
 * plan's work (num_items items) and merges (num_merges entries), and a
 * workspace (16-byte aligned) of at least the plan's size (needed only when
 * num_merges > 0, else PKV_ERR_WORKSPACE).  An item or merge entry that
 * names no sequence, or whose key range does not fit the sequence's lengths
 * on the device, sets PKV_DEVERR_BAD_ORDER and that unit's rows are not to
 * be trusted; a plan that leaves a unit out leaves its rows unwritten.
 */
pkv_status pkv_prefill_plan(const int32_t* query_start, const int32_t* context_lens,
                            int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                            int num_sms, int32_t* work, int work_capacity, int* num_items,
                            int32_t* merges, int merge_capacity, int* num_merges,
                            size_t* workspace_bytes);
pkv_status pkv_paged_attn_prefill_planned(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
    const int32_t* work, int num_items, const int32_t* merges, int num_merges, float scale,
    int num_seqs, int num_tokens, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int max_context_len, int max_query_len, int num_blocks,
    pkv_dtype dtype, void* workspace, size_t workspace_bytes, unsigned* dev_err, void* stream);
pkv_status pkv_paged_attn_prefill_fp8_planned(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
    const int32_t* work, int num_items, const int32_t* merges, int num_merges, float scale,
    const float* k_scales, const float* v_scales, int num_seqs, int num_tokens, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int max_context_len,
    int max_query_len, int num_blocks, pkv_dtype dtype, void* workspace, size_t workspace_bytes,
    unsigned* dev_err, void* stream);

/*
 * pkv_paged_attn_decode_cascade_fp8 — pkv_paged_attn_decode_cascade over E4M3
 * caches: the result is that of pkv_paged_attn_decode_fp8 on the same
 * arguments (K~, V~ = codes times the kv head's k_scales / v_scales entry).
 * The shared-prefix pass widens the codes to fp16 as
 * pkv_paged_attn_prefill_fp8 does (bf16 queries rounded to fp16 there), the
 * members' own blocks are read as pkv_paged_attn_decode_fp8 reads them.
 * Groups, workspace (pkv_paged_attn_cascade_workspace_bytes), head_dim 64 or
 * 128 and errors as in pkv_paged_attn_decode_cascade; null scale pointers give
 * PKV_ERR_INVALID_ARG and a scale that is not finite and > 0 sets
 * PKV_DEVERR_BAD_SCALE.  The shared pass widens every shared tile through
 * shared memory, so with 1-byte codes (whose repeats plain decode finds in
 * L2) it can be slower than pkv_paged_attn_decode_fp8 on the same batch.
 */
pkv_status pkv_paged_attn_decode_cascade_fp8(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* group_start,
    const int32_t* shared_blocks, float scale, const float* k_scales, const float* v_scales,
    int num_seqs, int num_groups, int max_group_size, int max_shared_blocks, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int max_context_len,
    int num_blocks, pkv_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes,
    unsigned* dev_err, void* stream);

/*
 * pkv_decode_step_host — one whole decode step from HOST buffers: copies the
 * step's inputs host->device, runs copy_blocks (if num_pairs > 0),
 * reshape_and_cache (if num_new_tokens > 0) and paged_attn_decode, and copies
 * the output back, all enqueued on `stream`.  The caches stay on the device.
 *
 *   *_host     host pointers; page-locked (pinned) memory makes the copies
 *              asynchronous, pageable memory works but copies synchronously.
 *              The host buffers must stay valid until the stream has finished.
 *   staging    device scratch of >= pkv_decode_step_staging_bytes(...) bytes
 *              (16-byte aligned) that receives the step's inputs and output.
 *   workspace  as for pkv_paged_attn_decode.
 * Shapes as for the three calls above.
 */
size_t pkv_decode_step_staging_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                     int head_dim, int max_blocks_per_seq, int num_new_tokens,
                                     int num_pairs);
pkv_status pkv_decode_step_host(
    void* out_host, const void* q_host, const void* key_host, const void* value_host,
    const int64_t* slot_mapping_host, int num_new_tokens, const int64_t* block_mapping_host,
    int num_pairs, const int32_t* block_tables_host, const int32_t* context_lens_host,
    void* k_cache, void* v_cache, float scale, int num_seqs, int num_heads, int num_kv_heads,
    int head_dim, int block_size, int max_blocks_per_seq, int max_context_len, int num_blocks,
    pkv_dtype dtype, int partition_size, void* staging, size_t staging_bytes, void* workspace,
    size_t workspace_bytes, unsigned* dev_err, void* stream);

/*
 * pkv_decode_pipeline — consecutive decode steps from HOST buffers, each the
 * work of pkv_decode_step_host, overlapped across three streams: step i+1's
 * inputs are copied host->device on an upload stream while step i computes on
 * the compute stream given at creation, and step i's output is copied back on
 * a download stream while step i+1 computes.  Every step still copies its
 * own inputs in and its output out.  No counterpart in the source pages,
 * which describe the serving loop only in words ([csdn] "典型工作流程拆解").
 *
 *   create   staging: device scratch of >= pkv_decode_pipeline_staging_bytes
 *            bytes (16-byte aligned): two areas, used by alternate steps, each
 *            sized for max_new_tokens new tokens and max_pairs copy pairs.
 *            The pipeline creates its two copy streams, six events and a
 *            pinned host buffer for two work lists (no device memory) and
 *            keeps `stream` as its compute stream.
 *   step     enqueues one step and returns; the cache work of consecutive
 *            steps stays in order on the compute stream.  The decode is
 *            planned on the host from the step's context lengths
 *            (pkv_decode_plan, with the partition pkv_paged_attn_partition_size
 *            gives for partition_size) and its work list is uploaded with the
 *            inputs.  num_new_tokens and
 *            num_pairs may vary per step up to the maxima.  The step's host
 *            buffers (pinned memory keeps the copies asynchronous) must stay
 *            valid and unchanged, and *out_host unread, until the step has
 *            completed (pkv_decode_pipeline_sync, or work ordered after
 *            pkv_decode_pipeline_join).  dev_err and workspace as in
 *            pkv_paged_attn_decode; the workspace is shared by the steps in
 *            compute-stream order.
 *   join     makes `stream` wait for every step enqueued so far (no host wait).
 *   sync     blocks the calling host thread until every step enqueued so far
 *            has completed.
 *   destroy  waits for the copy streams, then frees the streams and events.
 * Shapes and errors as for pkv_decode_step_host; a step beyond the maxima
 * returns PKV_ERR_INVALID_ARG and enqueues nothing.
 */
typedef struct pkv_decode_pipeline pkv_decode_pipeline;
size_t pkv_decode_pipeline_staging_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                         int head_dim, int max_blocks_per_seq,
                                         int max_new_tokens, int max_pairs);
pkv_status pkv_decode_pipeline_create(pkv_decode_pipeline** pipeline, int num_seqs,
                                      int num_heads, int num_kv_heads, int head_dim,
                                      int block_size, int max_blocks_per_seq,
                                      int max_new_tokens, int max_pairs, pkv_dtype dtype,
                                      void* staging, size_t staging_bytes, void* stream);
pkv_status pkv_decode_pipeline_step(
    pkv_decode_pipeline* pipeline, void* out_host, const void* q_host, const void* key_host,
    const void* value_host, const int64_t* slot_mapping_host, int num_new_tokens,
    const int64_t* block_mapping_host, int num_pairs, const int32_t* block_tables_host,
    const int32_t* context_lens_host, void* k_cache, void* v_cache, float scale,
    int max_context_len, int num_blocks, int partition_size, void* workspace,
    size_t workspace_bytes, unsigned* dev_err);
pkv_status pkv_decode_pipeline_join(pkv_decode_pipeline* pipeline, void* stream);
pkv_status pkv_decode_pipeline_sync(pkv_decode_pipeline* pipeline);
void pkv_decode_pipeline_destroy(pkv_decode_pipeline* pipeline);

/*
 * Host block allocator ([csdn] "分页式KV缓存" and "典型工作流程拆解" step 7;
 * [betteryeah] §2.2; [cortexgrid] FAQ on parallel sampling).  Host memory
 * only; not thread-safe (one allocator per scheduler thread).
 *
 *  - The free list is a FIFO queue: allocation takes the front, release
 *    appends at the back.  Its initial order is `free_order` (a permutation of
 *    0..num_blocks-1, copied) or the identity when NULL.
 *  - add_seq takes ceil(num_tokens / block_size) blocks, or none if short.
 *  - fork makes `child` share all of `parent`'s blocks (refcount + 1 each).
 *  - append_slot reserves the slot of the sequence's next token.  At a block
 *    boundary it takes a fresh block.  Inside a block whose refcount exceeds
 *    one it copies on write: it takes a fresh block, returns (old, new) in
 *    *cow_src / *cow_dst for pkv_copy_blocks, decrements the old block's
 *    refcount and points the table at the new block.  Otherwise both are -1.
 *    The last holder of a block (refcount 1) writes in place.
 *  - free_seq drops one reference per block, front to back; a block that
 *    reaches zero is appended to the free queue.
 * Errors: unknown / duplicate ids or bad sizes -> PKV_ERR_INVALID_ARG;
 * empty free list -> PKV_ERR_OUT_OF_BLOCKS (the state is left unchanged).
 */
typedef struct pkv_alloc pkv_alloc;

/* NULL on bad arguments (num_blocks <= 0, block_size <= 0, free_order not a permutation). */
pkv_alloc* pkv_alloc_create(int num_blocks, int block_size, const int32_t* free_order);
void pkv_alloc_destroy(pkv_alloc* a);
pkv_status pkv_alloc_add_seq(pkv_alloc* a, int64_t seq_id, int64_t num_tokens);
pkv_status pkv_alloc_fork(pkv_alloc* a, int64_t parent, int64_t child);
pkv_status pkv_alloc_append_slot(pkv_alloc* a, int64_t seq_id, int64_t* slot,
                                 int64_t* cow_src, int64_t* cow_dst);
/* Appends one token to each of seq_ids[0..n) in order.  slots[n] receives the
 * slots; cow_pairs[2*k], cow_pairs[2*k+1] the k-th copy pair (capacity n
 * pairs); *num_cow their count; *num_done how many appends succeeded (all n
 * unless an error status is returned). */
pkv_status pkv_alloc_append_slots(pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* slots,
                                  int64_t* cow_pairs, int* num_cow, int* num_done);
pkv_status pkv_alloc_free_seq(pkv_alloc* a, int64_t seq_id);
/* table_out: host int32 [n, max_blocks], padded with -1. */
pkv_status pkv_alloc_block_table(const pkv_alloc* a, const int64_t* seq_ids, int n,
                                 int max_blocks, int32_t* table_out);
/* lens_out: host int32 [n], each sequence's token count. */
pkv_status pkv_alloc_context_lens(const pkv_alloc* a, const int64_t* seq_ids, int n,
                                  int32_t* lens_out);
int pkv_alloc_num_free(const pkv_alloc* a);
/* Cached blocks with refcount 0 (kept for reuse, evicted when the free list is empty). */
int pkv_alloc_num_evictable(const pkv_alloc* a);
/* -1 for an out-of-range block. */
int pkv_alloc_refcount(const pkv_alloc* a, int block);
/* -1 for an unknown sequence. */
int64_t pkv_alloc_seq_len(const pkv_alloc* a, int64_t seq_id);
int pkv_alloc_seq_num_blocks(const pkv_alloc* a, int64_t seq_id);
/* Cached tokens and allocated blocks, each physical block counted once (a
 * block's fill is the most slots any holder has filled); utilization is
 * cached_tokens / (used_blocks * block_size). */
pkv_status pkv_alloc_usage(const pkv_alloc* a, int64_t* cached_tokens, int64_t* used_blocks);

/*
 * Prefix caching ([csdn] API example: `enable_prefix_caching`, and the
 * `cache_hit_rate` it recommends monitoring; sequences with a common prompt
 * point at the same first pages, [csdn] "分页式KV缓存").
 *
 * pkv_alloc_add_seq_cached admits a sequence whose prompt is token_ids[0..n).
 * A full block is identified by its whole token prefix.  The prompt's full
 * blocks are looked up in order; the cached ones are reused (refcount + 1) up
 * to the first miss, the rest are taken fresh, and each fresh full block is
 * registered under its prefix (the caller writes its K/V in the same step).
 * Partial blocks are never cached.  *num_cached_tokens receives the number of
 * leading prompt tokens whose K/V are already in the cache.
 *
 * A cached block whose refcount drops to zero stays cached and is evictable,
 * least recently released first; an allocation that finds the free list empty
 * evicts the oldest one.  Prefixes are compared through a 64-bit chain hash
 * plus the block's own tokens, so two different prefixes are confused only
 * on a 64-bit hash collision.  OUT_OF_BLOCKS leaves the state unchanged.
 */
pkv_status pkv_alloc_add_seq_cached(pkv_alloc* a, int64_t seq_id, const int32_t* token_ids,
                                    int64_t num_tokens, int64_t* num_cached_tokens);
/* Full blocks looked up, hits among them, blocks cached now, blocks evicted so far.
 * cache_hit_rate = hit_blocks / queried_blocks.  Any output may be NULL. */
pkv_status pkv_alloc_cache_stats(const pkv_alloc* a, int64_t* queried_blocks,
                                 int64_t* hit_blocks, int64_t* cached_blocks,
                                 int64_t* evicted_blocks);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */
