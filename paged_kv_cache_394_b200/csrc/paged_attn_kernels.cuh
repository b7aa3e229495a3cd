// paged_attn_kernels.cuh — PagedAttention decode kernels for B200 (sm_100a).
//
// What it computes.  Each sequence's one new query token attends over the
// sequence's cached keys and values, which live in fixed-size blocks scattered
// through a physical pool and are found through the sequence's block table;
// the kernel assembles the data from the page table across non-contiguous
// regions, transparently to the model ([csdn] "分页式KV缓存：让显存利用接近理论
// 极限"; [betteryeah] §2.2 and §2.4 "技术实现细节").  So, for sequence i and
// query head h (kv head g = h / G, G = num_heads / num_kv_heads):
//     out[i,h,:] = softmax(scale * q[i,h,:] . K^T) . V  over context_lens[i] tokens.
//
// How (B200 design).  The work is HBM-bound: every cached K/V byte is read
// once, and there are G multiply-adds per byte at most.  So:
//  * One CTA per (sequence, kv head, partition).  It serves all G query heads
//    of that kv head, so each K/V byte leaves HBM once.
//  * The partition's slice of the block table is staged in shared memory.
//  * Each warp owns a ring of NS stages in shared memory and streams its own
//    blocks (blocks w, w+W, w+2W, ... of the partition) with the TMA engine's
//    1-D bulk copy: one (block, kv head) of K is one contiguous block_size *
//    head_dim run (4 KiB at block 16 / dim 128), likewise V, so a stage is two
//    bulk copies completing on one mbarrier.  Lane 0 refills a stage as soon
//    as the warp has consumed it, so NS blocks per warp are always in flight.
//  * q·K: lane (c, r) holds 8 dims (chunk c) of q for all G heads and reads
//    8 dims of R rows at a time (conflict-free 16-byte shared loads); the
//    partial dot products are summed across the NC = D/8 lanes of a row by a
//    butterfly reduce-scatter, which leaves each lane one finished logit.
//  * Online softmax in base 2 (q is pre-scaled by scale*log2(e)); running max
//    and sum per head; the accumulator is rescaled only when the max moves.
//  * P·V with fp32 accumulators, 8 dims x G heads per lane.
//  * Warps merge their (max, sum, acc) in shared memory at the end.
//  * Long contexts: partitions of partition_size tokens write (max, sum,
//    unnormalised output) to the workspace and a reduce kernel merges them;
//    a sequence with a single partition is written directly.
//  * No waits on other CTAs anywhere; mbarrier waits are bounded in time.
#pragma once

#include <math.h>

#include <type_traits>

#include "common.cuh"

namespace pkv {

struct DecodeParams {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float qscale;  // scale * log2(e)
  const float* k_scales;  // 8-bit cache: per-kv-head K scales [num_kv_heads], else null
  const float* v_scales;  // 8-bit cache: per-kv-head V scales [num_kv_heads], else null
  int num_seqs;
  int num_heads;
  int num_kv_heads;
  int max_blocks_per_seq;
  int max_context_len;
  int num_blocks;
  int block_size;
  int part_blocks;  // blocks per partition
  int max_parts;    // workspace slots per (sequence, head)
  int grid_parts;   // partitions per (sequence, kv head) in the grid: max_parts,
                    // or max_parts - 1 under cascade decode (slot 0 is the prefix)
  float* ws_out;    // [S, H, max_parts, D]
  float* ws_max;    // [S, H, max_parts]
  float* ws_sum;    // [S, H, max_parts]
  unsigned* err;
  // Cascade decode (else null / 0): sequences come in groups, group g being
  // sequences group_start[g] .. group_start[g+1]-1, whose first
  // shared_blocks[g] blocks a separate prefix pass covers (its partial sits in
  // workspace slot 0).  The decode kernels then read only each sequence's
  // blocks after them, write partials from slot 1 on, and the reduce merges
  // every slot.
  const int32_t* group_start;
  const int32_t* shared_blocks;
  int num_groups;
  int max_shared_blocks;  // the host's bound on shared_blocks[g]; the prefix pass ran iff > 0
  // Bound on a warp's wait for its own loads (kWaitTimeoutNs unless a test
  // lowers it), and a test switch: CTA 0's warp 0 never issues its first
  // load, so that its wait runs out and the timeout path runs.
  uint64_t wait_ns;
  int withhold_first_load;
  // Optional order of the sequences over the grid (a permutation of
  // 0 .. num_seqs-1, longest first; see pkv_decode_order), else null.
  const int32_t* seq_order;
  // 1: the preceding kernel in the stream writes nothing this one reads (the
  // cascade suffix after its prefix pass, whose CTAs all waited for the cache
  // writes before letting this grid start), so skip griddepcontrol.wait.
  int independent_of_prior;
  // Optional work list (see pkv_decode_plan), else null: CTA b serves item
  // b / num_kv_heads for kv head b % num_kv_heads, and item i is the pair
  // (sequence, partition | partitions the planner counted for it << 16).
  // The grid then holds no CTA for a partition past a sequence's end.
  const int2* work;
};

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
// The (sequence, kv head, partition) a decode CTA serves: from the grid
// (sequence-major, in index order or the caller's order, partitions
// innermost) or from the work list.  `planned` is the work list's partition
// count for the sequence (0 without one); seq is not yet range-checked.
struct DecodeCta {
  int seq, kvh, part, planned;
};
__device__ __forceinline__ DecodeCta decode_cta(const DecodeParams& p) {
  DecodeCta c;
  if (p.work != nullptr) {
    const int2 w = p.work[blockIdx.x / p.num_kv_heads];
    c.kvh = blockIdx.x % p.num_kv_heads;
    c.seq = w.x;
    c.part = w.y & 0xffff;
    c.planned = static_cast<int>(static_cast<unsigned>(w.y) >> 16);
  } else {
    const int unit = blockIdx.x / p.grid_parts;
    c.part = blockIdx.x % p.grid_parts;
    c.kvh = unit % p.num_kv_heads;
    const int rank = unit / p.num_kv_heads;
    c.seq = p.seq_order != nullptr ? p.seq_order[rank] : rank;
    c.planned = 0;
  }
  return c;
}

// Whether a work item disagrees with the context length the kernel read: a
// list built from other lengths may miss partitions, so the call reports it.
__device__ __forceinline__ bool plan_mismatch(const DecodeParams& p, const DecodeCta& c,
                                              int nparts) {
  return p.work != nullptr && (c.planned != (nparts > 1 ? nparts : 1) || c.part >= c.planned);
}

__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

// First block a decode kernel reads for `seq`: 0, or under cascade decode the
// shared blocks of its group (binary search over group_start), at most nblk.
// A group's shared_blocks above the host's max_shared_blocks is clamped to it
// (the prefix pass covered no more; with max_shared_blocks = 0 it did not run
// and workspace slot 0 holds nothing of this call) and reported as
// PKV_DEVERR_BAD_CONTEXT by the thread that passes `report`.
__device__ __forceinline__ int cascade_start_block(const DecodeParams& p, int seq, int nblk,
                                                   bool report) {
  if (p.group_start == nullptr) return 0;
  int lo = 0, hi = p.num_groups;  // invariant: group_start[lo] <= seq < group_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.group_start[mid] <= seq) lo = mid; else hi = mid;
  }
  int shared = max(p.shared_blocks[lo], 0);
  if (shared > p.max_shared_blocks) {
    if (report) set_err(p.err, PKV_DEVERR_BAD_CONTEXT);
    shared = p.max_shared_blocks;
  }
  return min(shared, nblk);
}

template <int D_, int BS_, int G_, class DT_, int W_, int NS_, class KV_ = DT_>
struct DecodeTraits {
  static constexpr int D = D_, BS = BS_, G = G_, W = W_, NS = NS_;
  using DT = DT_;   // q and out
  using T = typename DT::T;
  using KV = KV_;   // cache elements: 16-bit like q, or 8-bit E4M3
  using KT = typename KV::T;
  static constexpr int KV_BYTES = static_cast<int>(sizeof(KT));
  static constexpr int NC = D / 8;                // 16-byte chunks per row
  static constexpr int LOG2_NC = ilog2(NC);
  static constexpr int R = 32 / NC;               // rows per warp-wide load
  static constexpr int ROWS_PER_LANE = BS / R;
  // rows per lane per sub-tile: keeps G * JS partial logits <= NC per lane
  static constexpr int JS = cmin(ROWS_PER_LANE, cmax(1, NC / G));
  static constexpr int TS = R * JS;               // tokens per sub-tile
  static constexpr int NSUB = BS / TS;
  static constexpr int NV = G * JS;               // partial logits per lane
  static constexpr int LOG2_NV = ilog2(NV);
  static constexpr int REP = NC / NV;             // lanes holding each logit
  static constexpr int SEG = JS * REP;            // lanes of one head within a row group
  static constexpr int CHUNK_ELEMS = BS * D;
  static constexpr int CHUNK_BYTES = CHUNK_ELEMS * KV_BYTES;
  static constexpr int STAGE_BYTES = 2 * CHUNK_BYTES;
  static constexpr int THREADS = W * 32;
  static constexpr int PB_FLOATS = R * NV + 8;    // p values + per-head alpha (G <= 8)
  static constexpr int RING_BYTES = W * NS * STAGE_BYTES;
  static constexpr int BAR_BYTES = W * NS * 8;
  static constexpr int PBUF_BYTES = W * 2 * PB_FLOATS * 4;
  static constexpr int COMBINE_BYTES = W * G * (D + 2) * 4;
  static_assert(NV <= NC && NC % NV == 0, "logit layout");
  static_assert(BS % TS == 0, "sub-tiles must tile a block");
  static_assert(COMBINE_BYTES <= RING_BYTES, "combine scratch reuses the ring");
  static_assert(G <= 8, "alpha slots");

  static size_t smem_bytes(int part_blocks) {
    return static_cast<size_t>(RING_BYTES) + BAR_BYTES + PBUF_BYTES +
           static_cast<size_t>(part_blocks) * 4;
  }
};

// Butterfly reduce-scatter of NV values over the NC lanes of a row group.
// Afterwards lane l holds the full sum of value index (l % NC) / (NC / NV).
template <int NV, int NC>
__device__ __forceinline__ float reduce_scatter(float (&v)[NV], int lane) {
  constexpr int LOG2_NC = ilog2(NC);
  constexpr int LOG2_NV = ilog2(NV);
#pragma unroll
  for (int step = 0; step < LOG2_NC; ++step) {
    const int mask = NC >> (step + 1);
    if (step < LOG2_NV) {
      const int half = NV >> (step + 1);
      const bool upper = (lane & mask) != 0;
#pragma unroll
      for (int k = 0; k < half; ++k) {
        const float send = upper ? v[k] : v[k + half];
        const float keep = upper ? v[k + half] : v[k];
        v[k] = keep + __shfl_xor_sync(kFullMask, send, mask);
      }
    } else {
      v[0] += __shfl_xor_sync(kFullMask, v[0], mask);
    }
  }
  return v[0];
}

// Max / sum over the lanes that hold logits of one head: SEG lanes in each
// row group (skipping replica lanes for the sum) times the R row groups.
template <class Tr>
__device__ __forceinline__ float segment_max(float x) {
#pragma unroll
  for (int m = Tr::REP; m < Tr::SEG; m <<= 1) x = fmaxf(x, __shfl_xor_sync(kFullMask, x, m));
#pragma unroll
  for (int m = Tr::NC; m < 32; m <<= 1) x = fmaxf(x, __shfl_xor_sync(kFullMask, x, m));
  return x;
}

template <class Tr>
__device__ __forceinline__ float segment_sum(float x) {
#pragma unroll
  for (int m = Tr::REP; m < Tr::SEG; m <<= 1) x += __shfl_xor_sync(kFullMask, x, m);
#pragma unroll
  for (int m = Tr::NC; m < 32; m <<= 1) x += __shfl_xor_sync(kFullMask, x, m);
  return x;
}

// 8 consecutive cache elements of a shared-memory row -> floats.
template <class KV>
__device__ __forceinline__ void load_row8(const typename KV::T* at, float (&f)[8]) {
  if constexpr (sizeof(typename KV::T) == 1) {
    unpack8(*reinterpret_cast<const uint2*>(at), f, KV());
  } else {
    unpack8(*reinterpret_cast<const uint4*>(at), f, KV());
  }
}

// Per-warp running state of the online softmax.
template <class Tr>
struct WarpState {
  float q[Tr::G][8];    // q chunk of each head, pre-scaled
  float acc[Tr::G][8];  // unnormalised output chunk, rows r (mod R) of this lane
  float m;              // running max of this lane's head (base-2 logits)
  float l;              // running exp-sum of this lane's head
};

// Consumes one block (K and V chunks in shared memory): `valid` leading
// tokens of it belong to the sequence.
template <class Tr, bool kFull>
__device__ __forceinline__ void process_block(WarpState<Tr>& st, const typename Tr::KT* kch,
                                              const typename Tr::KT* vch, int valid, float* pbuf,
                                              int& buf, int lane) {
  constexpr int NC = Tr::NC, R = Tr::R, JS = Tr::JS, TS = Tr::TS, NV = Tr::NV, G = Tr::G;
  const int c = lane & (NC - 1);
  const int r0 = lane >> Tr::LOG2_NC;
  const int li = (lane & (NC - 1)) / Tr::REP;  // logit index held after the reduce
  const int lg = li / JS;                      // its head
  const int lj = li % JS;                      // its row within the lane's rows
  const int ltok = r0 + R * lj;                // its token within the sub-tile
#pragma unroll
  for (int sub = 0; sub < Tr::NSUB; ++sub) {
    const int tb = sub * TS;
    if (!kFull && tb >= valid) break;
    // ---- q . K for TS tokens --------------------------------------------
    float part[NV];
#pragma unroll
    for (int j = 0; j < JS; ++j) {
      const int row = tb + r0 + R * j;
      float kf[8];
      load_row8<typename Tr::KV>(kch + row * Tr::D + c * 8, kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float s = st.q[g][0] * kf[0];
#pragma unroll
        for (int e = 1; e < 8; ++e) s = fmaf(st.q[g][e], kf[e], s);
        part[g * JS + j] = s;
      }
    }
    float x = reduce_scatter<NV, NC>(part, lane);
    const bool in_seq = kFull || (tb + ltok) < valid;
    x = in_seq ? x : -INFINITY;
    // ---- online softmax update of this lane's head ----------------------
    const float m_new = fmaxf(st.m, segment_max<Tr>(x));
    const float alpha = exp2_approx(st.m - m_new);
    const float p = in_seq ? exp2_approx(x - m_new) : 0.f;
    st.l = st.l * alpha + segment_sum<Tr>(p);
    st.m = m_new;
    float* pb = pbuf + buf * Tr::PB_FLOATS;
    if ((lane & (Tr::REP - 1)) == 0) {
      pb[r0 * NV + li] = p;
      if (r0 == 0 && lj == 0) pb[R * NV + lg] = alpha;
    }
    __syncwarp();
    // ---- P . V ------------------------------------------------------------
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float a = pb[R * NV + g];
      if (a != 1.f) {
#pragma unroll
        for (int e = 0; e < 8; ++e) st.acc[g][e] *= a;
      }
    }
    float pv[NV];
#pragma unroll
    for (int k = 0; k < NV; k += 4) {
      const float4 f = *reinterpret_cast<const float4*>(pb + r0 * NV + k);
      pv[k] = f.x;
      pv[k + 1] = f.y;
      pv[k + 2] = f.z;
      pv[k + 3] = f.w;
    }
#pragma unroll
    for (int j = 0; j < JS; ++j) {
      const int row = tb + r0 + R * j;
      if (kFull || row < valid) {
        float vf[8];
        load_row8<typename Tr::KV>(vch + row * Tr::D + c * 8, vf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pg = pv[g * JS + j];
#pragma unroll
          for (int e = 0; e < 8; ++e) st.acc[g][e] = fmaf(pg, vf[e], st.acc[g][e]);
        }
      }
    }
    buf ^= 1;
  }
}

// Merges the W warps' (max, sum, unnormalised output) of one CTA and stores
// the result: the normalised output when the sequence has one partition,
// else the partition's (m, l, o) triple in the workspace.
//   cm, cl: [W][G] per-warp running max and exp-sum (base-2 logits)
//   cacc:   [W][G][D] per-warp unnormalised outputs
template <int W, int G, int D, class DT>
__device__ __forceinline__ void merge_warps_and_store(const DecodeParams& p, const float* cm,
                                                      const float* cl, const float* cacc,
                                                      int seq, int kvh, int part, bool direct) {
  using T = typename DT::T;
  constexpr int NC = D / 8;
  for (int idx = threadIdx.x; idx < G * NC; idx += W * 32) {
    const int g = idx / NC;
    const int cc = idx % NC;
    float big_m = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) big_m = fmaxf(big_m, cm[w * G + g]);
    float num[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float den = 0.f;
    if (big_m != -INFINITY) {
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const float f = exp2_approx(cm[w * G + g] - big_m);
        den = fmaf(f, cl[w * G + g], den);
        const float* a = cacc + (w * G + g) * D + cc * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) num[e] = fmaf(f, a[e], num[e]);
      }
    }
    const int head = kvh * G + g;
    if (p.v_scales != nullptr) {
      const float vs = p.v_scales[kvh];
#pragma unroll
      for (int e = 0; e < 8; ++e) num[e] *= vs;
    }
    if (direct) {
      const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) num[e] *= inv;
      T* o = static_cast<T*>(p.out) + (static_cast<size_t>(seq) * p.num_heads + head) * D + cc * 8;
      *reinterpret_cast<uint4*>(o) = pack8(num, DT());
    } else {
      const size_t slot = (static_cast<size_t>(seq) * p.num_heads + head) * p.max_parts + part +
                          (p.group_start != nullptr ? 1 : 0);
      float4* o = reinterpret_cast<float4*>(p.ws_out + slot * D + cc * 8);
      o[0] = make_float4(num[0], num[1], num[2], num[3]);
      o[1] = make_float4(num[4], num[5], num[6], num[7]);
      if (cc == 0) {
        p.ws_max[slot] = big_m;
        p.ws_sum[slot] = den;
      }
    }
  }
}

template <class Tr>
__global__ void __launch_bounds__(Tr::THREADS) paged_decode_kernel(const DecodeParams p) {
  using T = typename Tr::T;
  using KT = typename Tr::KT;
  constexpr int W = Tr::W, NS = Tr::NS, G = Tr::G, D = Tr::D, BS = Tr::BS, NC = Tr::NC;
  extern __shared__ __align__(128) unsigned char smem[];
  KT* ring = reinterpret_cast<KT*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tr::RING_BYTES);
  float* pbuf_all = reinterpret_cast<float*>(smem + Tr::RING_BYTES + Tr::BAR_BYTES);
  int* tbl = reinterpret_cast<int*>(smem + Tr::RING_BYTES + Tr::BAR_BYTES + Tr::PBUF_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Inputs may come from the previous kernel in the stream (e.g. the cache
  // write); wait for it before reading anything, then let the next one start.
  if (!p.independent_of_prior) grid_dependency_wait();
  trigger_dependents();
  const DecodeCta cta = decode_cta(p);
  const int seq = cta.seq, kvh = cta.kvh, part = cta.part;
  if (static_cast<unsigned>(seq) >= static_cast<unsigned>(p.num_seqs)) {
    if (threadIdx.x == 0) set_err(p.err, PKV_DEVERR_BAD_ORDER);
    return;
  }

  // Everything below depends only on the sequence: the context length, q
  // and (without cascade) the partition's table slice, which starts at
  // part * part_blocks whatever the length.  Their loads are issued together
  // so that their latencies overlap; table entries past the context are
  // never used.  Under cascade the slice starts after the group's shared
  // blocks and is staged once those are known.
  const int ctx_cap = min(p.max_context_len, p.max_blocks_per_seq * BS);
  int ctx = p.context_lens[seq];
  const int c = lane & (NC - 1);
  uint4 qraw[G];
  {
    const T* qrow = static_cast<const T*>(p.q) +
                    (static_cast<size_t>(seq) * p.num_heads + kvh * G) * D + c * 8;
#pragma unroll
    for (int g = 0; g < G; ++g) qraw[g] = *reinterpret_cast<const uint4*>(qrow + g * D);
  }
  const bool cascade = p.group_start != nullptr;
  const int32_t* seq_row = p.block_tables + static_cast<size_t>(seq) * p.max_blocks_per_seq;
  if (!cascade) {
    const int b0 = part * p.part_blocks;
    const int n0 = min(p.part_blocks, p.max_blocks_per_seq - b0);
    for (int i = threadIdx.x; i < n0; i += Tr::THREADS) tbl[i] = seq_row[b0 + i];
  }
  if (ctx < 0 || ctx > ctx_cap) {
    if (threadIdx.x == 0 && part == 0 && kvh == 0) set_err(p.err, PKV_DEVERR_BAD_CONTEXT);
    ctx = min(max(ctx, 0), ctx_cap);
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int start_blk =
      cascade_start_block(p, seq, nblk, threadIdx.x == 0 && part == 0 && kvh == 0);
  const int nparts = (nblk - start_blk + p.part_blocks - 1) / p.part_blocks;
  if (threadIdx.x == 0 && plan_mismatch(p, cta, nparts)) set_err(p.err, PKV_DEVERR_BAD_ORDER);
  if (part >= (cascade ? nparts : max(nparts, 1))) return;
  const bool direct = !cascade && nparts <= 1;
  const int blk_begin = start_blk + part * p.part_blocks;
  const int nb = min(nblk, blk_begin + p.part_blocks) - blk_begin;

  // ---- under cascade, stage the block-table slice; initialise this warp's barriers
  if (cascade) {
    for (int i = threadIdx.x; i < nb; i += Tr::THREADS) tbl[i] = seq_row[blk_begin + i];
  }
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < NS; ++s) mbar_init(smem_addr(bars + warp * NS + s), 1);
    fence_mbar_init();
  }
  __syncthreads();

  // ---- this lane's q chunk for the G heads, pre-scaled ---------------------
  // (an 8-bit cache's K scale folds into the q pre-scale: q.(code*s) = (s*q).code)
  float qscale = p.qscale;
  if (p.k_scales != nullptr) {
    const float ks = p.k_scales[kvh];
    const float vs = p.v_scales[kvh];
    if (!(ks > 0.f && ks < INFINITY && vs > 0.f && vs < INFINITY) && threadIdx.x == 0 &&
        part == 0)
      set_err(p.err, PKV_DEVERR_BAD_SCALE);
    qscale *= ks;
  }
  WarpState<Tr> st;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    unpack8(qraw[g], st.q[g], typename Tr::DT());
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      st.q[g][e] *= qscale;
      st.acc[g][e] = 0.f;
    }
  }
  st.m = -INFINITY;
  st.l = 0.f;

  // ---- stream this warp's blocks through its ring ---------------------------
  const int nbw = nb > warp ? (nb - warp + W - 1) / W : 0;
  KT* wring = ring + static_cast<size_t>(warp) * NS * 2 * Tr::CHUNK_ELEMS;
  const uint32_t bar0 = smem_addr(bars + warp * NS);
  const KT* kbase = static_cast<const KT*>(p.k_cache);
  const KT* vbase = static_cast<const KT*>(p.v_cache);
  const size_t head_off = static_cast<size_t>(kvh) * Tr::CHUNK_ELEMS;
  const size_t block_stride = static_cast<size_t>(p.num_kv_heads) * Tr::CHUNK_ELEMS;

  auto issue = [&](int k) {  // lane 0 only
    if (p.withhold_first_load && blockIdx.x == 0 && warp == 0 && k == 0) return;
    const int stage = k % NS;
    const int pb = tbl[warp + k * W];
    const uint32_t bar = bar0 + stage * 8;
    if (static_cast<unsigned>(pb) < static_cast<unsigned>(p.num_blocks)) {
      const size_t off = static_cast<size_t>(pb) * block_stride + head_off;
      mbar_arrive_expect_tx(bar, 2 * Tr::CHUNK_BYTES);
      bulk_copy_g2s(smem_addr(wring + (2 * stage) * Tr::CHUNK_ELEMS), kbase + off,
                    Tr::CHUNK_BYTES, bar);
      bulk_copy_g2s(smem_addr(wring + (2 * stage + 1) * Tr::CHUNK_ELEMS), vbase + off,
                    Tr::CHUNK_BYTES, bar);
    } else {
      set_err(p.err, PKV_DEVERR_BAD_BLOCK);
      mbar_arrive(bar);  // complete the phase with no data; consumers skip it
    }
  };

  if (lane == 0) {
    for (int k = 0; k < min(NS, nbw); ++k) issue(k);
  }
  float* pbuf = pbuf_all + warp * 2 * Tr::PB_FLOATS;
  int buf = 0;
  for (int k = 0; k < nbw; ++k) {
    const int stage = k % NS;
    const bool ok = mbar_wait_bounded(bar0 + stage * 8, (k / NS) & 1, p.wait_ns);
    if (!__all_sync(kFullMask, ok)) {
      // Give up on this warp's blocks: report, then wait (bounded) for the
      // copies still in flight so none lands after the CTA has exited.
      if (lane == 0) {
        set_err(p.err, PKV_DEVERR_TIMEOUT);
        for (int j = k; j < min(k + NS, nbw); ++j)
          (void)mbar_wait_bounded(bar0 + (j % NS) * 8, (j / NS) & 1);
      }
      __syncwarp();
      break;
    }
    const int pb = tbl[warp + k * W];
    if (static_cast<unsigned>(pb) < static_cast<unsigned>(p.num_blocks)) {
      const KT* kch = wring + (2 * stage) * Tr::CHUNK_ELEMS;
      const KT* vch = kch + Tr::CHUNK_ELEMS;
      const int lb = blk_begin + warp + k * W;
      const int valid = min(BS, ctx - lb * BS);
      if (valid == BS)
        process_block<Tr, true>(st, kch, vch, BS, pbuf, buf, lane);
      else
        process_block<Tr, false>(st, kch, vch, valid, pbuf, buf, lane);
    }
    __syncwarp();
    if (lane == 0 && k + NS < nbw) {
      fence_proxy_async_smem();  // the warp's reads of this stage precede the refill
      issue(k + NS);
    }
  }

  // ---- merge the row groups, then the warps ---------------------------------
#pragma unroll
  for (int m = NC; m < 32; m <<= 1)
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < 8; ++e) st.acc[g][e] += __shfl_xor_sync(kFullMask, st.acc[g][e], m);

  __syncthreads();  // every warp is done with the ring; reuse it
  float* cm = reinterpret_cast<float*>(smem);  // [W][G]
  float* cl = cm + W * G;                      // [W][G]
  float* cacc = cl + W * G;                    // [W][G][D]
  {
    const int li = (lane & (NC - 1)) / Tr::REP;
    const int r0 = lane >> Tr::LOG2_NC;
    if ((lane & (Tr::REP - 1)) == 0 && r0 == 0 && li % Tr::JS == 0) {
      cm[warp * G + li / Tr::JS] = st.m;
      cl[warp * G + li / Tr::JS] = st.l;
    }
    if (r0 == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float4* dst = reinterpret_cast<float4*>(cacc + (warp * G + g) * D + c * 8);
        dst[0] = make_float4(st.acc[g][0], st.acc[g][1], st.acc[g][2], st.acc[g][3]);
        dst[1] = make_float4(st.acc[g][4], st.acc[g][5], st.acc[g][6], st.acc[g][7]);
      }
    }
  }
  __syncthreads();
  merge_warps_and_store<W, G, D, typename Tr::DT>(p, cm, cl, cacc, seq, kvh, part, direct);
}

// ---------------------------------------------------------------------------
// Grouped-query decode on the tensor cores (G >= 2; with an E4M3 cache every G,
// see mma_sub_block_fp8).
//
// With G query heads per kv head, q.K and P.V carry G multiply-adds per
// cached element; on the CUDA cores that makes the kernel instruction-bound
// (about 1,700 warp instructions per 16 tokens at G = 8).  Here each warp runs
// them as mma.sync m16n8k16 with the 16 tokens of a sub-block as M and the
// heads as N (N = 8 covers G <= 8 with no padding at G = 8):
//   q.K:  S^T[t][n] = sum_d K[t][d] q[n][d]      A = K   (ldmatrix)
//   P.V:  O^T[d][n] += sum_t V[t][d] P[n][t]     A = V^T (ldmatrix.trans),
//                                                B = P, transposed in registers
//                                                from the S^T accumulator by movmatrix
// K and V of a (block, kv head) reach shared memory by 2-D tiled TMA loads
// with the 128-byte swizzle: boxes of 16 rows x 64 elements, so ldmatrix rows
// fall in distinct banks.  A stage is one 16-token sub-block (a block of 32
// is two stages).  The ring, the table slice, the bounded waits, the split-K
// partitions and the final merge are as in paged_decode_kernel.
// ---------------------------------------------------------------------------
template <int D_, int BS_, int G_, class DT_, int W_, int NS_, class KV_ = DT_>
struct MmaTraits {
  static constexpr int D = D_, BS = BS_, G = G_, W = W_, NS = NS_;
  using DT = DT_;
  using T = typename DT::T;
  using KV = KV_;
  static constexpr bool kFp8 = std::is_same<KV, Fp8E4M3>::value;
  static constexpr int SUB = 16;                   // tokens per stage (the mma M)
  static constexpr int SUBS_PER_BLOCK = BS / SUB;
  static constexpr int ROW_BYTES = D * (kFp8 ? 1 : 2);
  static constexpr int BOXES = ROW_BYTES / 128;    // 128-byte-wide boxes per row
  static constexpr int BOX_BYTES = SUB * 128;      // one 16-row x 128-byte box
  static constexpr int TILE_BYTES = BOXES * BOX_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K tile + V tile
  static constexpr int KSTEPS = D / 16;            // q.K k-steps = P.V m-tiles
  static constexpr int THREADS = W * 32;
  static constexpr int RING_BYTES = W * NS * STAGE_BYTES;
  static constexpr int BAR_BYTES = W * NS * 8;
  static constexpr int COMBINE_BYTES = W * G * (D + 2) * 4;
  static_assert(G >= (kFp8 ? 1 : 2) && G <= 8, "tensor-core path: up to 8 heads per kv head");
  static_assert(BS % SUB == 0 && D % 64 == 0 && ROW_BYTES % 128 == 0, "shape");
  static_assert(COMBINE_BYTES <= RING_BYTES, "combine scratch reuses the ring");
  static size_t smem_bytes(int part_blocks) {
    return 1024 + static_cast<size_t>(RING_BYTES) + BAR_BYTES +
           static_cast<size_t>(part_blocks) * 4;
  }
};

// Byte offset of 16-byte chunk `ch` of row `t` in a tile of BOXES swizzled
// 16 x 128-byte boxes (chunk index XOR row % 8, per 1024-byte swizzle atom).
__device__ __forceinline__ uint32_t swizzled(int t, int ch) {
  return static_cast<uint32_t>((ch >> 3) * 2048 + t * 128 + (((ch & 7) ^ (t & 7)) << 4));
}

// The reference max of the tensor-core kernels' online softmax moves only
// when a logit exceeds it by more than this (base-2 units), so P stays at
// most 2^8 (fp16 and bf16 hold it) and most sub-blocks skip the max and its
// shuffles.
constexpr float kLazyMax = 8.f;

// Online softmax of one 16-token sub-block for the two heads a lane holds in
// the S^T fragment (x0, x2: head 2(lane % 4) at tokens lane / 4 and
// lane / 4 + 8; x1, x3: head 2(lane % 4) + 1).  m[] is the reference max, the
// same in the 8 lanes that share lane % 4; it is recomputed (a max over those
// lanes, the O accumulator and l rescaled) only when a logit passes
// m + kLazyMax.  l[] holds this lane's own partial sums, reduced over the 8
// lanes once at the end.  Returns p = 2^(x - m).
template <int KS>
__device__ __forceinline__ void mma_softmax(float x0, float x1, float x2, float x3,
                                            float (&m)[2], float (&l)[2], float (&acc)[KS][4],
                                            float& p0, float& p1, float& p2, float& p3) {
  const bool up = x0 > m[0] + kLazyMax || x2 > m[0] + kLazyMax || x1 > m[1] + kLazyMax ||
                  x3 > m[1] + kLazyMax;
  if (__any_sync(kFullMask, up)) {
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(kFullMask, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(kFullMask, mx1, o));
    }
    const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
    const float a0 = exp2_approx(m[0] - mn0), a1 = exp2_approx(m[1] - mn1);
    m[0] = mn0;
    m[1] = mn1;
    l[0] *= a0;
    l[1] *= a1;
    if (__any_sync(kFullMask, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        acc[mt][0] *= a0;
        acc[mt][1] *= a1;
        acc[mt][2] *= a0;
        acc[mt][3] *= a1;
      }
    }
  }
  p0 = exp2_approx(x0 - m[0]);
  p1 = exp2_approx(x1 - m[1]);
  p2 = exp2_approx(x2 - m[0]);
  p3 = exp2_approx(x3 - m[1]);
  l[0] += p0 + p2;
  l[1] += p1 + p3;
}

template <class Tr>
__device__ __forceinline__ void mma_sub_block(uint32_t kt, uint32_t vt, int valid,
                                              const uint32_t (&qf)[Tr::KSTEPS][2],
                                              float (&acc)[Tr::KSTEPS][4], float (&m)[2],
                                              float (&l)[2], float qscale, int lane) {
  constexpr int KS = Tr::KSTEPS;
  const int j = lane >> 3;  // which 8x8 matrix this lane addresses
  const int r = lane & 7;
  // ---- q.K: S^T (16 tokens x 8 heads) ----------------------------------------
  float s[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const int t = ((j & 1) << 3) + r;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a[4];
      ldsm_x4(kt + swizzled(t, 2 * ks + (j >> 1)), a);
      mma_16816(s, a, qf[ks][0], qf[ks][1], typename Tr::DT());
    }
  }
  // lane holds tokens t0 = lane/4 and t0 + 8, heads 2(lane%4) and 2(lane%4)+1
  const int t0 = lane >> 2;
  float x0 = s[0] * qscale, x1 = s[1] * qscale, x2 = s[2] * qscale, x3 = s[3] * qscale;
  if (valid < Tr::SUB) {
    if (t0 >= valid) x0 = x1 = -INFINITY;
    if (t0 + 8 >= valid) x2 = x3 = -INFINITY;
  }
  // ---- online softmax per head (see mma_softmax) ---------------------------------
  float p0, p1, p2, p3;
  mma_softmax<KS>(x0, x1, x2, x3, m, l, acc, p0, p1, p2, p3);
  // ---- P as the B operand: transpose the S^T fragments in registers -----------
  // bf16 keeps 8 mantissa bits, too few for p near 1 at the required accuracy,
  // so bf16 P is split as hi + lo (both bf16, |P - hi - lo| <= 2^-18 P) and
  // P.V runs twice; fp16 P (11 bits) is used as is.
  constexpr bool kSplitP = std::is_same<typename Tr::DT, Bf16>::value;
  const uint32_t h01 = pack2(p0, p1, typename Tr::DT());
  const uint32_t h23 = pack2(p2, p3, typename Tr::DT());
  const uint32_t b0 = movmatrix_trans(h01);
  const uint32_t b1 = movmatrix_trans(h23);
  uint32_t b0_lo = 0, b1_lo = 0;
  if constexpr (kSplitP) {
    b0_lo = movmatrix_trans(pack2(p0 - __uint_as_float(h01 << 16),
                                  p1 - __uint_as_float(h01 & 0xffff0000u), Bf16()));
    b1_lo = movmatrix_trans(pack2(p2 - __uint_as_float(h23 << 16),
                                  p3 - __uint_as_float(h23 & 0xffff0000u), Bf16()));
  }
  // ---- rows past the context hold stale data (maybe NaN): zero them in V so
  //      that 0 * V stays 0 inside the tensor-core sum
  if (valid < Tr::SUB) {
    const int chunks = (Tr::SUB - valid) * Tr::BOXES * 8;
    for (int i = lane; i < chunks; i += 32) {
      const int row = valid + i / (Tr::BOXES * 8);
      const int rem = i % (Tr::BOXES * 8);
      const uint32_t at = vt + (rem >> 3) * 2048 + row * 128 + ((rem & 7) << 4);
      asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(at), "r"(0u) : "memory");
    }
    __syncwarp();
  }
  // ---- P.V: O^T (D dims x 8 heads) -------------------------------------------
  {
    const int t = ((j >> 1) << 3) + r;
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
      uint32_t a[4];
      ldsm_x4_trans(vt + swizzled(t, 2 * mt + (j & 1)), a);
      mma_16816(acc[mt], a, b0, b1, typename Tr::DT());
      if constexpr (kSplitP) mma_16816(acc[mt], a, b0_lo, b1_lo, typename Tr::DT());
    }
  }
}

// Two E4M3 codes (a 16-bit half of x) -> fp16x2, exact.
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}

// The E4M3 form of mma_sub_block: the tile rows are 128 bytes of codes (one
// swizzled box), widened to fp16 in registers; the mma runs in fp16.
//   q.K: ldmatrix (16-bit lanes over byte pairs) gives lane (g, u) the codes of
//        dims 4u..4u+3 of a 16-dim chunk, so the mma's k order inside each
//        chunk is permuted (logical 2u+{0,1} = dims 4u+{0,1}, logical
//        8+2u+{0,1} = dims 4u+2+{0,1}); the q fragments use the same order.
//   P.V: lane (g, u) reads dims 16g..16g+15 of tokens 2u, 2u+1, 2u+8, 2u+9 and
//        pairs tokens with byte permutes; mma j covers dims 16g+2j (row g) and
//        16g+2j+1 (row g+8), so the lane's accumulators hold 16 consecutive dims.
// Returns nothing; updates acc / m / l like mma_sub_block.  x = s * qscale is
// the base-2 logit (qscale includes the kv head's K scale).
template <class Tr>
__device__ __forceinline__ void mma_sub_block_fp8(uint32_t kt, uint32_t vt, int valid,
                                                  const uint32_t (&qf)[Tr::KSTEPS][2],
                                                  float (&acc)[Tr::KSTEPS][4], float (&m)[2],
                                                  float (&l)[2], float qscale, int lane) {
  constexpr int KS = Tr::KSTEPS;
  const int j = lane >> 3;
  const int r = lane & 7;
  float s[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const int t = ((j & 1) << 3) + r;
#pragma unroll
    for (int cc = 0; cc < KS / 2; ++cc) {
      uint32_t w[4];
      ldsm_x4(kt + swizzled(t, 2 * cc + (j >> 1)), w);
      uint32_t a[4];
      e4m3x4_to_f16x2(w[0], a[0], a[2]);
      e4m3x4_to_f16x2(w[1], a[1], a[3]);
      mma_16816(s, a, qf[2 * cc][0], qf[2 * cc][1], Fp16());
      e4m3x4_to_f16x2(w[2], a[0], a[2]);
      e4m3x4_to_f16x2(w[3], a[1], a[3]);
      mma_16816(s, a, qf[2 * cc + 1][0], qf[2 * cc + 1][1], Fp16());
    }
  }
  const int t0 = lane >> 2;
  float x0 = s[0] * qscale, x1 = s[1] * qscale, x2 = s[2] * qscale, x3 = s[3] * qscale;
  if (valid < Tr::SUB) {
    if (t0 >= valid) x0 = x1 = -INFINITY;
    if (t0 + 8 >= valid) x2 = x3 = -INFINITY;
  }
  float p0, p1, p2, p3;
  mma_softmax<KS>(x0, x1, x2, x3, m, l, acc, p0, p1, p2, p3);
  // P in (0, 1] as fp16 (11 significant bits), transposed into the B operand
  const uint32_t b0 = movmatrix_trans(pack2(p0, p1, Fp16()));
  const uint32_t b1 = movmatrix_trans(pack2(p2, p3, Fp16()));
  // rows past the context hold stale codes (maybe NaN): zero them
  if (valid < Tr::SUB) {
    for (int i = lane; i < (Tr::SUB - valid) * 8; i += 32) {
      const uint32_t at = vt + (valid + i / 8) * 128 + ((i & 7) << 4);
      asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(at), "r"(0u) : "memory");
    }
    __syncwarp();
  }
  {
    const int g = lane >> 2, u = lane & 3;
    uint4 v[4];  // tokens 2u, 2u+1, 2u+8, 2u+9: dims 16g .. 16g+15
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tok = 2 * u + (i & 1) + ((i >> 1) << 3);
      const uint32_t at = vt + tok * 128 + ((g ^ (tok & 7)) << 4);
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(v[i].x), "=r"(v[i].y), "=r"(v[i].z), "=r"(v[i].w)
                   : "r"(at));
    }
    const uint32_t w0[4] = {v[0].x, v[0].y, v[0].z, v[0].w};
    const uint32_t w1[4] = {v[1].x, v[1].y, v[1].z, v[1].w};
    const uint32_t w8[4] = {v[2].x, v[2].y, v[2].z, v[2].w};
    const uint32_t w9[4] = {v[3].x, v[3].y, v[3].z, v[3].w};
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
      // bytes (tok a dim d, tok b dim d, tok a dim d+1, tok b dim d+1), d = 16g + 2mt
      const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
      const uint32_t lo = __byte_perm(w0[mt >> 1], w1[mt >> 1], sel);
      const uint32_t hi = __byte_perm(w8[mt >> 1], w9[mt >> 1], sel);
      uint32_t a[4];
      e4m3x4_to_f16x2(lo, a[0], a[1]);
      e4m3x4_to_f16x2(hi, a[2], a[3]);
      mma_16816(acc[mt], a, b0, b1, Fp16());
    }
  }
}

template <class Tr>
__global__ void __launch_bounds__(Tr::THREADS)
    paged_decode_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                            const __grid_constant__ CUtensorMap vmap) {
  using T = typename Tr::T;
  constexpr int W = Tr::W, NS = Tr::NS, G = Tr::G, D = Tr::D, BS = Tr::BS, KS = Tr::KSTEPS;
  constexpr int SPB = Tr::SUBS_PER_BLOCK;
  extern __shared__ unsigned char smem_raw[];
  // the 128-byte swizzle needs 1024-byte-aligned boxes
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tr::RING_BYTES);
  int* tbl = reinterpret_cast<int*>(smem + Tr::RING_BYTES + Tr::BAR_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (!p.independent_of_prior) grid_dependency_wait();
  trigger_dependents();
  const DecodeCta cta = decode_cta(p);
  const int seq = cta.seq, kvh = cta.kvh, part = cta.part;
  if (static_cast<unsigned>(seq) >= static_cast<unsigned>(p.num_seqs)) {
    if (threadIdx.x == 0) set_err(p.err, PKV_DEVERR_BAD_ORDER);
    return;
  }

  // Over E4M3 the context length and (without cascade) the partition's
  // table slice, which starts at part * part_blocks whatever the length, are
  // loaded together so that their latencies overlap; entries past the
  // context are never used.  Otherwise (16-bit caches, where staging whole
  // one-pass slices measured slower, or under cascade, where the slice
  // starts after the group's shared blocks) the slice is staged once the
  // length is known.
  const int ctx_cap = min(p.max_context_len, p.max_blocks_per_seq * BS);
  int ctx = p.context_lens[seq];
  const bool cascade = p.group_start != nullptr;
  const bool early_table = Tr::kFp8 && !cascade;
  const int32_t* seq_row = p.block_tables + static_cast<size_t>(seq) * p.max_blocks_per_seq;
  if (early_table) {
    const int b0 = part * p.part_blocks;
    const int n0 = min(p.part_blocks, p.max_blocks_per_seq - b0);
    for (int i = threadIdx.x; i < n0; i += Tr::THREADS) tbl[i] = seq_row[b0 + i];
  }
  if (ctx < 0 || ctx > ctx_cap) {
    if (threadIdx.x == 0 && part == 0 && kvh == 0) set_err(p.err, PKV_DEVERR_BAD_CONTEXT);
    ctx = min(max(ctx, 0), ctx_cap);
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int start_blk =
      cascade_start_block(p, seq, nblk, threadIdx.x == 0 && part == 0 && kvh == 0);
  const int nparts = (nblk - start_blk + p.part_blocks - 1) / p.part_blocks;
  if (threadIdx.x == 0 && plan_mismatch(p, cta, nparts)) set_err(p.err, PKV_DEVERR_BAD_ORDER);
  if (part >= (cascade ? nparts : max(nparts, 1))) return;
  const bool direct = !cascade && nparts <= 1;
  const int blk_begin = start_blk + part * p.part_blocks;
  const int nb = min(nblk, blk_begin + p.part_blocks) - blk_begin;
  const int sb_begin = blk_begin * SPB;
  const int nsb = max(0, min((ctx + Tr::SUB - 1) / Tr::SUB, (blk_begin + nb) * SPB) - sb_begin);

  if (!early_table) {
    for (int i = threadIdx.x; i < nb; i += Tr::THREADS) tbl[i] = seq_row[blk_begin + i];
  }
  // q as mma B fragments: lane holds head lane/4, dims 16ks + 2(lane%4) +
  // {0,1,8,9} (E4M3 cache: dims 16ks + 4(lane%4) + {0,1,2,3}, the permuted k
  // order of mma_sub_block_fp8, as fp16).  Over 16-bit caches they load
  // after the barrier; over E4M3 after the first K/V loads are issued, since
  // the bf16 -> fp16 conversion and the scale check wait for them.
  uint32_t qf[KS][2];
  float qscale = p.qscale;
  auto load_q = [&]() {
    const int n = lane >> 2;
    const int c = lane & 3;
    const T* qrow = static_cast<const T*>(p.q) +
                    (static_cast<size_t>(seq) * p.num_heads + kvh * G + min(n, G - 1)) * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      if constexpr (Tr::kFp8) {
        uint2 u = n < G ? *reinterpret_cast<const uint2*>(qrow + 16 * ks + 4 * c) : make_uint2(0, 0);
        if constexpr (std::is_same<typename Tr::DT, Bf16>::value) {
          // bf16 -> fp16 for the fp16 mma; magnitudes beyond fp16 saturate
          auto cv = [](uint32_t w) {
            const float lo = fminf(fmaxf(__uint_as_float(w << 16), -65504.f), 65504.f);
            const float hi = fminf(fmaxf(__uint_as_float(w & 0xffff0000u), -65504.f), 65504.f);
            return pack2(lo, hi, Fp16());
          };
          u = make_uint2(cv(u.x), cv(u.y));
        }
        qf[ks][0] = u.x;
        qf[ks][1] = u.y;
      } else {
        qf[ks][0] = n < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * c) : 0u;
        qf[ks][1] = n < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * c) : 0u;
      }
    }
    if constexpr (Tr::kFp8) {
      const float ks = p.k_scales[kvh];
      const float vs = p.v_scales[kvh];
      if (!(ks > 0.f && ks < INFINITY && vs > 0.f && vs < INFINITY) && threadIdx.x == 0 &&
          part == 0)
        set_err(p.err, PKV_DEVERR_BAD_SCALE);
      qscale *= ks;
    }
  };
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < NS; ++s) mbar_init(smem_addr(bars + warp * NS + s), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if constexpr (!Tr::kFp8) load_q();

  float acc[KS][4];
#pragma unroll
  for (int mt = 0; mt < KS; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY};
  float l[2] = {0.f, 0.f};

  const int nbw = nsb > warp ? (nsb - warp + W - 1) / W : 0;
  const uint32_t ring0 = smem_addr(smem) + warp * NS * Tr::STAGE_BYTES;
  const uint32_t bar0 = smem_addr(bars + warp * NS);

  auto table_entry = [&](int k) {  // physical block of this warp's k-th sub-block
    const int sb = sb_begin + warp + k * W;
    return tbl[sb / SPB - blk_begin];
  };
  auto issue = [&](int k) {  // lane 0 only
    if (p.withhold_first_load && blockIdx.x == 0 && warp == 0 && k == 0) return;
    const int stage = k % NS;
    const int sb = sb_begin + warp + k * W;
    const int pb = tbl[sb / SPB - blk_begin];
    const uint32_t bar = bar0 + stage * 8;
    if (static_cast<unsigned>(pb) < static_cast<unsigned>(p.num_blocks)) {
      const int y = (pb * p.num_kv_heads + kvh) * BS + (sb % SPB) * Tr::SUB;
      const uint32_t kdst = ring0 + stage * Tr::STAGE_BYTES;
      mbar_arrive_expect_tx(bar, Tr::STAGE_BYTES);
#pragma unroll
      for (int b = 0; b < Tr::BOXES; ++b) {
        tma_load_2d(kdst + b * Tr::BOX_BYTES, &kmap, b * 64, y, bar);
        tma_load_2d(kdst + Tr::TILE_BYTES + b * Tr::BOX_BYTES, &vmap, b * 64, y, bar);
      }
    } else {
      set_err(p.err, PKV_DEVERR_BAD_BLOCK);
      mbar_arrive(bar);
    }
  };

  if (lane == 0) {
    for (int k = 0; k < min(NS, nbw); ++k) issue(k);
  }
  if constexpr (Tr::kFp8) load_q();
  for (int k = 0; k < nbw; ++k) {
    const int stage = k % NS;
    const bool ok = mbar_wait_bounded(bar0 + stage * 8, (k / NS) & 1, p.wait_ns);
    if (!__all_sync(kFullMask, ok)) {
      if (lane == 0) {
        set_err(p.err, PKV_DEVERR_TIMEOUT);
        for (int jj = k; jj < min(k + NS, nbw); ++jj)
          (void)mbar_wait_bounded(bar0 + (jj % NS) * 8, (jj / NS) & 1);
      }
      __syncwarp();
      break;
    }
    const int pb = table_entry(k);
    if (static_cast<unsigned>(pb) < static_cast<unsigned>(p.num_blocks)) {
      const int sb = sb_begin + warp + k * W;
      const int valid = min(Tr::SUB, ctx - sb * Tr::SUB);
      const uint32_t kt = ring0 + stage * Tr::STAGE_BYTES;
      if constexpr (Tr::kFp8)
        mma_sub_block_fp8<Tr>(kt, kt + Tr::TILE_BYTES, valid, qf, acc, m, l, qscale, lane);
      else
        mma_sub_block<Tr>(kt, kt + Tr::TILE_BYTES, valid, qf, acc, m, l, qscale, lane);
    }
    __syncwarp();
    if (lane == 0 && k + NS < nbw) {
      fence_proxy_async_smem();
      issue(k + NS);
    }
  }

  // ---- merge the warps -------------------------------------------------------
  // each lane summed its own p: the sums of a head pair over its 8 lanes
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l[0] += __shfl_xor_sync(kFullMask, l[0], o);
    l[1] += __shfl_xor_sync(kFullMask, l[1], o);
  }
  __syncthreads();
  float* cm = reinterpret_cast<float*>(smem);
  float* cl = cm + W * G;
  float* cacc = cl + W * G;
  {
    const int c = lane & 3;
    const int d_lo = lane >> 2;
    if (lane < 4) {
      if (2 * c < G) {
        cm[warp * G + 2 * c] = m[0];
        cl[warp * G + 2 * c] = l[0];
      }
      if (2 * c + 1 < G) {
        cm[warp * G + 2 * c + 1] = m[1];
        cl[warp * G + 2 * c + 1] = l[1];
      }
    }
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
      // rows g and g+8 of mma mt: dims 16mt + g and +8 (E4M3: 16g + 2mt and +1)
      const int d = Tr::kFp8 ? 16 * d_lo + 2 * mt : 16 * mt + d_lo;
      const int d2 = Tr::kFp8 ? d + 1 : d + 8;
      if (2 * c < G) {
        cacc[(warp * G + 2 * c) * D + d] = acc[mt][0];
        cacc[(warp * G + 2 * c) * D + d2] = acc[mt][2];
      }
      if (2 * c + 1 < G) {
        cacc[(warp * G + 2 * c + 1) * D + d] = acc[mt][1];
        cacc[(warp * G + 2 * c + 1) * D + d2] = acc[mt][3];
      }
    }
  }
  __syncthreads();
  merge_warps_and_store<W, G, D, typename Tr::DT>(p, cm, cl, cacc, seq, kvh, part, direct);
}

// Context length as the kernels use it: negative or oversized values are
// clamped (and reported by the partition kernel).
__device__ __forceinline__ int clamped_context(const DecodeParams& p, int seq) {
  const int cap = min(p.max_context_len, p.max_blocks_per_seq * p.block_size);
  return min(max(p.context_lens[seq], 0), cap);
}

// Merges the partitions of each (sequence, head): M = max_p m_p,
// out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.  One warp per
// (sequence, head); sequences with a single partition were written directly
// by the partition kernel and are skipped here.
template <int D, class DT>
__global__ void __launch_bounds__(128) paged_decode_reduce_kernel(const DecodeParams p) {
  using T = typename DT::T;
  constexpr int PER_LANE = D / 32;
  grid_dependency_wait();
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= p.num_seqs * p.num_heads) return;
  const int seq = gw / p.num_heads;
  const int head = gw % p.num_heads;
  const int ctx = clamped_context(p, seq);
  const int nblk = (ctx + p.block_size - 1) / p.block_size;
  const bool cascade = p.group_start != nullptr;
  const int start_blk = cascade_start_block(p, seq, nblk, false);
  const int nsuffix = (nblk - start_blk + p.part_blocks - 1) / p.part_blocks;
  // slots [first, last): the prefix partial (slot 0, cascade only) and the suffix partitions
  const int first = cascade && start_blk == 0 ? 1 : 0;
  const int last = cascade ? 1 + nsuffix : nsuffix;
  if (!cascade && nsuffix <= 1) return;
  const size_t base = static_cast<size_t>(gw) * p.max_parts;
  float big_m = -INFINITY;
  for (int q = first + lane; q < last; q += 32) big_m = fmaxf(big_m, p.ws_max[base + q]);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) big_m = fmaxf(big_m, __shfl_xor_sync(kFullMask, big_m, m));
  float num[PER_LANE];
#pragma unroll
  for (int e = 0; e < PER_LANE; ++e) num[e] = 0.f;
  float den = 0.f;
#pragma unroll 4
  for (int q = first; q < last; ++q) {
    const float f = exp2_approx(p.ws_max[base + q] - big_m);
    den = fmaf(f, p.ws_sum[base + q], den);
    const float* o = p.ws_out + (base + q) * D + lane * PER_LANE;
    if constexpr (PER_LANE == 4) {
      const float4 v = *reinterpret_cast<const float4*>(o);
      num[0] = fmaf(f, v.x, num[0]);
      num[1] = fmaf(f, v.y, num[1]);
      num[2] = fmaf(f, v.z, num[2]);
      num[3] = fmaf(f, v.w, num[3]);
    } else {
      const float2 v = *reinterpret_cast<const float2*>(o);
      num[0] = fmaf(f, v.x, num[0]);
      num[1] = fmaf(f, v.y, num[1]);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  T* out = static_cast<T*>(p.out) + static_cast<size_t>(gw) * D + lane * PER_LANE;
  T vals[PER_LANE];
#pragma unroll
  for (int e = 0; e < PER_LANE; ++e) vals[e] = static_cast<T>(num[e] * inv);
  if constexpr (PER_LANE == 4)
    *reinterpret_cast<uint2*>(out) = *reinterpret_cast<const uint2*>(vals);
  else
    *reinterpret_cast<uint32_t*>(out) = *reinterpret_cast<const uint32_t*>(vals);
  (void)seq;
  (void)head;
}

}  // namespace pkv
