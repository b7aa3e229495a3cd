// paged_prefill_kernels.cuh — chunked-prefill attention over the paged KV
// cache for B200 (sm_100a).
//
// What it computes.  Sequence i appends q_len_i tokens in this step; their
// K/V are already in the cache (written by reshape_and_cache), so the
// sequence caches C_i tokens and its j-th new token sits at position
// p = C_i - q_len_i + j.  That token's query attends causally to tokens 0..p,
// gathered through the block table like decode does ([csdn] "分页式KV缓存";
// [betteryeah] §2.2, §2.4): out = softmax(scale * q . K[0..p]^T) . V[0..p].
//
// How.  One CTA per (sequence, kv head, tile of 64 query rows), a row being a
// (new token, query head of this kv head) pair.  Four consumer warps own 16
// rows each and run FlashAttention-style on the tensor cores:
//   S = Q K^T   mma.sync m16n8k16, rows x 16 keys (two n-tiles), K by ldmatrix
//   P = online softmax of S (base 2), straight from the S accumulator layout
//   O += P V    V by ldmatrix.trans, D/8 n-tiles
// A fifth warp produces: it streams the sequence's keys 16 at a time into a
// ring of NS stages (2-D tiled TMA with the 128-byte swizzle, one full and one
// empty mbarrier per stage) and reads the block table 32 entries at a time.
// Every wait is bounded.  Causal masking uses -inf before the max; keys past
// the context are zeroed in the V fragments so stale NaN never enters a sum.
#pragma once

#include <math.h>

#include <type_traits>

#include "common.cuh"

namespace pkv {

struct PrefillParams {
  void* out;  // [T, H, D]
  const void* q;  // [T, H, D]
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start;  // [S + 1]
  float qscale;  // scale * log2(e)
  int num_seqs;
  int num_heads;
  int num_kv_heads;
  int max_blocks_per_seq;
  int max_context_len;
  int max_query_len;
  int num_blocks;
  int q_tiles;  // query tiles per (sequence, kv head) at max_query_len
  unsigned* err;
  // E4M3 caches (tcgen05 kernel): per-kv-head scales, value = code x scale
  const float* k_scales;  // [num_kv_heads]
  const float* v_scales;  // [num_kv_heads]
  // Shared-prefix pass of cascade decode (tcgen05 kernel in prefix mode): the
  // units are groups of sequences instead of sequences, the queries are the
  // members' decode queries, the keys the group's shared_blocks[g] leading
  // blocks, and the result is a split-K partial (m, l, unnormalised o) in
  // slot 0 of each member's workspace row.
  const int32_t* group_start;    // [num_groups + 1] first member of each group
  const int32_t* shared_blocks;  // [num_groups]
  int max_shared_blocks;         // host bound on shared_blocks[g]; larger values are clamped
  float* ws_out;                 // [S, H, max_parts, D]
  float* ws_max;                 // [S, H, max_parts]
  float* ws_sum;                 // [S, H, max_parts]
  int max_parts;
  // Planned prefill (tcgen05 kernel, else null): CTA b serves work item
  // b / num_kv_heads for kv head b % num_kv_heads.  An item is kPlanItemInts
  // ints {sequence, query tile, first key, end key (-1: the tile's causal
  // end), piece, merge, pieces, 0}: a (sequence, query tile) unit whole
  // (pieces = 1), or one of the pieces its keys are cut into, whose partials
  // (m, l, unnormalised o) go to the workspace rows of merge entry `merge`
  // (ws_out / ws_max / ws_sum as [num_merges][H_kv][ROWS][kMaxPieces] (x D))
  // for the merge kernel.
  const int32_t* work;
  int num_merges;
  // the merge entries {sequence, query tile, pieces, 0} and the query rows
  // of a unit (the tcgen05 kernel's rows per CTA)
  const int32_t* merges;
  int unit_rows;
};

constexpr int kPlanItemInts = 8;
constexpr int kMaxPieces = 4;

// Two E4M3 codes (the low 16 bits of `two`, low byte first) -> two values
// packed as fp16x2 or bf16x2; exact, since every E4M3 value is an fp16 and a
// bf16 value.
__device__ __forceinline__ uint32_t e4m3x2_to(uint32_t two, Fp16) {
  uint32_t r;
  asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}"
      : "=r"(r)
      : "r"(two));
  return r;
}
__device__ __forceinline__ uint32_t e4m3x2_to(uint32_t two, Bf16) {
  const uint32_t h = e4m3x2_to(two, Fp16());
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack2(f.x, f.y, Bf16());
}

// A bf16 pair rounded to an fp16 pair; magnitudes beyond fp16 saturate at
// +-65504.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_sat(uint32_t w) {
  const float lo = fminf(fmaxf(__uint_as_float(w << 16), -65504.f), 65504.f);
  const float hi = fminf(fmaxf(__uint_as_float(w & 0xffff0000u), -65504.f), 65504.f);
  return pack2(lo, hi, Fp16());
}

template <int D_, int BS_, int G_, class DT_, int NS_, bool PREFIX_ = false, bool FP8_ = false>
struct PrefillTraits {
  static constexpr int D = D_, BS = BS_, G = G_, NS = NS_;
  // prefix mode: the shared-prefix pass of cascade decode (see PrefillParams)
  static constexpr bool kPrefix = PREFIX_;
  // E4M3 cache: the producer warp stages the codes by TMA and widens them into
  // the 16-bit stages the consumers read
  static constexpr bool kFp8 = FP8_;
  using DT = DT_;
  using T = typename DT::T;
  // Type of the MMAs and of P.  Over E4M3 caches it is fp16 for bf16 queries
  // too: the codes widen exactly to fp16, the query fragments are rounded to
  // fp16 once (saturating at +-65504), and fp16 P needs no hi + lo split.
  using MT = std::conditional_t<kFp8, Fp16, DT>;
  static constexpr bool kSplitP = std::is_same<MT, Bf16>::value;
  static constexpr bool kQToFp16 = kFp8 && std::is_same<DT, Bf16>::value;
  static constexpr int CW = 4;                       // consumer warps
  static constexpr int THREADS = (CW + 1) * 32;      // + the producer warp
  static constexpr int ROWS = CW * 16;               // query rows per CTA
  static constexpr int SUB = 16;                     // keys per stage
  static constexpr int SUBS_PER_BLOCK = BS / SUB;
  static constexpr int BOXES = D / 64;
  static constexpr int BOX_BYTES = SUB * 128;
  static constexpr int TILE_BYTES = BOXES * BOX_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // a 16-bit stage: K, then V
  static constexpr int KSTEPS = D / 16;
  static constexpr int NTD = D / 8;                  // output n-tiles
  // E4M3: NS code stages (TMA, rows of D codes, unswizzled) and NW 16-bit
  // stages the producer widens them into; the consumers cycle through CR
  // stages (the 16-bit ring itself for 16-bit caches)
  static constexpr int CODE_TILE = SUB * D;
  static constexpr int CODE_STAGE = 2 * CODE_TILE;
  static constexpr int NW = kFp8 ? 2 : 0;
  static constexpr int CR = kFp8 ? NW : NS;
  static constexpr int RING_BYTES = CR * STAGE_BYTES + (kFp8 ? NS * CODE_STAGE : 0);
  // barriers: full[NS], empty[NS] (TMA ring), then (E4M3) wide_full[NW],
  // wide_empty[NW]; then stage_ok[CR]
  static constexpr int NBAR = 2 * NS + 2 * NW;
  static_assert(BS % SUB == 0 && D % 64 == 0 && G >= 1 && G <= 8, "shape");
  static_assert(!kFp8 || D == 64, "E4M3 codes: head_dim 64 (128 runs the tcgen05 kernel)");
  static size_t smem_bytes() {
    return 1024 + static_cast<size_t>(RING_BYTES) + NBAR * 8 + CR * 4;
  }
};

// Byte offset of 16-byte chunk `ch` of row `t` in a tile of swizzled
// 16 x 128-byte boxes (the 128-byte TMA swizzle: chunk XOR row % 8).
__device__ __forceinline__ uint32_t prefill_swz(int t, int ch) {
  return static_cast<uint32_t>((ch >> 3) * 2048 + t * 128 + (((ch & 7) ^ (t & 7)) << 4));
}

template <class Tr>
__global__ void __launch_bounds__(Tr::THREADS)
    paged_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap) {
  using T = typename Tr::T;
  using MT = typename Tr::MT;
  constexpr int NS = Tr::NS, CR = Tr::CR, G = Tr::G, D = Tr::D, BS = Tr::BS, KS = Tr::KSTEPS;
  constexpr int NTD = Tr::NTD, ROWS = Tr::ROWS, CW = Tr::CW, SPB = Tr::SUBS_PER_BLOCK;
  constexpr bool kSplitP = Tr::kSplitP;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Tr::RING_BYTES);
  uint64_t* empty = full + NS;
  uint64_t* wide_full = empty + NS;
  uint64_t* wide_empty = wide_full + Tr::NW;
  int* stage_ok = reinterpret_cast<int*>(wide_empty + Tr::NW);
  // the barriers the consumers wait on and release
  uint64_t* cons_full = Tr::kFp8 ? wide_full : full;
  uint64_t* cons_empty = Tr::kFp8 ? wide_empty : empty;

  // heavier tiles (later queries see more keys) are launched first
  const int tile = p.q_tiles - 1 - static_cast<int>(blockIdx.x % p.q_tiles);
  const int unit = blockIdx.x / p.q_tiles;
  const int kvh = unit % p.num_kv_heads;
  // a sequence, or in prefix mode a group whose members are the "tokens"
  // q0 .. q0 + q_len - 1 and whose keys are its shared blocks
  const int seq = unit / p.num_kv_heads;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  grid_dependency_wait();
  trigger_dependents();
  int ctx = 0;
  if constexpr (Tr::kPrefix) {
    // the decode kernels start after the same clamped count
    int shared = p.shared_blocks[seq];
    if (shared > p.max_shared_blocks) {
      if (threadIdx.x == 0 && tile == 0 && kvh == 0) set_err(p.err, PKV_DEVERR_BAD_CONTEXT);
      shared = p.max_shared_blocks;
    }
    ctx = shared * BS;
  } else {
    ctx = p.context_lens[seq];
  }
  const int q0 = Tr::kPrefix ? p.group_start[seq] : p.query_start[seq];
  const int q_len = (Tr::kPrefix ? p.group_start[seq + 1] : p.query_start[seq + 1]) - q0;
  const int cap = min(p.max_context_len, p.max_blocks_per_seq * BS);
  if (ctx < 0 || ctx > cap || q_len < 0 || (!Tr::kPrefix && q_len > ctx) ||
      q_len > p.max_query_len) {
    if (threadIdx.x == 0 && tile == 0 && kvh == 0) set_err(p.err, PKV_DEVERR_BAD_CONTEXT);
    return;
  }
  const int rows_total = q_len * G;
  if (tile * ROWS >= rows_total || (Tr::kPrefix && ctx == 0)) return;
  const int last_tok = (min(rows_total, (tile + 1) * ROWS) - 1) / G;
  // keys this tile needs: 0 .. nkv-1
  const int nkv = Tr::kPrefix ? ctx : ctx - q_len + last_tok + 1;
  const int nsub = (nkv + Tr::SUB - 1) / Tr::SUB;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_addr(full + s), 1);
      mbar_init(smem_addr(empty + s), CW);
    }
#pragma unroll
    for (int s = 0; s < Tr::NW; ++s) {
      mbar_init(smem_addr(wide_full + s), 1);
      mbar_init(smem_addr(wide_empty + s), CW);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const uint32_t ring0 = smem_addr(smem);

  if (warp == CW) {
    // ---- producer: keys 16 at a time through the ring ----------------------
    // prefix mode: the group's first member holds the shared blocks' ids
    const int32_t* trow = p.block_tables +
                          static_cast<size_t>(Tr::kPrefix ? q0 : seq) * p.max_blocks_per_seq;
    const int nblk = (nkv + BS - 1) / BS;
    int chunk = -1, entry = -1;
    // physical block of stage k (warp-wide; k must not decrease from call to
    // call: the table is read 32 entries at a time)
    auto block_of = [&](int k) {
      const int blk = k / SPB;
      if ((blk >> 5) != chunk) {
        chunk = blk >> 5;
        const int i = (chunk << 5) + lane;
        entry = i < nblk ? trow[i] : -1;
      }
      return __shfl_sync(kFullMask, entry, blk & 31);
    };
    if constexpr (!Tr::kFp8) {
      for (int k = 0; k < nsub; ++k) {
        const int pb = block_of(k);
        bool ok = true;
        if (lane == 0) {
          const int stage = k % NS;
          ok = mbar_wait_bounded(smem_addr(empty + stage), ((k / NS) & 1) ^ 1);
          if (!ok) {
            set_err(p.err, PKV_DEVERR_TIMEOUT);
          } else if (static_cast<unsigned>(pb) < static_cast<unsigned>(p.num_blocks)) {
            stage_ok[stage] = 1;
            const int y = (pb * p.num_kv_heads + kvh) * BS + (k % SPB) * Tr::SUB;
            const uint32_t dst = ring0 + stage * Tr::STAGE_BYTES;
            const uint32_t bar = smem_addr(full + stage);
            mbar_arrive_expect_tx(bar, Tr::STAGE_BYTES);
#pragma unroll
            for (int b = 0; b < Tr::BOXES; ++b) {
              tma_load_2d(dst + b * Tr::BOX_BYTES, &kmap, b * 64, y, bar);
              tma_load_2d(dst + Tr::TILE_BYTES + b * Tr::BOX_BYTES, &vmap, b * 64, y, bar);
            }
          } else {
            set_err(p.err, PKV_DEVERR_BAD_BLOCK);
            stage_ok[stage] = 0;
            mbar_arrive(smem_addr(full + stage));
          }
        }
        if (!__shfl_sync(kFullMask, ok, 0)) break;
      }
    } else {
      // E4M3: TMA brings stage k's codes (one box of 16 rows x D codes per
      // kind) into code slot k % NS; the warp widens them into 16-bit stage
      // k % NW (the layout the 16-bit caches load), signals the consumers and
      // refills the slot with stage k + NS.
      const uint32_t codes0 = ring0 + CR * Tr::STAGE_BYTES;
      auto issue_codes = [&](int k) {  // warp-wide; true if the block is valid
        const int pb = block_of(k);
        const bool valid = static_cast<unsigned>(pb) < static_cast<unsigned>(p.num_blocks);
        if (lane == 0) {
          const uint32_t bar = smem_addr(full + k % NS);
          if (valid) {
            const int y = (pb * p.num_kv_heads + kvh) * BS + (k % SPB) * Tr::SUB;
            const uint32_t dst = codes0 + (k % NS) * Tr::CODE_STAGE;
            mbar_arrive_expect_tx(bar, Tr::CODE_STAGE);
            tma_load_2d(dst, &kmap, 0, y, bar);
            tma_load_2d(dst + Tr::CODE_TILE, &vmap, 0, y, bar);
          } else {
            set_err(p.err, PKV_DEVERR_BAD_BLOCK);
            mbar_arrive(bar);
          }
        }
        return valid;
      };
      unsigned loaded = 0;  // bit s: code slot s holds a valid block's codes
      for (int k = 0; k < min(NS, nsub); ++k) loaded |= (issue_codes(k) ? 1u : 0u) << k;
      for (int k = 0; k < nsub; ++k) {
        const int ws = k % Tr::NW, slot = k % NS;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(smem_addr(wide_empty + ws), ((k / Tr::NW) & 1) ^ 1) &&
               mbar_wait_bounded(smem_addr(full + slot), (k / NS) & 1);
          if (!ok) {
            set_err(p.err, PKV_DEVERR_TIMEOUT);
            // let the code loads still in flight land before the CTA can exit
            for (int jj = k; jj < min(k + NS, nsub); ++jj)
              (void)mbar_wait_bounded(smem_addr(full + jj % NS), (jj / NS) & 1);
          }
        }
        if (!__shfl_sync(kFullMask, ok, 0)) break;
        const bool valid = (loaded >> slot) & 1u;
        if (valid) {
          // 2 x 16 rows x D/16 chunks of 16 codes; chunk c of row r (dims
          // 16c .. 16c + 15) becomes 16-bit chunks 2(c % 4), 2(c % 4) + 1 of
          // row r in dim box c / 4, 128-byte swizzled
          const uint32_t src = codes0 + slot * Tr::CODE_STAGE;
          const uint32_t dst = ring0 + ws * Tr::STAGE_BYTES;
          constexpr int kChunks = Tr::CODE_STAGE / 16;
#pragma unroll
          for (int i = lane; i < kChunks; i += 32) {
            const int kind = i / (kChunks / 2);  // 0: K, 1: V
            const int ii = i % (kChunks / 2);
            const int r = ii / (D / 16), c = ii % (D / 16);
            uint32_t w[4];
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(src + i * 16)
                         : "memory");
            uint32_t h[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              h[2 * e] = e4m3x2_to(w[e] & 0xffffu, MT());
              h[2 * e + 1] = e4m3x2_to(w[e] >> 16, MT());
            }
            const uint32_t row =
                dst + kind * Tr::TILE_BYTES + (c >> 2) * Tr::BOX_BYTES + r * 128;
            const int c0 = (c & 3) * 2;
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                             row + ((c0 ^ (r & 7)) << 4)),
                         "r"(h[0]), "r"(h[1]), "r"(h[2]), "r"(h[3])
                         : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                             row + (((c0 + 1) ^ (r & 7)) << 4)),
                         "r"(h[4]), "r"(h[5]), "r"(h[6]), "r"(h[7])
                         : "memory");
          }
        }
        __syncwarp();
        if (lane == 0) {
          stage_ok[ws] = valid ? 1 : 0;
          mbar_arrive(smem_addr(wide_full + ws));
        }
        if (k + NS < nsub) {
          // this warp's reads of the slot come before TMA rewrites it
          fence_proxy_async_smem();
          __syncwarp();
          loaded = (loaded & ~(1u << slot)) | ((issue_codes(k + NS) ? 1u : 0u) << slot);
        }
      }
    }
    return;
  }

  // ---- consumers ---------------------------------------------------------
  const int c = lane & 3;
  const int rbase = tile * ROWS + warp * 16 + (lane >> 2);  // this lane's rows: rbase, rbase + 8
  int pos[2];
  const T* qrow[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = rbase + 8 * h;
    const bool active = r < rows_total;
    const int j = active ? r / G : 0;
    const int g = active ? r % G : 0;
    pos[h] = !active ? -1 : Tr::kPrefix ? ctx - 1 : ctx - q_len + j;
    qrow[h] = static_cast<const T*>(p.q) +
              (static_cast<size_t>(q0 + j) * p.num_heads + kvh * G + g) * D;
  }
  // Q as A fragments: a0 (row lo, d 2c..), a1 (row hi), a2 (row lo, d 8+2c..), a3 (row hi)
  uint32_t qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    qa[ks][0] = pos[0] >= 0 ? *reinterpret_cast<const uint32_t*>(qrow[0] + 16 * ks + 2 * c) : 0u;
    qa[ks][1] = pos[1] >= 0 ? *reinterpret_cast<const uint32_t*>(qrow[1] + 16 * ks + 2 * c) : 0u;
    qa[ks][2] =
        pos[0] >= 0 ? *reinterpret_cast<const uint32_t*>(qrow[0] + 16 * ks + 8 + 2 * c) : 0u;
    qa[ks][3] =
        pos[1] >= 0 ? *reinterpret_cast<const uint32_t*>(qrow[1] + 16 * ks + 8 + 2 * c) : 0u;
    if constexpr (Tr::kQToFp16) {
#pragma unroll
      for (int e = 0; e < 4; ++e) qa[ks][e] = bf16x2_to_f16x2_sat(qa[ks][e]);
    }
  }
  // E4M3: a cached value is code x scale; the K scale folds into the logit
  // scale and the V scale into the output
  float qscale = p.qscale, v_scale = 1.f;
  if constexpr (Tr::kFp8) {
    const float ks = p.k_scales[kvh];
    v_scale = p.v_scales[kvh];
    if (!(ks > 0.f && ks < INFINITY && v_scale > 0.f && v_scale < INFINITY) &&
        threadIdx.x == 0 && tile == 0)
      set_err(p.err, PKV_DEVERR_BAD_SCALE);
    qscale *= ks;
  }
  float acc[NTD][4];
#pragma unroll
  for (int n = 0; n < NTD; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY};
  float l[2] = {0.f, 0.f};

  // keys this warp can see: up to the position of its last active row
  const int wfirst = tile * ROWS + warp * 16;
  const int wlast = min(rows_total, wfirst + 16) - 1;
  const int warp_max_pos =
      wlast < wfirst ? -1 : Tr::kPrefix ? ctx - 1 : ctx - q_len + wlast / G;
  const int warp_min_pos = Tr::kPrefix ? ctx - 1 : ctx - q_len + wfirst / G;
  const int j8 = lane >> 3, r8 = lane & 7;

  for (int k = 0; k < nsub; ++k) {
    const int stage = k % CR;
    const bool ok = mbar_wait_bounded(smem_addr(cons_full + stage), (k / CR) & 1);
    if (!__all_sync(kFullMask, ok)) {
      if (lane == 0) {
        set_err(p.err, PKV_DEVERR_TIMEOUT);
        // 16-bit caches: let the loads still in flight land before the CTA
        // can exit (E4M3: the producer drains its own code loads)
        if constexpr (!Tr::kFp8)
          for (int jj = k; jj < min(k + NS, nsub); ++jj)
            (void)mbar_wait_bounded(smem_addr(full + jj % NS), (jj / NS) & 1);
      }
      __syncwarp();
      break;
    }
    const int kv0 = k * Tr::SUB;
    if (stage_ok[stage] && kv0 <= warp_max_pos) {
      const uint32_t kt = ring0 + stage * Tr::STAGE_BYTES;
      const uint32_t vt = kt + Tr::TILE_BYTES;
      // ---- S = Q K^T for 16 keys (two n-tiles) -------------------------------
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int t = ((j8 >> 1) << 3) + r8;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b[4];
          ldsm_x4(kt + prefill_swz(t, 2 * ks + (j8 & 1)), b);
          mma_16816(s[0], qa[ks], b[0], b[1], MT());
          mma_16816(s[1], qa[ks], b[2], b[3], MT());
        }
      }
      float x[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) x[nt][e] = s[nt][e] * qscale;
      if (kv0 + Tr::SUB - 1 > warp_min_pos) {  // the causal boundary crosses this stage
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = kv0 + nt * 8 + 2 * c + (e & 1);
            if (key > pos[e >> 1]) x[nt][e] = -INFINITY;
          }
      }
      // ---- online softmax per row (rows lo, hi; a quad of lanes shares a row)
      float pr[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float mx = fmaxf(fmaxf(x[0][2 * h], x[0][2 * h + 1]), fmaxf(x[1][2 * h], x[1][2 * h + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 2));
        const float m_new = fmaxf(m[h], mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;  // fully masked row so far
        const float alpha = exp2_approx(m[h] - m_use);
        float sum = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            pr[nt][2 * h + e] = exp2_approx(x[nt][2 * h + e] - m_use);
            sum += pr[nt][2 * h + e];
          }
        sum += __shfl_xor_sync(kFullMask, sum, 1);
        sum += __shfl_xor_sync(kFullMask, sum, 2);
        l[h] = l[h] * alpha + sum;
        m[h] = m_new;
        if (__any_sync(kFullMask, alpha != 1.f)) {
#pragma unroll
          for (int n = 0; n < NTD; ++n) {
            acc[n][2 * h] *= alpha;
            acc[n][2 * h + 1] *= alpha;
          }
        }
      }
      // ---- P as A fragments, straight from the S layout ----------------------
      uint32_t pa[4], pl[4];
      pa[0] = pack2(pr[0][0], pr[0][1], MT());
      pa[1] = pack2(pr[0][2], pr[0][3], MT());
      pa[2] = pack2(pr[1][0], pr[1][1], MT());
      pa[3] = pack2(pr[1][2], pr[1][3], MT());
      if constexpr (kSplitP) {
        // bf16 P as hi + lo so P.V keeps ~16 mantissa bits
        pl[0] = pack2(pr[0][0] - __uint_as_float(pa[0] << 16),
                      pr[0][1] - __uint_as_float(pa[0] & 0xffff0000u), Bf16());
        pl[1] = pack2(pr[0][2] - __uint_as_float(pa[1] << 16),
                      pr[0][3] - __uint_as_float(pa[1] & 0xffff0000u), Bf16());
        pl[2] = pack2(pr[1][0] - __uint_as_float(pa[2] << 16),
                      pr[1][1] - __uint_as_float(pa[2] & 0xffff0000u), Bf16());
        pl[3] = pack2(pr[1][2] - __uint_as_float(pa[3] << 16),
                      pr[1][3] - __uint_as_float(pa[3] & 0xffff0000u), Bf16());
      }
      // keys past the context may hold stale data: zero them in the V fragments
      const int vkeep = ctx - kv0;  // keys of this stage inside the context
      uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
      if (vkeep < Tr::SUB) {
        const int t0 = 2 * c, t1 = 8 + 2 * c;
        keep_lo = (t0 < vkeep ? 0x0000ffffu : 0u) | (t0 + 1 < vkeep ? 0xffff0000u : 0u);
        keep_hi = (t1 < vkeep ? 0x0000ffffu : 0u) | (t1 + 1 < vkeep ? 0xffff0000u : 0u);
      }
      // ---- O += P V -------------------------------------------------------------
      {
        const int t = ((j8 & 1) << 3) + r8;
#pragma unroll
        for (int pair = 0; pair < NTD / 2; ++pair) {
          uint32_t b[4];
          ldsm_x4_trans(vt + prefill_swz(t, 2 * pair + (j8 >> 1)), b);
          b[0] &= keep_lo;
          b[1] &= keep_hi;
          b[2] &= keep_lo;
          b[3] &= keep_hi;
          mma_16816(acc[2 * pair], pa, b[0], b[1], MT());
          mma_16816(acc[2 * pair + 1], pa, b[2], b[3], MT());
          if constexpr (kSplitP) {
            mma_16816(acc[2 * pair], pl, b[0], b[1], MT());
            mma_16816(acc[2 * pair + 1], pl, b[2], b[3], MT());
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(cons_empty + stage));
  }

  // ---- this lane's rows: normalised out, or (prefix mode) the split-K partial
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (pos[h] < 0) continue;
    const size_t row = static_cast<size_t>(qrow[h] - static_cast<const T*>(p.q)) / D;
    if constexpr (Tr::kPrefix) {
      // (m, l, unnormalised o) in slot 0 of the member's row
      const size_t slot = row * p.max_parts;
      if (c == 0) {
        if (p.context_lens[row / p.num_heads] < ctx) set_err(p.err, PKV_DEVERR_BAD_CONTEXT);
        p.ws_max[slot] = m[h];
        p.ws_sum[slot] = l[h];
      }
      float* o = p.ws_out + slot * D;
#pragma unroll
      for (int n = 0; n < NTD; ++n)
        *reinterpret_cast<float2*>(o + n * 8 + 2 * c) =
            make_float2(acc[n][2 * h] * v_scale, acc[n][2 * h + 1] * v_scale);
    } else {
      const float inv = l[h] > 0.f ? v_scale / l[h] : 0.f;
      T* orow = static_cast<T*>(p.out) + row * D;
#pragma unroll
      for (int n = 0; n < NTD; ++n) {
        *reinterpret_cast<uint32_t*>(orow + n * 8 + 2 * c) =
            pack2(acc[n][2 * h] * inv, acc[n][2 * h + 1] * inv, typename Tr::DT());
      }
    }
  }
}

}  // namespace pkv
