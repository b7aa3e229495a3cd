// paged_prefill_tc_kernels.cuh — chunked-prefill attention on the 5th-generation
// tensor cores (tcgen05 + TMEM) for head_dim 128 on B200 (sm_100a).
//
// Computes what paged_prefill_kernels.cuh computes (causal attention of each
// new token over its sequence's paged cache).  A CTA covers QT query tiles of
// 128 rows (a row is a (token, head-of-this-kv-head) pair) that share every
// K/V tile of 64 keys:
//   * warp 0 (K producer): TMA loads of the query tiles (3-D tensor map over
//     [T, H, D]) and of the K tiles, gathered from 16-key pieces of the paged
//     cache through the block table into an NS-stage ring; the 8 boxes of a
//     tile are issued by 8 lanes at once.
//   * warp 2 (V producer): the same for the V tiles.  K of a stage is released
//     once S has read it, V once P.V has, so K loads run further ahead.
//   * warp 1 (S issuer): allocates 256 TMEM columns per query tile; one thread
//     issues S = Q K^T (M=128, N=64, K=128; A, B K-major) into one of two TMEM
//     S buffers per query tile.  The last warp (P.V issuer): one thread issues
//     O += P V (M=128, N=128, K=64) with A = P read from TMEM (the TS form) and
//     B = V (MN-major) from shared memory.  Completion goes to mbarriers
//     through tcgen05.commit; each issuer takes its MMAs in tile order.
//   * 4 softmax warps per query tile: thread r owns row r (TMEM lane r): it
//     reads its S row from TMEM, masks causally (only on tiles that reach past
//     the row), keeps the running max / sum in base 2 with the scale folded
//     into the exponent's FFMA, rescales its O row in TMEM when the max moves,
//     and writes P (fp16, or bf16 split into hi + lo halves) into TMEM over
//     the S it just read.  At the end it reads O, divides by the sum and
//     stores the row (or, for the cascade prefix pass, writes the partial).
// All operand tiles use the 128-byte swizzle (8-row x 128-byte atoms, stride
// 1024 bytes).  Keys past the context (or not loaded) are zeroed in the V tile
// before P.V so stale NaN never enters the tensor-core sum.  Every mbarrier
// wait is bounded; TMEM is released on every path.
#pragma once

#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "paged_prefill_kernels.cuh"

// The cascade prefix pass (one query tile, 256 TMEM columns): two K/V stages
// and at most 128 registers a thread, so that two CTAs share an SM and one's
// start and end overlap the other's tiles.  Measured on B200 (prefix-sharing
// batch, one cascade decode): 6 stages, one CTA per SM 0.1778 ms; 4 stages
// 0.1781; 3 stages 0.1799; 2 stages, two CTAs per SM 0.1616.
#ifndef PKV_PREFIX_STAGES
#define PKV_PREFIX_STAGES 2
#endif
#ifndef PKV_PREFIX_MIN_BLOCKS
#define PKV_PREFIX_MIN_BLOCKS 2
#endif
// K/V stages of a one-query-tile prefill CTA (PKV_PREFILL_QUERY_TILES=1)
#ifndef PKV_QT1_STAGES
#define PKV_QT1_STAGES 6
#endif

namespace pkv {
namespace tc {

// ---- tcgen05 wrappers --------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]; issued by one thread.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]: A (M x 16, K-major) sits in tensor
// memory, row m in lane m, two 16-bit K elements per 32-bit column.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// Arrives once on `bar` when all earlier tcgen05.mma of this thread complete.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// 16 consecutive 32-bit columns of this warp's 32 TMEM lanes (one per thread).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---- sm_100 packed fp32 pairs and three-input max (fewer softmax instructions)
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// (a * b + c) on both halves, each rounded to nearest even as fmaf
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// max of three, with fmaxf's treatment of NaN
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 layout: start
// address, leading / stride byte offsets in 16-byte units, version 1, layout 2).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                   uint32_t sbo_bytes) {
  return (static_cast<uint64_t>((saddr >> 4) & 0x3FFFu)) |
         (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         (2ull << 61);
}

// Instruction descriptor, kind::f16, fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_f16(bool bf16, int m, int n, bool b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

}  // namespace tc

template <int BS_, int G_, class DT_, int QT_, bool PREFIX_ = false, bool FP8_ = false,
          int NKEY_ = 64>
struct TcPrefillTraits {
  static constexpr int D = 128, BS = BS_, G = G_, QT = QT_;
  // prefix mode: the shared-prefix pass of cascade decode (no causal mask,
  // split-K partials out; see PrefillParams)
  static constexpr bool kPrefix = PREFIX_;
  // E4M3 cache: the producer warps stage each tile's codes by TMA and widen
  // them into the 16-bit stage the MMAs read; K and V scales are per kv head
  static constexpr bool kFp8 = FP8_;
  using DT = DT_;
  using T = typename DT::T;
  // Element type of the MMAs and of P.  Over E4M3 caches it is fp16 for bf16
  // queries too: the codes widen exactly to fp16, the query tiles are rounded
  // to fp16 in shared memory once per CTA (saturating at +-65504, as the E4M3
  // decode does), and fp16 P needs no hi + lo split, so P.V runs once.
  using MT = std::conditional_t<kFp8, Fp16, DT>;
  static constexpr bool kBf16 = std::is_same<MT, Bf16>::value;
  static constexpr bool kQToFp16 = kFp8 && std::is_same<DT, Bf16>::value;
  static constexpr int M = 128;                  // rows of one query tile (one TMEM lane each)
  static constexpr int ROWS = QT * M;            // query rows per CTA; they share every KV tile
  // keys per KV tile: 64 with two S buffers per query tile, or 128 with one
  // (two query tiles then fill TMEM with S 128 + O 128 each, and each S MMA
  // reads Q once per 128 keys)
  static constexpr int NKEY = NKEY_;
  static constexpr int NSB = NKEY == 128 ? 1 : 2;   // S buffers per query tile
  static constexpr int PIECES = NKEY / 16;          // 16-key TMA boxes per tile and kind
  static constexpr int HALVES = NKEY / 64;          // 64-column passes of the softmax
  // bf16 P as hi + lo: with 128-key tiles each 16-key group keeps its 8 hi
  // columns and 8 lo columns together, so the P of one 64-key half lies
  // within the S columns that half has already been read from
  static constexpr int kSortUnits = 512;         // (sequence, tile) units ranked per CTA
  // KV stages: what fits beside QT query tiles (P lives in TMEM, over S); the
  // cascade prefix pass (one query tile) keeps PKV_PREFIX_STAGES
  static constexpr int NS = NKEY == 128 ? 2
                            : kFp8 ? 4 : QT == 2 ? 5 : kPrefix ? PKV_PREFIX_STAGES : PKV_QT1_STAGES;
  static constexpr int NSTG = kFp8 ? 2 : 0;      // E4M3 staging slots per kind
  static constexpr int MIN_BLOCKS = kPrefix && !kFp8 ? PKV_PREFIX_MIN_BLOCKS : 1;  // CTAs per SM
  // warps: K producer, S issuer, V producer, 4 softmax warps per query tile,
  // P.V issuer
  static constexpr int PV_WARP = 3 + 4 * QT;
  // E4M3: two warps per kind widen each tile (the producer warp and a helper,
  // warps PV_WARP + 1 for K and PV_WARP + 2 for V), 32 rows each
  static constexpr int NWIDEN = kFp8 ? 2 : 1;
  static constexpr int THREADS = (PV_WARP + 1 + (NWIDEN - 1) * 2) * 32;
  // shared-memory layout (all 1024-byte aligned)
  static constexpr int Q_HALF = M * 128;         // [128 rows][64 dims] = 16 KiB
  static constexpr int Q_TILE = 2 * Q_HALF;
  static constexpr int KV_HALF = NKEY * 128;     // [NKEY keys][64 dims]
  static constexpr int STAGE = 4 * KV_HALF;      // K0 K1 V0 V1
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = QT * Q_TILE;
  static constexpr int STG_TILE = NKEY * 128;   // [NKEY keys][128 codes], 128-byte swizzle
  static constexpr int OFF_STG = OFF_KV + NS * STAGE;            // K slots, then V slots
  static constexpr int OFF_BAR = OFF_STG + 2 * NSTG * STG_TILE;
  // barriers: q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], then
  // per query tile s_full[NSB], p_full[NSB], o_done[NSB]; then (E4M3) the staging
  // slots' stg_full[2][NSTG]; then q_ready (query tiles rounded to fp16);
  // then (E4M3) stg_read[2][NSTG] (both widening warps are done with a
  // slot); then the TMEM address slot
  static constexpr int BAR_Q_READY = 1 + 4 * NS + 3 * NSB * QT + 2 * NSTG;
  static constexpr int BAR_STG_READ = BAR_Q_READY + 1;
  static constexpr int NBAR = BAR_STG_READ + 2 * NSTG;
  // the softmax reference max moves only when a row max exceeds it by more
  // than this (base-2 units), so P stays below 2^8 and O is rarely rescaled
  static constexpr float kRescaleThreshold = 8.f;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16;
  // TMEM per query tile q, from q * QCOLS: NSB S buffers of NKEY columns (P
  // over S), then O (128 columns)
  static constexpr int O_COL = NSB * NKEY;
  static constexpr int QCOLS = O_COL + 128;
  static constexpr uint32_t TMEM_COLS = QT * QCOLS <= 256 ? 256 : 512;
  static_assert(QT == 1 || QT == 2, "one or two query tiles per CTA");
  static_assert(NKEY == 64 || (NKEY == 128 && !kFp8), "128-key tiles: 16-bit caches");
  static_assert(QT * QCOLS <= 512, "tensor memory");
  static_assert(1024 + SMEM <= 232448, "shared memory per CTA");
  static size_t smem_bytes() { return 1024 + static_cast<size_t>(SMEM); }
};

template <class Tr>
__global__ void __launch_bounds__(Tr::THREADS, Tr::MIN_BLOCKS)
    paged_prefill_tc_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap qmap,
                            const __grid_constant__ CUtensorMap kmap,
                            const __grid_constant__ CUtensorMap vmap) {
  using T = typename Tr::T;
  using DT = typename Tr::DT;
  constexpr int G = Tr::G, BS = Tr::BS, M = Tr::M, NKEY = Tr::NKEY, NS = Tr::NS;
  constexpr int QT = Tr::QT, ROWS = Tr::ROWS;
  constexpr uint32_t IDESC_S = tc::idesc_f16(Tr::kBf16, M, NKEY, false);
  constexpr int PIECES = Tr::PIECES, NSB = Tr::NSB;
  // TMEM column (within a tile's S buffer) of 16-key group kk's P: hi, lo
  auto p_col_hi = [](int kk) { return Tr::NKEY == 128 && Tr::kBf16 ? 16 * kk : 8 * kk; };
  auto p_col_lo = [](int kk) { return Tr::NKEY == 128 ? 16 * kk + 8 : Tr::NKEY / 2 + 8 * kk; };
  constexpr uint32_t IDESC_O = tc::idesc_f16(Tr::kBf16, M, 128, true);
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BAR);
  const uint32_t bar_q = smem_addr(bars + 0);
  auto bar_k_full = [&](int s) { return smem_addr(bars + 1 + s); };
  auto bar_k_empty = [&](int s) { return smem_addr(bars + 1 + NS + s); };
  auto bar_v_full = [&](int s) { return smem_addr(bars + 1 + 2 * NS + s); };
  auto bar_v_empty = [&](int s) { return smem_addr(bars + 1 + 3 * NS + s); };
  auto bar_s_full = [&](int q, int b) {
    return smem_addr(bars + 1 + 4 * NS + 3 * Tr::NSB * q + b);
  };
  auto bar_p = [&](int q, int b) {
    return smem_addr(bars + 1 + 4 * NS + 3 * Tr::NSB * q + Tr::NSB + b);
  };
  auto bar_o = [&](int q, int b) {
    return smem_addr(bars + 1 + 4 * NS + 3 * Tr::NSB * q + 2 * Tr::NSB + b);
  };
  auto bar_stg = [&](int kind, int s) {
    return smem_addr(bars + 1 + 4 * NS + 3 * Tr::NSB * QT + kind * Tr::NSTG + s);
  };
  const uint32_t bar_q_ready = smem_addr(bars + Tr::BAR_Q_READY);
  auto bar_stg_read = [&](int kind, int s) {
    return smem_addr(bars + Tr::BAR_STG_READ + kind * Tr::NSTG + s);
  };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Tr::NBAR);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  grid_dependency_wait();
  trigger_dependents();

  // Which (sequence, query tile) this CTA serves.  The kv heads of one unit
  // are adjacent CTAs.  Units are taken longest first (the most keys to
  // read), so the long ones do not start last and leave a tail: each CTA
  // ranks every (sequence, tile) unit by its key count from context_lens and
  // query_start (staged in the K/V ring before any load uses it) and takes
  // the unit whose rank is its own index.  Beyond kSortUnits units, or in
  // prefix mode, later query tiles of a sequence simply come first.
  const int kvh = static_cast<int>(blockIdx.x % p.num_kv_heads);
  const int rank = static_cast<int>(blockIdx.x / p.num_kv_heads);
  int seq = rank / p.q_tiles;
  int tile = p.q_tiles - 1 - rank % p.q_tiles;
  // a planned item: keys [kb, ke) of the unit (ke = -1: to its causal end),
  // piece `piece` of `pieces`, partials to merge entry `merge`
  int kb = 0, ke = -1, piece = 0, pieces = 1, merge = 0;
  if constexpr (!Tr::kPrefix) {
    if (p.work != nullptr) {
      const int32_t* it = p.work + static_cast<size_t>(rank) * kPlanItemInts;
      seq = it[0];
      tile = it[1];
      kb = it[2];
      ke = it[3];
      piece = it[4];
      merge = it[5];
      pieces = it[6];
      if (static_cast<unsigned>(seq) >= static_cast<unsigned>(p.num_seqs)) {
        if (threadIdx.x == 0) set_err(p.err, PKV_DEVERR_BAD_ORDER);
        return;
      }
    } else if (p.num_seqs * p.q_tiles <= Tr::kSortUnits) {
      int* keys_of = reinterpret_cast<int*>(smem + Tr::OFF_KV);  // [num_seqs] first key, tiles
      int* chosen = keys_of + 2 * p.num_seqs;
      const int cap = min(p.max_context_len, p.max_blocks_per_seq * BS);
      for (int i = threadIdx.x; i < p.num_seqs; i += Tr::THREADS) {
        const int c = min(max(p.context_lens[i], 0), cap);
        const int ql = p.query_start[i + 1] - p.query_start[i];
        keys_of[2 * i] = c - ql;   // keys before the sequence's first new token
        keys_of[2 * i + 1] = ql;
      }
      if (threadIdx.x == 0) chosen[0] = rank;
      __syncthreads();
      const int units = p.num_seqs * p.q_tiles;
      // keys CTA-unit u reads (-1: no rows); later tiles see more keys
      auto unit_keys = [&](int u) {
        const int s = u / p.q_tiles, t = p.q_tiles - 1 - u % p.q_tiles;
        const int ql = keys_of[2 * s + 1];
        const int rows = ql * G;
        if (ql <= 0 || t * ROWS >= rows) return -1;
        return keys_of[2 * s] + (min(rows, (t + 1) * ROWS) - 1) / G + 1;
      };
      for (int u = threadIdx.x; u < units; u += Tr::THREADS) {
        const int ku = unit_keys(u);
        int r = 0;
        for (int v = 0; v < units; ++v) {
          const int kv = unit_keys(v);
          r += (kv > ku || (kv == ku && v < u)) ? 1 : 0;
        }
        if (r == rank) chosen[0] = u;
      }
      __syncthreads();
      const int u = chosen[0];
      seq = u / p.q_tiles;
      tile = p.q_tiles - 1 - u % p.q_tiles;
      // the ring is written by TMA (the async proxy) later
      fence_proxy_async_smem();
      __syncthreads();
    }
  }

  // seq is a sequence, or in prefix mode a group whose members are the
  // "tokens" q0 .. q0 + q_len - 1 and whose keys are its shared blocks
  int ctx = 0;
  if constexpr (!Tr::kPrefix) {
    ctx = p.context_lens[seq];
  } else {
    // the decode kernels start after the same clamped count
    int shared = p.shared_blocks[seq];
    if (shared > p.max_shared_blocks) {
      if (threadIdx.x == 0 && tile == 0 && kvh == 0) set_err(p.err, PKV_DEVERR_BAD_CONTEXT);
      shared = p.max_shared_blocks;
    }
    ctx = shared * BS;
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
  if (p.work != nullptr) {
    // a piece before the last covers whole tiles of history keys, which every
    // row sees; the last starts within the history and runs to the causal end
    const int hist = ctx - q_len;
    const bool last = piece == pieces - 1;
    const bool bad =
        tile < 0 || tile * ROWS >= rows_total || pieces < 1 || pieces > kMaxPieces ||
        piece < 0 || piece >= pieces || kb < 0 || kb % NKEY != 0 ||
        (pieces > 1 && static_cast<unsigned>(merge) >= static_cast<unsigned>(p.num_merges)) ||
        (last ? (ke != -1 || kb > hist || (pieces == 1 && kb != 0))
              : (ke % NKEY != 0 || ke <= kb || ke > hist));
    if (bad) {
      if (threadIdx.x == 0) set_err(p.err, PKV_DEVERR_BAD_ORDER);
      return;
    }
  }
  if (tile * ROWS >= rows_total || (Tr::kPrefix && ctx == 0)) return;
  const int tok0 = tile * (ROWS / G);  // first query token of this CTA
  // KV tiles each query tile needs (later rows see more keys; 0 = no rows)
  int ntq[QT];
#pragma unroll
  for (int q = 0; q < QT; ++q) {
    const int r0 = tile * ROWS + q * M;
    const int last = (min(rows_total, r0 + M) - 1) / G;
    const int keys = Tr::kPrefix ? ctx : ctx - q_len + last + 1;
    const int kq = ke >= 0 ? min(keys, ke) : keys;
    ntq[q] = r0 < rows_total ? (kq - kb + NKEY - 1) / NKEY : 0;
  }
  const int last_tok = (min(rows_total, (tile + 1) * ROWS) - 1) / G;
  const int nkv_all = Tr::kPrefix ? ctx : ctx - q_len + last_tok + 1;
  const int nkv = ke >= 0 ? min(nkv_all, ke) : nkv_all;  // end of the keys the CTA reads
  const int ntiles = (nkv - kb + NKEY - 1) / NKEY;
  // From here on key indices count from kb (a whole number of blocks): the
  // table row starts at block kb / BS, and positions and ends are shifted.
  const int nkv_r = nkv - kb;

  if (threadIdx.x == 0) {
    // one arrival each (an expect_tx arrive or a tcgen05.commit), except p_full:
    // one arrival per softmax warp of the query tile
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_k_full(s), Tr::NWIDEN);  // E4M3: each widening warp arrives
      mbar_init(bar_k_empty(s), 1);
      mbar_init(bar_v_full(s), Tr::NWIDEN);
      mbar_init(bar_v_empty(s), 1);
    }
    for (int q = 0; q < QT; ++q) {
      for (int b = 0; b < Tr::NSB; ++b) {
        mbar_init(bar_s_full(q, b), 1);
        mbar_init(bar_p(q, b), 4);
        mbar_init(bar_o(q, b), 1);
      }
    }
    for (int s = 0; s < Tr::NSTG; ++s) {
      mbar_init(bar_stg(0, s), 1);
      mbar_init(bar_stg(1, s), 1);
      mbar_init(bar_stg_read(0, s), Tr::NWIDEN);
      mbar_init(bar_stg_read(1, s), Tr::NWIDEN);
    }
    mbar_init(bar_q_ready, 4 * QT);  // one arrival per softmax warp
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_addr(tmem_slot), Tr::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 || warp == 2 || warp > Tr::PV_WARP) {
    // ---- producers: warp 0 loads Q and the K tiles, warp 2 the V tiles ---------------
    // K of a stage is released once S has read it, V once P.V has, so the K
    // loads can run further ahead than the V loads.  E4M3: a helper warp per
    // kind widens half of each tile.
    const bool helper = warp > Tr::PV_WARP;
    const bool is_k = warp == 0 || warp == Tr::PV_WARP + 1;
    // prefix mode: the group's first member holds the shared blocks' ids
    const int32_t* trow = p.block_tables +
                          static_cast<size_t>(Tr::kPrefix ? q0 : seq) * p.max_blocks_per_seq +
                          kb / BS;
    const int nblk = (nkv_r + BS - 1) / BS;
    if (warp == 0 && lane == 0) {
      mbar_arrive_expect_tx(bar_q, QT * Tr::Q_TILE);
#pragma unroll
      for (int q = 0; q < QT; ++q) {
        const uint32_t dst = sbase + Tr::OFF_Q + q * Tr::Q_TILE;
        const int z = q0 + tok0 + q * (M / G);
        tc::tma_load_3d(dst, &qmap, 0, kvh * G, z, bar_q);
        tc::tma_load_3d(dst + Tr::Q_HALF, &qmap, 64, kvh * G, z, bar_q);
      }
    }
    int chunk = -1, entry = -1;
    // the 16-key pieces of tile t that hold keys this CTA needs (pb = -1 past
    // them); t must not decrease from call to call (the table is read in
    // 32-entry chunks)
    auto lookup = [&](int t, int (&pb)[PIECES]) {
      int npieces = 0;
#pragma unroll
      for (int i = 0; i < PIECES; ++i) {
        const int key0 = t * NKEY + i * 16;
        pb[i] = -1;
        if (key0 < nkv_r) {
          const int blk = key0 / BS;
          if ((blk >> 5) != chunk) {
            chunk = blk >> 5;
            const int idx = (chunk << 5) + lane;
            entry = idx < nblk ? trow[idx] : -1;
          }
          pb[i] = __shfl_sync(kFullMask, entry, blk & 31);
          npieces = i + 1;
        }
      }
      return npieces;
    };
    auto valid_block = [&](int b) {
      return static_cast<unsigned>(b) < static_cast<unsigned>(p.num_blocks);
    };
    if constexpr (Tr::kFp8) {
      // E4M3: TMA brings tile t's codes into staging slot t % NSTG (one box of
      // 16 rows x 128 codes per piece); once a 16-bit stage is free the warp
      // widens them into it, signals the MMAs, and refills the slot with tile
      // t + NSTG.
      const int kind = is_k ? 0 : 1;
      const uint32_t stg0 = sbase + Tr::OFF_STG + kind * Tr::NSTG * Tr::STG_TILE;
      auto stage_codes = [&](int t) {  // all lanes (the table lookup is warp-wide)
        int pb[PIECES];
        const int npieces = lookup(t, pb);
        int bytes = 0;
#pragma unroll
        for (int i = 0; i < PIECES; ++i)
          if (i < npieces && valid_block(pb[i])) bytes += 2048;
        const uint32_t bar = bar_stg(kind, t % Tr::NSTG);
        if (lane == 0) {
          for (int i = 0; i < npieces; ++i)
            if (is_k && !valid_block(pb[i])) set_err(p.err, PKV_DEVERR_BAD_BLOCK);
          if (bytes > 0)
            mbar_arrive_expect_tx(bar, bytes);
          else
            mbar_arrive(bar);
        }
        __syncwarp();
        if (lane < PIECES) {
          int pbi = -1;
#pragma unroll
          for (int i = 0; i < PIECES; ++i)
            if (i == lane) pbi = pb[i];
          if (lane < npieces && valid_block(pbi)) {
            const int key0 = t * NKEY + lane * 16;
            const int y = (pbi * p.num_kv_heads + kvh) * BS + (key0 % BS);
            tma_load_2d(stg0 + (t % Tr::NSTG) * Tr::STG_TILE + lane * 2048,
                        is_k ? &kmap : &vmap, 0, y, bar);
          }
        }
        __syncwarp();
      };
      if (!helper)
        for (int t = 0; t < min(Tr::NSTG, ntiles); ++t) stage_codes(t);
      for (int t = 0; t < ntiles; ++t) {
        const int stage = t % NS;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(is_k ? bar_k_empty(stage) : bar_v_empty(stage),
                                 ((t / NS) & 1) ^ 1) &&
               mbar_wait_bounded(bar_stg(kind, t % Tr::NSTG), (t / Tr::NSTG) & 1);
          if (!ok) set_err(p.err, PKV_DEVERR_TIMEOUT);
        }
        ok = __shfl_sync(kFullMask, ok, 0);
        if (!ok) break;
        // 64 rows x 8 chunks of 16 codes; this warp's half of the rows, lane
        // takes chunks lane, lane + 32, ...  Chunk c of row r (dims 16c ..
        // 16c + 15) becomes 16-bit chunks 2(c % 4) and 2(c % 4) + 1 of row r in
        // dim half c / 4; both layouts use the 128-byte swizzle (16-byte chunk
        // index XOR row % 8).
        const uint32_t src = stg0 + (t % Tr::NSTG) * Tr::STG_TILE;
        const uint32_t dst = sbase + Tr::OFF_KV + stage * Tr::STAGE + (is_k ? 0 : 2 * Tr::KV_HALF);
        const int first = helper ? NKEY * 8 / 2 : 0;
#pragma unroll 4
        for (int k = 0; k < NKEY * 8 / Tr::NWIDEN / 32; ++k) {
          const int idx = first + lane + 32 * k;
          const int r = idx >> 3, c = idx & 7;
          uint32_t w[4];
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                       : "r"(src + r * 128 + ((c ^ (r & 7)) << 4))
                       : "memory");
          uint32_t h[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            h[2 * e] = e4m3x2_to(w[e] & 0xffffu, typename Tr::MT());
            h[2 * e + 1] = e4m3x2_to(w[e] >> 16, typename Tr::MT());
          }
          const uint32_t row = dst + (c >> 2) * Tr::KV_HALF + r * 128;
          const int c0 = (c & 3) * 2;
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((c0 ^ (r & 7)) << 4)),
                       "r"(h[0]), "r"(h[1]), "r"(h[2]), "r"(h[3])
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                           row + (((c0 + 1) ^ (r & 7)) << 4)),
                       "r"(h[4]), "r"(h[5]), "r"(h[6]), "r"(h[7])
                       : "memory");
        }
        // the widened rows are for the MMAs (async proxy); this warp is done
        // with the slot's codes
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(is_k ? bar_k_full(stage) : bar_v_full(stage));
          mbar_arrive(bar_stg_read(kind, t % Tr::NSTG));
        }
        if (!helper && t + Tr::NSTG < ntiles) {
          // TMA refills the slot once both widening warps have read it
          bool read = true;
          if (lane == 0) {
            read = mbar_wait_bounded(bar_stg_read(kind, t % Tr::NSTG), (t / Tr::NSTG) & 1);
            if (!read) set_err(p.err, PKV_DEVERR_TIMEOUT);
          }
          if (!__shfl_sync(kFullMask, read, 0)) break;
          stage_codes(t + Tr::NSTG);
        }
      }
    } else {
      for (int t = 0; t < ntiles; ++t) {
        const int stage = t % NS;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(is_k ? bar_k_empty(stage) : bar_v_empty(stage),
                                 ((t / NS) & 1) ^ 1);
          if (!ok) set_err(p.err, PKV_DEVERR_TIMEOUT);
        }
        ok = __shfl_sync(kFullMask, ok, 0);
        if (!ok) break;
        // the 16-key pieces of this tile that hold keys this CTA needs
        int npieces = 0;
        int pb[PIECES];
#pragma unroll
        for (int i = 0; i < PIECES; ++i) {
          const int key0 = t * NKEY + i * 16;
          pb[i] = -1;
          if (key0 < nkv_r) {
            const int blk = key0 / BS;
            if ((blk >> 5) != chunk) {
              chunk = blk >> 5;
              const int idx = (chunk << 5) + lane;
              entry = idx < nblk ? trow[idx] : -1;
            }
            pb[i] = __shfl_sync(kFullMask, entry, blk & 31);
            npieces = i + 1;
          }
        }
        int bytes = 0;
#pragma unroll
        for (int i = 0; i < PIECES; ++i)
          if (i < npieces && static_cast<unsigned>(pb[i]) < static_cast<unsigned>(p.num_blocks))
            bytes += 2 * 2048;
        const uint32_t bar = is_k ? bar_k_full(stage) : bar_v_full(stage);
        if (lane == 0) {
          for (int i = 0; i < npieces; ++i)
            if (is_k && static_cast<unsigned>(pb[i]) >= static_cast<unsigned>(p.num_blocks))
              set_err(p.err, PKV_DEVERR_BAD_BLOCK);
          if (bytes > 0)
            mbar_arrive_expect_tx(bar, bytes);
          else
            mbar_arrive(bar);
        }
        __syncwarp();
        // lanes 0 .. 2 PIECES - 1 issue the tile's boxes of K (or V) at once:
        // lane = piece * 2 + half; kind 0 / 1 = K low / high dims, 2 / 3 = V
        // low / high dims
        if (lane < 2 * PIECES) {
          const int i = lane >> 1, kind = (is_k ? 0 : 2) + (lane & 1);
          int pbi = -1;
#pragma unroll
          for (int i2 = 0; i2 < PIECES; ++i2)
            if (i2 == i) pbi = pb[i2];
          if (i < npieces && static_cast<unsigned>(pbi) < static_cast<unsigned>(p.num_blocks)) {
            const uint32_t st = sbase + Tr::OFF_KV + stage * Tr::STAGE;
            const int key0 = t * NKEY + i * 16;
            const int y = (pbi * p.num_kv_heads + kvh) * BS + (key0 % BS);
            tma_load_2d(st + kind * Tr::KV_HALF + i * 2048, kind < 2 ? &kmap : &vmap,
                        (kind & 1) * 64, y, bar);
          }
        }
        __syncwarp();
      }
    }
  } else if (warp == 1 || warp == Tr::PV_WARP) {
    // ---- MMA issuers ----------------------------------------------------------------
    if (lane == 0) {
      // only S reads Q (rounded to fp16 first when the MMAs run in fp16 for bf16 queries)
      bool ok = warp != 1 || mbar_wait_bounded(Tr::kQToFp16 ? bar_q_ready : bar_q, 0);
      // Operand descriptors as a base plus a start-address step: the 14-bit
      // start field holds address / 16 and never carries, since shared memory
      // ends below 2^18 bytes.  This keeps the issuing thread's work per MMA to
      // one add.
      const uint64_t d_q = tc::smem_desc_sw128(sbase + Tr::OFF_Q, 16, 1024);
      const uint64_t d_k = tc::smem_desc_sw128(sbase + Tr::OFF_KV, 16, 1024);
      const uint64_t d_v = tc::smem_desc_sw128(sbase + Tr::OFF_KV + 2 * Tr::KV_HALF, Tr::KV_HALF, 1024);
      // O_q += P_q V for tile t
      auto issue_pv = [&](int q, int t) {
        const uint64_t v0 = d_v + static_cast<uint32_t>((t % NS) * (Tr::STAGE >> 4));
        const uint32_t o_tmem = tmem + q * Tr::QCOLS + Tr::O_COL;
        // P in TMEM over the tile's S buffer (p_col_hi / p_col_lo)
        const uint32_t p_tmem = tmem + q * Tr::QCOLS + (t % NSB) * NKEY;
#pragma unroll
        for (int kk = 0; kk < NKEY / 16; ++kk) {
          const uint64_t bdesc = v0 + kk * (2048 >> 4);
          const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
          tc::umma_f16_ts(o_tmem, p_tmem + p_col_hi(kk), bdesc, IDESC_O, acc);
          if constexpr (Tr::kBf16)
            tc::umma_f16_ts(o_tmem, p_tmem + p_col_lo(kk), bdesc, IDESC_O, 1u);
        }
        tc::umma_commit(bar_o(q, t % NSB));
      };
      // S_q = Q_q K^T of tile t
      auto issue_s = [&](int q, int t) {
        const uint64_t k0 = d_k + static_cast<uint32_t>((t % NS) * (Tr::STAGE >> 4));
        const uint64_t q0d = d_q + q * (Tr::Q_TILE >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t step = (ks < 4 ? 0 : Tr::Q_HALF >> 4) + (ks & 3) * 2;
          const uint32_t kstep = (ks < 4 ? 0 : Tr::KV_HALF >> 4) + (ks & 3) * 2;
          tc::umma_f16(tmem + q * Tr::QCOLS + (t % NSB) * NKEY, q0d + step, k0 + kstep, IDESC_S,
                       ks > 0 ? 1u : 0u);
        }
        tc::umma_commit(bar_s_full(q, t % NSB));
      };
      // Two issuing threads, each taking its MMAs in order with one wait at a
      // time: warp 1 issues S of tile u once its K has landed and P.V of tile
      // u - 2 has read the P held in the S buffer it overwrites; warp PV_WARP
      // issues P.V of tile t once that tile's P and V are in.  (One thread
      // polling for both measured slower on B200.)
      // Each query tile's MMAs go out as soon as that tile's inputs are in,
      // except P.V of the CTA's last KV tile, whose V rows past the context
      // the softmax warps of every query tile zero: it waits for all of them.
      if (warp == 1) {
        for (int u = 0; ok && u < ntiles; ++u) {
          ok = mbar_wait_bounded(bar_k_full(u % NS), (u / NS) & 1);
#pragma unroll
          for (int q = 0; q < QT; ++q) {
            if (!ok || u >= ntq[q]) continue;
            // the S buffer of tile u - NSB holds that tile's P until P.V has read it
            if (u >= NSB) ok = mbar_wait_bounded(bar_o(q, u % NSB), ((u - NSB) / NSB) & 1);
            if (!ok) break;
            tc::tc_fence_after();
            issue_s(q, u);
          }
          if (!ok) break;
          tc::umma_commit(bar_k_empty(u % NS));
        }
      } else {
        for (int t = 0; ok && t < ntiles; ++t) {
          const bool last = t == ntiles - 1;
#pragma unroll
          for (int q = 0; q < QT; ++q)
            if (ok && last && t < ntq[q]) ok = mbar_wait_bounded(bar_p(q, t % NSB), (t / NSB) & 1);
          if (ok) ok = mbar_wait_bounded(bar_v_full(t % NS), (t / NS) & 1);
#pragma unroll
          for (int q = 0; q < QT; ++q) {
            if (!ok || t >= ntq[q]) continue;
            if (!last) ok = mbar_wait_bounded(bar_p(q, t % NSB), (t / NSB) & 1);
            if (!ok) break;
            tc::tc_fence_after();
            issue_pv(q, t);
          }
          if (!ok) break;
          tc::umma_commit(bar_v_empty(t % NS));
        }
      }
      if (!ok) set_err(p.err, PKV_DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ---- softmax warps: query tile qg, thread <-> row <-> TMEM lane -------------------
    const int qg = (warp - 3) >> 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + qg * Tr::QCOLS + (static_cast<uint32_t>(quarter * 32) << 16);
    const int crow = qg * M + r;   // row within the CTA
    const bool active = crow < rows_total - tile * ROWS;
    const int j = tok0 + crow / G;
    const int g = crow % G;
    // the last key the row sees, counted from kb
    const int pos = (!active ? -1 : Tr::kPrefix ? ctx - 1 : ctx - q_len + j) - kb;
    const int ctx_r = ctx - kb;
    const int my_tiles = qg == 0 ? ntq[0] : ntq[QT - 1];
    // E4M3: a cached value is code x scale; the K scale folds into the logit
    // scale and the V scale into the final normalisation
    float k_scale = 1.f, v_scale = 1.f;
    if constexpr (Tr::kFp8) {
      k_scale = p.k_scales[kvh];
      v_scale = p.v_scales[kvh];
      if (!(k_scale > 0.f && k_scale < INFINITY && v_scale > 0.f && v_scale < INFINITY) &&
          warp == 3 && lane == 0 && tile == 0)
        set_err(p.err, PKV_DEVERR_BAD_SCALE);
    }
    bool ok = true;
    if constexpr (Tr::kQToFp16) {
      // round this query tile from bf16 to fp16 in place (the MMAs run in
      // fp16 over E4M3 caches); every softmax warp arrives, whatever its rows
      ok = __all_sync(kFullMask, mbar_wait_bounded(bar_q, 0));
      if (ok) {
        unsigned char* qt = smem + Tr::OFF_Q + qg * Tr::Q_TILE;
        for (int idx = r; idx < Tr::Q_TILE / 16; idx += 128) {
          uint4* at = reinterpret_cast<uint4*>(qt + idx * 16);
          const uint4 u = *at;
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
          uint32_t h[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo = fminf(fmaxf(__uint_as_float(w[e] << 16), -65504.f), 65504.f);
            const float hi = fminf(fmaxf(__uint_as_float(w[e] & 0xffff0000u), -65504.f), 65504.f);
            h[e] = pack2(lo, hi, Fp16());
          }
          *at = make_uint4(h[0], h[1], h[2], h[3]);
        }
      }
      fence_proxy_async_smem();  // the MMAs read the tile through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_q_ready);
    }
    float m = -INFINITY, l = 0.f;
    for (int t = 0; ok && t < my_tiles; ++t) {
      const int kv0 = t * NKEY;
      ok = mbar_wait_bounded(bar_s_full(qg, t % NSB), (t / NSB) & 1);
      if (!__all_sync(kFullMask, ok)) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const uint32_t sbuf = lane_addr + (t % NSB) * NKEY;  // this tile's S (then P) columns
      // Scaled logits are x = s * qscale.  For qscale > 0 the row max of x is
      // (max s) * qscale exactly, so s is masked and reduced unscaled and the
      // scale folds into the exponent's FFMA: p = 2^(s * qscale - m).
      const float mult0 = p.qscale * k_scale;
      const float mult = mult0 > 0.f ? mult0 : 1.f;
      // 64 columns of the row from TMEM (half hf of a 128-key tile), masked
      // (and, for a scale <= 0, scaled before the max)
      auto load_half = [&](int hf, float (&v64)[64]) {
#pragma unroll
        for (int c = 0; c < 64; c += 16) {
          float v[16];
          tc::tmem_ld16(sbuf + hf * 64 + c, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) v64[c + i] = v[i];
        }
        tc::tmem_wait_ld();
        const int k0 = kv0 + hf * 64;
        if (mult0 > 0.f) {
          if (k0 + 63 > pos) {  // these keys reach past the row
#pragma unroll
            for (int c = 0; c < 64; ++c) v64[c] = (k0 + c <= pos) ? v64[c] : -INFINITY;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) v64[c] = (k0 + c <= pos) ? v64[c] * mult0 : -INFINITY;
        }
      };
      auto max64 = [&](const float (&v64)[64]) {
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
#pragma unroll
          for (int u = 0; u < 4; ++u) mx4[u] = tc::max3(mx4[u], v64[c + u], v64[c + 4 + u]);
        }
        return fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      };
      float s[64];
      float smax = -INFINITY;
#pragma unroll
      for (int hf = 0; hf < Tr::HALVES; ++hf) {
        // the max pass (with 128-key tiles both halves are read again below)
        load_half(hf, s);
        smax = fmaxf(smax, max64(s));
      }
      const float mx = smax * mult;
      // move the reference max only when this tile would push P above 2^8
      float alpha = 1.f;
      if (active && mx > m + Tr::kRescaleThreshold) {
        alpha = exp2_approx(m - mx);  // 0 on the first tile (m = -inf)
        m = mx;
      }
      const float neg_m = m == -INFINITY ? 0.f : -m;
      // p = 2^(s * mult - m) in fp32 pairs: the same roundings as fmaf and a
      // float sum per chain (four chains: lanes of sum2[0] and sum2[1])
      const uint64_t mult2 = tc::f2_pack(mult, mult), neg_m2 = tc::f2_pack(neg_m, neg_m);
      uint64_t sum2[2] = {tc::f2_pack(0.f, 0.f), tc::f2_pack(0.f, 0.f)};
#pragma unroll
      for (int hf = 0; hf < Tr::HALVES; ++hf) {
        // a 64-key tile is still in registers; each half of a 128-key tile is
        // read again, and its P goes over S columns already read (keys
        // 64 hf .. 64 hf + 63 -> the P columns of groups 4 hf .. 4 hf + 3)
        if (Tr::HALVES > 1) load_half(hf, s);
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float x0, x1;
            tc::f2_unpack(tc::f2_fma(tc::f2_pack(s[c + 2 * h], s[c + 2 * h + 1]), mult2, neg_m2),
                          x0, x1);
            s[c + 2 * h] = exp2_approx(x0);
            s[c + 2 * h + 1] = exp2_approx(x1);
            sum2[h] = tc::f2_add(sum2[h], tc::f2_pack(s[c + 2 * h], s[c + 2 * h + 1]));
          }
        }
        // P (16-bit; bf16 as hi + lo) into TMEM over the S just read, 16 keys
        // (8 columns of 2 values) per group kk
#pragma unroll
        for (int g4 = 0; g4 < 4; g4 += 2) {
          const int kk = 4 * hf + g4;  // two groups: 16 columns per store
          uint32_t w[16], wl[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float a = s[16 * g4 + 2 * e], b = s[16 * g4 + 2 * e + 1];
            w[e] = pack2(a, b, typename Tr::MT());
            if constexpr (Tr::kBf16)
              wl[e] = pack2(a - __uint_as_float(w[e] << 16),
                            b - __uint_as_float(w[e] & 0xffff0000u), Bf16());
          }
          if constexpr (NKEY == 128 && Tr::kBf16) {
            // hi and lo of each group side by side: group kk -> columns
            // 16 kk .. 16 kk + 7 (hi) and 16 kk + 8 .. 16 kk + 15 (lo)
            uint32_t h0[16], h1[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              h0[e] = w[e];
              h0[8 + e] = wl[e];
              h1[e] = w[8 + e];
              h1[8 + e] = wl[8 + e];
            }
            tc::tmem_st16u(sbuf + p_col_hi(kk), h0);
            tc::tmem_st16u(sbuf + p_col_hi(kk + 1), h1);
          } else {
            tc::tmem_st16u(sbuf + p_col_hi(kk), w);
            if constexpr (Tr::kBf16) tc::tmem_st16u(sbuf + p_col_lo(kk), wl);
          }
        }
      }
      tc::tmem_wait_st();
      float sum4[4];
      tc::f2_unpack(sum2[0], sum4[0], sum4[1]);
      tc::f2_unpack(sum2[1], sum4[2], sum4[3]);
      const float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      l = l * alpha + sum;
      if (t > 0 && __any_sync(kFullMask, alpha != 1.f)) {
        // O must hold every earlier tile before it is rescaled
        ok = mbar_wait_bounded(bar_o(qg, (t - 1) % NSB), ((t - 1) / NSB) & 1);
        if (!__all_sync(kFullMask, ok)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 128; c += 16) {
          float v[16];
          tc::tmem_ld16(lane_addr + Tr::O_COL + c, v);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] *= alpha;
          tc::tmem_st16(lane_addr + Tr::O_COL + c, v);
        }
        tc::tmem_wait_st();
      }
      // keys past the context, or not loaded, hold stale data: zero their V rows
      // (every query tile that uses the stage writes the same zeros)
      const int loaded_end = min(kv0 + NKEY, ((nkv_r + 15) / 16) * 16);
      const int vz = min(ctx_r, loaded_end) - kv0;  // V rows [vz, NKEY) must be zero
      if (vz < NKEY) {
        // V of this tile may still be in flight: let it land before zeroing rows
        ok = mbar_wait_bounded(bar_v_full(t % NS), (t / NS) & 1);
        if (!__all_sync(kFullMask, ok)) {
          ok = false;
          break;
        }
        unsigned char* vt = smem + Tr::OFF_KV + (t % NS) * Tr::STAGE + 2 * Tr::KV_HALF;
        const int nrows = NKEY - vz;
        for (int idx = r; idx < nrows * 16; idx += 128) {
          const int row = vz + idx / 16;
          const int part = idx % 16;  // 8 chunks in each of the two dim halves
          *reinterpret_cast<uint4*>(vt + (part >> 3) * Tr::KV_HALF + row * 128 + (part & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p(qg, t % NSB));
    }
    // ---- epilogue ------------------------------------------------------------------------
    if (ok && my_tiles > 0) {
      ok = mbar_wait_bounded(bar_o(qg, (my_tiles - 1) % NSB), ((my_tiles - 1) / NSB) & 1);
      ok = __all_sync(kFullMask, ok);
    }
    if (ok && my_tiles > 0 && Tr::kPrefix) {
      // split-K partial of the prefix: (m, l, unnormalised o) in slot 0
      tc::tc_fence_after();
      const size_t slot = (static_cast<size_t>(q0 + j) * p.num_heads + kvh * G + g) * p.max_parts;
      if (active) {
        if (p.context_lens[q0 + j] < ctx) set_err(p.err, PKV_DEVERR_BAD_CONTEXT);
        p.ws_max[slot] = m;
        p.ws_sum[slot] = l;
      }
#pragma unroll 1
      for (int c = 0; c < 128; c += 16) {
        float v[16];
        tc::tmem_ld16(lane_addr + Tr::O_COL + c, v);
        tc::tmem_wait_ld();
        if (active) {
          // E4M3: the V scale goes into o (m and l do not hold it)
          float4* o = reinterpret_cast<float4*>(p.ws_out + slot * Tr::D + c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            o[i] = make_float4(v[4 * i] * v_scale, v[4 * i + 1] * v_scale, v[4 * i + 2] * v_scale,
                               v[4 * i + 3] * v_scale);
        }
      }
    } else if (ok && my_tiles > 0 && !Tr::kPrefix && p.work != nullptr &&
               p.work[static_cast<size_t>(rank) * kPlanItemInts + 6] > 1) {
      // a piece of a planned unit: its partial for the merge kernel (the
      // item is read again here rather than held in registers all along)
      const int32_t* it = p.work + static_cast<size_t>(rank) * kPlanItemInts;
      const size_t slot =
          ((static_cast<size_t>(it[5]) * p.num_kv_heads + kvh) * ROWS + crow) * kMaxPieces + it[4];
      if (active) {
        p.ws_max[slot] = m;
        p.ws_sum[slot] = l;
      }
      float4* dst = reinterpret_cast<float4*>(p.ws_out + slot * Tr::D);
      tc::tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 128; c += 16) {
        float v[16];
        tc::tmem_ld16(lane_addr + Tr::O_COL + c, v);
        tc::tmem_wait_ld();
        if (active) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[c / 4 + i] = make_float4(v[4 * i] * v_scale, v[4 * i + 1] * v_scale,
                                         v[4 * i + 2] * v_scale, v[4 * i + 3] * v_scale);
        }
      }
    } else if (ok && my_tiles > 0) {
      tc::tc_fence_after();
      const float inv = l > 0.f ? v_scale / l : 0.f;
      T* orow = static_cast<T*>(p.out) +
                (static_cast<size_t>(q0 + j) * p.num_heads + kvh * G + g) * Tr::D;
#pragma unroll 1
      for (int c = 0; c < 128; c += 16) {
        float v[16];
        tc::tmem_ld16(lane_addr + Tr::O_COL + c, v);
        tc::tmem_wait_ld();
        if (active) {
          float a[8], b[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            a[i] = v[i] * inv;
            b[i] = v[8 + i] * inv;
          }
          *reinterpret_cast<uint4*>(orow + c) = pack8(a, DT());
          *reinterpret_cast<uint4*>(orow + c + 8) = pack8(b, DT());
        }
      }
    } else if (!ok) {
      if (lane == 0) set_err(p.err, PKV_DEVERR_TIMEOUT);
    }
  }
  // ---- release TMEM (every path reaches here) ---------------------------------------------
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, Tr::TMEM_COLS);
  }
}

// Merge of a planned unit's pieces (the same combination the decode reduce
// makes of split-K partitions): for each (token, head) row of the unit,
//   out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s,   M = max_s m_s.
// A warp per row, each lane 4 of the 128 dims; CTA b serves rows
// 8 (b % R8) .. 8 (b % R8) + 7 of entry (b / R8) / H_kv for kv head
// (b / R8) % H_kv, R8 = unit_rows / 8, so every row's loads are in flight at
// once.  Launched after the planned prefill kernel, whose partials it waits
// for in griddepcontrol.wait.
template <class DT>
__global__ void __launch_bounds__(256) paged_prefill_merge_kernel(const PrefillParams p) {
  using T = typename DT::T;
  constexpr int D = 128;
  grid_dependency_wait();
  trigger_dependents();
  const int r8 = p.unit_rows / 8;
  const int unit = static_cast<int>(blockIdx.x) / r8;
  const int e = unit / p.num_kv_heads;
  const int kvh = unit % p.num_kv_heads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = (static_cast<int>(blockIdx.x) % r8) * 8 + warp;
  const int32_t* me = p.merges + 4 * static_cast<size_t>(e);
  const int seq = me[0], tile = me[1], pieces = me[2];
  if (static_cast<unsigned>(seq) >= static_cast<unsigned>(p.num_seqs) || pieces < 2 ||
      pieces > kMaxPieces || tile < 0) {
    if (threadIdx.x == 0) set_err(p.err, PKV_DEVERR_BAD_ORDER);
    return;
  }
  const int group = p.num_heads / p.num_kv_heads;
  const int q0 = p.query_start[seq];
  const int q_len = p.query_start[seq + 1] - q0;
  const int nrows = min(p.unit_rows, q_len * group - tile * p.unit_rows);
  if (q_len <= 0 || q_len > p.max_query_len || nrows <= 0) {
    if (threadIdx.x == 0) set_err(p.err, PKV_DEVERR_BAD_ORDER);
    return;
  }
  if (r >= nrows) return;
  const size_t base =
      ((static_cast<size_t>(e) * p.num_kv_heads + kvh) * p.unit_rows + r) * kMaxPieces;
  float ms[kMaxPieces], ls[kMaxPieces];
  float4 os[kMaxPieces];
#pragma unroll
  for (int s = 0; s < kMaxPieces; ++s) {
    if (s < pieces) {
      ms[s] = p.ws_max[base + s];
      ls[s] = p.ws_sum[base + s];
      os[s] = *reinterpret_cast<const float4*>(p.ws_out + (base + s) * D + lane * 4);
    }
  }
  float big_m = -INFINITY;
#pragma unroll
  for (int s = 0; s < kMaxPieces; ++s)
    if (s < pieces) big_m = fmaxf(big_m, ms[s]);
  float num[4] = {0.f, 0.f, 0.f, 0.f};
  float den = 0.f;
#pragma unroll
  for (int s = 0; s < kMaxPieces; ++s) {
    if (s < pieces) {
      const float f = ms[s] == -INFINITY ? 0.f : exp2_approx(ms[s] - big_m);
      den = fmaf(f, ls[s], den);
      num[0] = fmaf(f, os[s].x, num[0]);
      num[1] = fmaf(f, os[s].y, num[1]);
      num[2] = fmaf(f, os[s].z, num[2]);
      num[3] = fmaf(f, os[s].w, num[3]);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const int row = tile * p.unit_rows + r;
  T* out = static_cast<T*>(p.out) +
           (static_cast<size_t>(q0 + row / group) * p.num_heads + kvh * group + row % group) * D +
           lane * 4;
  *reinterpret_cast<uint2*>(out) =
      make_uint2(pack2(num[0] * inv, num[1] * inv, DT()), pack2(num[2] * inv, num[3] * inv, DT()));
}

}  // namespace pkv
