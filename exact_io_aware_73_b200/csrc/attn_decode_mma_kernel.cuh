// attn_decode_mma_kernel.cuh -- split-KV decode on the tensor cores for
// B200 (sm_100a), d = 64 or 128, up to 16 queries per head.
//
// Source: the briefgpt.xyz summary page of FlashAttention-2 (arXiv
// 2307.08691), entry "LeanAttention": the decode phase of long contexts is
// computed in parallel over the key/value sequence.  Same result as
// attn_decode_kernel (exact attention of Nq new queries, the last Nq
// positions, against Nk keys; causal: query i sees keys 0 .. Nk - Nq + i),
// for Nq <= 16.
//
// The CUDA-core decode keeps at most 4 queries in registers and streams K/V
// once per group of 4.  Here one pass over K/V serves up to 16 queries, and
// both contractions run on tcgen05 with the roles of the operands turned
// around, so that the M = 128 side of the MMA is the key tile (and the head
// dimension), never the handful of queries:
//   * a tile is 32 KB of K and 32 KB of V: 128 keys at d = 128, 256 at
//     d = 64 (so that a tile's fixed cost -- waits, barrier, reductions,
//     commits -- is spread over as many bytes as at d = 128);
//   * S^T = K Q^T per 128-key block of the tile: M = 128 keys, N = 16 query
//     columns (Q rows beyond Nq are zero), K = d; A = the K block and B = Q,
//     both K-major with the 128-byte swizzle, exactly as the TMA writes
//     them.  Softmax thread t (warp t / 32 reads TMEM lanes 32 (t / 32) ..)
//     owns key t of each block and holds its 16 scores per block;
//   * per query, the tile maximum over its keys (a warp max reduction, then
//     the four warps through shared memory); the reference maximum moves
//     lazily as in the forward kernel (only when a score exceeds it by more
//     than 2^8, which every thread decides identically), O^T is then
//     rescaled in TMEM;
//   * p = 2^(s scale log2(e) - m) rounded to bf16 and written to shared
//     memory as a 16-row K-major tile of the tile's keys (64-key panels,
//     128-byte swizzle); each thread adds its keys' p to its own part of
//     every query's row sum;
//   * O^T += V^T P^T per 128-key block: at d = 128, M = d (the V block read
//     MN-major), N = 16, K = 128 keys.  At d = 64 the block's two 64-key
//     halves stand side by side instead: M = 128 holds the 64 dimensions of
//     the first half's keys and then of the second half's (the V block's
//     two halves, 8 KB apart), N = 32 holds P of the first half's keys for
//     the 16 queries and then of the second half's (the block's 4 KB of P
//     read as 32 rows of 64 keys), K = 64 keys; the quadrants (dims 0-63,
//     columns 0-15) and (dims 64-127, columns 16-31) are the two halves'
//     sums, added at the end of the part, and the other two quadrants are
//     not used.  O^T accumulates in TMEM over the tiles of a head part;
//   * at the end of a part the row-sum parts are added, O^T is read back
//     (thread = dimension, so every query's row is stored coalesced) and
//     written out, or recorded as a part and merged exactly by the CTA that
//     finishes the head's last part: lse = log sum_s exp(lse_s),
//     O = sum_s exp(lse_s - lse) O_s.
// Work split: stream-K over the key tiles of all heads, an equal share per
// CTA, one CTA per SM (the three-stage ring of 64 KB K/V tiles fills the
// shared memory).  Roles: warps 0-3 softmax, warp 4 TMA loader (one lane),
// warp 5 MMA issuer (one lane) and TMEM owner.  TMEM: two S^T buffers (16
// columns per 128-key block) and O^T (16 columns, or 32 at d = 64).  The MMA
// thread issues S^T of tile i + 1 before O^T of tile i, so the softmax of one
// tile overlaps the other's P.V.  Every wait is bounded; a wait that runs
// out flags the device status word, the CTA drains its in-flight copies and
// MMAs, frees its TMEM and leaves without writing.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <math_constants.h>

#include "attn_fwd_kernel.cuh"

namespace attn_b200 {

constexpr int kDmQ = 16;        // query columns per head (padded)
constexpr int kDmBlock = 128;   // keys per S^T MMA (its M)
constexpr int kDmSoftmaxThreads = 128;
constexpr int kDmThreads = kDmSoftmaxThreads + 64;  // + loader warp + MMA warp
constexpr int kDmLoaderWarp = 4, kDmMmaWarp = 5;
constexpr uint32_t kDmTmemCols = 128;  // S^T x 2 (16 or 32 each), O^T (16 or 32)
constexpr int kDmMaxCtas = 1024;      // bound on the grid (workspace sizing)
constexpr float kDmLazy = 8.f;        // log2 units: p <= 2^8

template <int D>
struct DmSmem {
  // keys per tile: 32 KB of K (and of V) either way, so that the fixed cost
  // of a tile (waits, barrier, reductions, commits) is spread over as many
  // bytes at d = 64 as at d = 128
  static constexpr int kKeys = (D == 64) ? 256 : 128;
  static constexpr int kBlocks = kKeys / kDmBlock;        // S^T MMAs per tile
  static constexpr int kSub = D / 64;                     // 128-byte panels per row
  static constexpr uint32_t kPanel = 128 * 128;           // 128 rows x 128 B
  static constexpr uint32_t kTile = kBlocks * kSub * kPanel;  // a K or V tile (32 KB)
  static constexpr uint32_t kSmallPanel = kDmQ * 128;     // 16 rows x 128 B
  static constexpr uint32_t kQTile = kSub * kSmallPanel;  // Q: 16 rows x D
  static constexpr uint32_t kPTile = (kKeys / 64) * kSmallPanel;  // P: 16 rows x kKeys
  static constexpr int kScols = kBlocks * kDmQ;           // TMEM columns of one S^T
  static constexpr int kStages = 3;
  static constexpr uint32_t kK = 0;                       // K ring
  static constexpr uint32_t kV = kK + kStages * kTile;    // V ring
  static constexpr uint32_t kQ = kV + kStages * kTile;    // 2 Q buffers
  static constexpr uint32_t kP = kQ + 2 * kQTile;         // 2 P buffers
  static constexpr uint32_t kRed = kP + 2 * kPTile;       // [2][4 warps][16] tile maxima
  static constexpr uint32_t kStat = kRed + 2 * 4 * kDmQ * 4;  // [4 warps][16] row sums
  static constexpr uint32_t kBars = kStat + 4 * kDmQ * 4;
  static constexpr int KV_FULL = 0, KV_EMPTY = kStages, Q_FULL = 2 * kStages,
                       Q_EMPTY = Q_FULL + 2, S_FULL = Q_EMPTY + 2, S_EMPTY = S_FULL + 2,
                       P_FULL = S_EMPTY + 2, P_EMPTY = P_FULL + 2, DRAIN = P_EMPTY + 2,
                       NUM_BARS = DRAIN + 1;
  static constexpr uint32_t kMisc = kBars + NUM_BARS * 8;  // tmem slot, abort, last flag
  static constexpr uint32_t kBytes = kMisc + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kQ % 1024 == 0 && kP % 1024 == 0, "swizzle atoms are 1024-byte aligned");
  static_assert(kAlloc <= 232448, "shared memory budget");
};

struct DecodeMmaParams {
  uint16_t *o;         // [BH, Nq, D]
  float *lse;          // [BH, Nq]
  float *part_o;       // [slots, Nq, D] partial outputs (normalised)
  float *part_lse;     // [slots, Nq]
  int *counters;       // [BH] parts finished per head (zero at launch)
  uint32_t *status;
  int bh, nq, nk;
  int ntiles;          // key tiles per head
  int total;           // bh * ntiles
  int per_cta;         // tiles per CTA
  int causal;
  float c_log2;        // scale * log2(e)
  unsigned long long timeout_ns;
  uint32_t debug_flags;  // bit 1: CTA 0's loader skips its first K/V tile
};

__device__ __forceinline__ int dm_first_cta(int h, const DecodeMmaParams &p) {
  return static_cast<int>((static_cast<int64_t>(h) * p.ntiles) / p.per_cta);
}
__device__ __forceinline__ int dm_last_cta(int h, const DecodeMmaParams &p) {
  return static_cast<int>((static_cast<int64_t>(h + 1) * p.ntiles - 1) / p.per_cta);
}

// The 128 softmax threads meet at named barrier 1; the result is the AND of
// their predicates (so that a thread whose wait ran out takes all of them
// out of the loop together).
__device__ __forceinline__ bool dm_bar_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "n"(kDmSoftmaxThreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
        "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
        "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
        "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])::"memory");
}

// Byte offset of element (row, col) in a K-major bf16 tile of `rows` rows
// and 128 columns stored as two 64-column panels with the 128-byte swizzle
// (the 16-byte chunk index within a 128-byte row is XORed with row % 8; the
// layout the TMA writes and the UMMA descriptors read).
__device__ __forceinline__ uint32_t sw128_offset(int rows, int row, int col) {
  const int panel = col >> 6, c = col & 63;
  return static_cast<uint32_t>(panel * rows * 128 + row * 128 +
                               ((((c >> 3) ^ (row & 7)) << 4) | ((c & 7) << 1)));
}

// ------------------------------------------------------------------ loader

template <int D>
__device__ __forceinline__ void dm_loader(uint32_t base, const CUtensorMap *tq,
                                          const CUtensorMap *tk, const CUtensorMap *tv,
                                          const DecodeMmaParams &p, const WaitCtx &wc,
                                          int g0, int g1) {
  using L = DmSmem<D>;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };
  int tc = 0, qc = 0;
  bool ok = true;
  // injected fault: the first tile's copies are never issued, so the MMA
  // thread's wait for it must run out (its stage is then not drained)
  const int skipped = ((p.debug_flags & 2u) && blockIdx.x == 0) ? 0 : -1;
  const uint64_t pol_kv = policy_evict_first();  // every K/V byte is read once
  for (int g = g0; ok && g < g1;) {
    const int h = g / p.ntiles;
    const int gend = min(g1, (h + 1) * p.ntiles);
    const int qb = qc & 1;
    ok = mbar_wait(bar(L::Q_EMPTY + qb), ((qc >> 1) & 1) ^ 1, wc, kRoleProducer);
    if (!ok) break;
    mbar_arrive_expect_tx(bar(L::Q_FULL + qb), L::kQTile);
    for (int s = 0; s < L::kSub; ++s)
      tma_load_3d(base + L::kQ + qb * L::kQTile + s * L::kSmallPanel, tq,
                  bar(L::Q_FULL + qb), s * 64, 0, h);
    ++qc;
    for (int gg = g; gg < gend; ++gg) {
      const int j = gg - h * p.ntiles;
      const int st = tc % L::kStages;
      ok = mbar_wait(bar(L::KV_EMPTY + st), ((tc / L::kStages) & 1) ^ 1, wc,
                     kRoleProducer);
      if (!ok) break;
      if (tc == skipped) {
        ++tc;
        continue;
      }
      mbar_arrive_expect_tx(bar(L::KV_FULL + st), 2 * L::kTile);
      // block b (128 keys) of the tile, panel s (64 dimensions)
      for (int b = 0; b < L::kBlocks; ++b)
        for (int s = 0; s < L::kSub; ++s) {
          const uint32_t off = st * L::kTile + (b * L::kSub + s) * L::kPanel;
          const int row = j * L::kKeys + b * kDmBlock;
          tma_load_3d_hint(base + L::kK + off, tk, bar(L::KV_FULL + st), s * 64, row, h,
                           pol_kv);
          tma_load_3d_hint(base + L::kV + off, tv, bar(L::KV_FULL + st), s * 64, row, h,
                           pol_kv);
        }
      ++tc;
    }
    g = gend;
  }
  if (*wc.abort) {
    // every copy issued must land before the CTA may exit
    for (int b = 0; b < 2; ++b)
      if (qc > b) {
        const int last = b + ((qc - 1 - b) / 2) * 2;
        mbar_wait_drain(bar(L::Q_FULL + b), (last >> 1) & 1, wc);
      }
    for (int st = 0; st < L::kStages; ++st)
      if (tc > st) {
        const int last = st + ((tc - 1 - st) / L::kStages) * L::kStages;
        if (last == skipped) continue;  // nothing was copied for it
        mbar_wait_drain(bar(L::KV_FULL + st), (last / L::kStages) & 1, wc);
      }
  }
}

// ------------------------------------------------------------------ MMA

// S^T[128 keys x 16] = K[128 x D] Q[16 x D]^T; both K-major, 128-byte
// swizzle; one instruction per 16 dimensions.
template <int D>
__device__ __forceinline__ void dm_issue_s(uint32_t d_tmem, uint32_t k_smem,
                                           uint32_t q_smem) {
  constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                             ((uint32_t)(kDmQ >> 3) << 17) |
                             ((uint32_t)(kDmBlock >> 4) << 24);
  const uint64_t kd = smem_desc_sw128(k_smem, 16, 1024);
  const uint64_t qd = smem_desc_sw128(q_smem, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t ka = ((kk >> 2) * DmSmem<D>::kPanel + (kk & 3) * 32) >> 4;
    const uint64_t qa = ((kk >> 2) * DmSmem<D>::kSmallPanel + (kk & 3) * 32) >> 4;
    mma_bf16_ss(d_tmem, kd + ka, qd + qa, idesc, kk > 0);
  }
}

// d = 128: O^T[128 dims x 16] (+)= V^T[128 x 128 keys] P^T[128 keys x 16]:
// A = the V tile read MN-major (the dimension contiguous; 64-dimension
// panels kPanel bytes apart, 8-key groups 1024 bytes apart), B = P K-major
// (16 query rows of 128 keys, two 64-key panels).  One instruction per 16
// keys.
// d = 64: O2[128 x 32] (+)= A[128 x 64 keys] B[64 keys x 32] with A rows
// 0-63 = the dimensions of keys 0-63 and rows 64-127 = those of keys
// 64-127 (the V tile's two halves, 64 rows x 128 B = 8 KB apart, as the two
// M panels), B columns 0-15 = P of keys 0-63 and 16-31 = P of keys 64-127
// (P's two 64-key panels read as one 32-row panel: row 16 + q of the second
// starts 2 KB after row q of the first and has the same swizzle phase).
// One instruction per 16 keys of each half.
template <int D>
__device__ __forceinline__ void dm_issue_o(uint32_t d_tmem, uint32_t v_smem,
                                           uint32_t p_smem, bool accumulate) {
  constexpr int kN = (D == 128) ? kDmQ : 2 * kDmQ;
  constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                             (1u << 15)  // A: MN-major
                             | ((uint32_t)(kN >> 3) << 17) |
                             ((uint32_t)(128 >> 4) << 24);
  constexpr uint32_t kLbo = (D == 128) ? DmSmem<D>::kPanel : 64 * 128;
  const uint64_t vd = smem_desc_sw128(v_smem, kLbo, 1024);
  const uint64_t pd = smem_desc_sw128(p_smem, 16, 1024);
  constexpr int kSteps = (D == 128) ? kDmBlock / 16 : kDmBlock / 32;
#pragma unroll
  for (int kk = 0; kk < kSteps; ++kk) {
    const uint64_t va = static_cast<uint64_t>((kk * 16 * 128) >> 4);
    const uint64_t pa = (D == 128)
        ? (((kk >> 2) * DmSmem<D>::kSmallPanel + (kk & 3) * 32) >> 4)
        : static_cast<uint64_t>((kk * 32) >> 4);
    mma_bf16_ss(d_tmem, vd + va, pd + pa, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void dm_mma(uint32_t base, uint32_t tmem,
                                       const DecodeMmaParams &p, const WaitCtx &wc,
                                       int g0, int g1) {
  using L = DmSmem<D>;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };
  const uint32_t tO = tmem + 2 * L::kScols;
  int tc = 0, qc = 0;
  bool ok = true;
  // O^T of global tile `t` (the i-th of its part), one MMA group per
  // 128-key block; releases P buffer t & 1 and the tile's K/V stage.
  auto issue_o = [&](int t, bool accumulate) -> bool {
    const int pb = t & 1;
    if (!mbar_wait_spin(bar(L::P_FULL + pb), (t >> 1) & 1, wc, kRoleMma)) return false;
    tc_fence_after_sync();
    const int st = t % L::kStages;
#pragma unroll
    for (int b = 0; b < L::kBlocks; ++b)
      dm_issue_o<D>(tO, base + L::kV + st * L::kTile + b * L::kSub * L::kPanel,
                    base + L::kP + pb * L::kPTile + b * 2 * L::kSmallPanel,
                    accumulate || b > 0);
    mma_commit(bar(L::P_EMPTY + pb));
    mma_commit(bar(L::KV_EMPTY + st));
    return true;
  };
  for (int g = g0; ok && g < g1;) {
    const int h = g / p.ntiles;
    const int gend = min(g1, (h + 1) * p.ntiles);
    const int qb = qc & 1;
    ok = mbar_wait_spin(bar(L::Q_FULL + qb), (qc >> 1) & 1, wc, kRoleMma);
    if (!ok) break;
    const int n = gend - g;
    for (int i = 0; i < n; ++i, ++tc) {
      const int st = tc % L::kStages, sb = tc & 1;
      ok = mbar_wait_spin(bar(L::KV_FULL + st), (tc / L::kStages) & 1, wc, kRoleMma);
      if (!ok) break;
      ok = mbar_wait_spin(bar(L::S_EMPTY + sb), ((tc >> 1) & 1) ^ 1, wc, kRoleMma);
      if (!ok) break;
      tc_fence_after_sync();
#pragma unroll
      for (int b = 0; b < L::kBlocks; ++b)
        dm_issue_s<D>(tmem + sb * L::kScols + b * kDmQ,
                      base + L::kK + st * L::kTile + b * L::kSub * L::kPanel,
                      base + L::kQ + qb * L::kQTile);
      mma_commit(bar(L::S_FULL + sb));
      if (i == n - 1) mma_commit(bar(L::Q_EMPTY + qb));  // last read of this Q
      if (i > 0) {
        ok = issue_o(tc - 1, i > 1);
        if (!ok) break;
      }
    }
    if (!ok) break;
    ok = issue_o(tc - 1, n > 1);
    ++qc;
    g = gend;
  }
  // All tensor-core work must finish before TMEM is released.
  mma_commit(bar(L::DRAIN));
  mbar_wait_drain(bar(L::DRAIN), 0, wc);
}

// ------------------------------------------------------------------ softmax

template <int D>
__device__ __forceinline__ void dm_softmax(uint32_t base, uint8_t *smem, uint32_t tmem,
                                           const DecodeMmaParams &p, const WaitCtx &wc,
                                           int g0, int g1, int warp, int lane) {
  using L = DmSmem<D>;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };
  const int tid = warp * 32 + lane;  // key of the tile / output dimension
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tO = tmem + lane_base + 2 * L::kScols;
  constexpr int KB = L::kBlocks;  // keys of the tile this thread owns: tid + 128 b
  float *red = reinterpret_cast<float *>(smem + L::kRed);
  float *stat = reinterpret_cast<float *>(smem + L::kStat);
  volatile int *last_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 8);
  int tc = 0;
  for (int g = g0; g < g1;) {
    const int h = g / p.ntiles;
    const int gend = min(g1, (h + 1) * p.ntiles);
    float m[kDmQ], l[kDmQ];
#pragma unroll
    for (int q = 0; q < kDmQ; ++q) {
      m[q] = -CUDART_INF_F;
      l[q] = 0.f;
    }
    // A wait that runs out sets `fail` (warp-uniform) for good; the next
    // barrier then takes every softmax thread out together.
    bool fail = false;
    for (int gg = g; gg < gend; ++gg, ++tc) {
      const int j = gg - h * p.ntiles;
      const int sb = tc & 1;
      // 1. the 16 scores of each of this thread's keys
      uint32_t sr[KB][16];
#pragma unroll
      for (int b = 0; b < KB; ++b)
#pragma unroll
        for (int q = 0; q < kDmQ; ++q) sr[b][q] = 0u;
      if (!fail)
        fail = !__all_sync(0xffffffffu, mbar_wait(bar(L::S_FULL + sb), (tc >> 1) & 1, wc,
                                                  kRoleSoftmax));
      if (!fail) {
        tc_fence_after_sync();
#pragma unroll
        for (int b = 0; b < KB; ++b) {
          tmem_ld_32x32b_x16(tmem + lane_base + sb * L::kScols + b * kDmQ, sr[b]);
          tmem_wait_ld16(sr[b]);
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::S_EMPTY + sb));
      }
      const int key0 = j * L::kKeys + tid;
      const bool tail = (j + 1) * L::kKeys > p.nk - (p.causal ? p.nq : 0);  // uniform
      float x[KB][kDmQ];
#pragma unroll
      for (int b = 0; b < KB; ++b) {
        const int key = key0 + b * kDmBlock;
#pragma unroll
        for (int q = 0; q < kDmQ; ++q) {
          x[b][q] = __uint_as_float(sr[b][q]) * p.c_log2;
          if (tail && (key >= p.nk || (p.causal && key > p.nk - p.nq + q)))
            x[b][q] = -CUDART_INF_F;
        }
      }
      // 2. per query, the tile's maximum over its keys
      float *rb = red + sb * (4 * kDmQ);
#pragma unroll
      for (int q = 0; q < kDmQ; ++q) {
        float xm = x[0][q];
#pragma unroll
        for (int b = 1; b < KB; ++b) xm = fmaxf(xm, x[b][q]);
        const float wm = warp_max_f32(xm);
        if (lane == q) rb[warp * kDmQ + q] = wm;
      }
      if (!dm_bar_and(!fail)) {
        fail = true;
        break;
      }
      bool rescale = false;
      float alpha[kDmQ];
#pragma unroll
      for (int q4 = 0; q4 < kDmQ; q4 += 4) {
        float4 a[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) a[w] = *reinterpret_cast<const float4 *>(rb + w * kDmQ + q4);
        const float tmx[4] = {fmaxf(fmaxf(a[0].x, a[1].x), fmaxf(a[2].x, a[3].x)),
                              fmaxf(fmaxf(a[0].y, a[1].y), fmaxf(a[2].y, a[3].y)),
                              fmaxf(fmaxf(a[0].z, a[1].z), fmaxf(a[2].z, a[3].z)),
                              fmaxf(fmaxf(a[0].w, a[1].w), fmaxf(a[2].w, a[3].w))};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = q4 + e;
          alpha[q] = 1.f;
          if (tmx[e] > m[q] + kDmLazy) {  // false while the tile sees no key of q
            if (m[q] != -CUDART_INF_F) {
              alpha[q] = ex2_approx(m[q] - tmx[e]);
              rescale = true;
            }
            m[q] = tmx[e];
            l[q] *= alpha[q];
          }
        }
      }
      // 3. probabilities, row-sum parts, P into its shared-memory buffer
      const int pb = tc & 1;
      fail = !__all_sync(0xffffffffu, mbar_wait(bar(L::P_EMPTY + pb), ((tc >> 1) & 1) ^ 1,
                                                wc, kRoleSoftmax));
      if (fail) continue;  // the next barrier takes every thread out
      uint8_t *pt = smem + L::kP + pb * L::kPTile;
#pragma unroll
      for (int b = 0; b < KB; ++b)
#pragma unroll
        for (int q = 0; q < kDmQ; ++q) {
          const float pq = (m[q] == -CUDART_INF_F) ? 0.f : ex2_approx(x[b][q] - m[q]);
          l[q] += pq;
          *reinterpret_cast<uint16_t *>(pt + sw128_offset(kDmQ, q, tid + b * kDmBlock)) =
              static_cast<uint16_t>(pack_bf16x2(pq, 0.f) & 0xFFFFu);
        }
      fence_proxy_async_smem();
      if (rescale) {  // uniform: every thread took the same decision
        // O^T must hold the previous tile's P.V before it is rescaled
        fail = !__all_sync(0xffffffffu, mbar_wait(bar(L::P_EMPTY + ((tc - 1) & 1)),
                                                  ((tc - 1) >> 1) & 1, wc, kRoleSoftmax));
        if (fail) continue;
        tc_fence_after_sync();
#pragma unroll
        for (int c = 0; c < ((D == 128) ? 1 : 2); ++c) {  // column n holds query n % 16
          uint32_t o[16];
          tmem_ld_32x32b_x16(tO + c * kDmQ, o);
          tmem_wait_ld16(o);
#pragma unroll
          for (int q = 0; q < kDmQ; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha[q]);
          tmem_st_32x32b_x16(tO + c * kDmQ, o);
        }
        tmem_wait_st();
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::P_FULL + pb));
    }
    if (!dm_bar_and(!fail)) return;  // a wait ran out: every softmax thread leaves

    // ---- end of the head part: row sums, O^T out of TMEM, store or merge
#pragma unroll
    for (int q = 0; q < kDmQ; ++q) {
      float t = l[q];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
      if (lane == q) stat[warp * kDmQ + q] = t;
    }
    const int last_t = tc - 1;
    fail = !__all_sync(0xffffffffu, mbar_wait(bar(L::P_EMPTY + (last_t & 1)),
                                              (last_t >> 1) & 1, wc, kRoleEpilogue));
    if (!dm_bar_and(!fail)) return;
    uint32_t o[16];
    tc_fence_after_sync();
    if constexpr (D == 128) {
      tmem_ld_32x32b_x16(tO, o);  // O^T row `tid` = dimension tid
      tmem_wait_ld16(o);
    } else {
      // dimension t: lane t, columns 0-15 (keys 0-63 of every tile) plus
      // lane 64 + t, columns 16-31 (keys 64-127); warps 2-3 hand their
      // quadrant over through the P buffers (free: every P.V is done)
      tmem_ld_32x32b_x16(tO + (warp >= 2 ? kDmQ : 0), o);
      tmem_wait_ld16(o);
      float *xch = reinterpret_cast<float *>(smem + L::kP);  // [16][64]
      if (warp >= 2) {
#pragma unroll
        for (int q = 0; q < kDmQ; ++q) xch[q * 64 + tid - 64] = __uint_as_float(o[q]);
      }
      dm_bar_and(true);
      if (warp < 2) {
#pragma unroll
        for (int q = 0; q < kDmQ; ++q)
          o[q] = __float_as_uint(__uint_as_float(o[q]) + xch[q * 64 + tid]);
      }
    }
    const int first = dm_first_cta(h, p), last = dm_last_cta(h, p);
    const bool whole = first == last;
    const int slot = h + static_cast<int>(blockIdx.x);
    const int64_t row0 = static_cast<int64_t>(h) * p.nq;
#pragma unroll
    for (int q = 0; q < kDmQ; ++q) {
      if (q >= p.nq) break;
      const float lsum = stat[q] + stat[kDmQ + q] + stat[2 * kDmQ + q] + stat[3 * kDmQ + q];
      const bool any = lsum > 0.f;  // a part may see no key of a causal row
      const float val = any ? __uint_as_float(o[q]) * __frcp_rn(lsum) : 0.f;
      const float lse2 = any ? m[q] + lg2_approx(lsum) : -CUDART_INF_F;  // log2 units
      if (tid >= D) continue;  // d = 64: warps 2-3 hold no dimension now
      if (whole) {
        p.o[(row0 + q) * D + tid] = static_cast<uint16_t>(pack_bf16x2(val, 0.f) & 0xFFFFu);
        if (tid == q) p.lse[row0 + q] = lse2 * kLn2;
      } else {
        p.part_o[(static_cast<int64_t>(slot) * p.nq + q) * D + tid] = val;
        if (tid == q)
          p.part_lse[static_cast<int64_t>(slot) * p.nq + q] = any ? lse2 * kLn2 : -CUDART_INF_F;
      }
    }
    if (!whole) {
      __threadfence();  // the part is visible device-wide before it is counted
      dm_bar_and(true);
      if (tid == 0) *last_flag = (atomicAdd(p.counters + h, 1) == last - first);
      dm_bar_and(true);
      if (*last_flag) {
        __threadfence();
        // One pass over the head's parts with a running maximum: thread t
        // combines dimensions 4 (t % C) .. + 3 of queries t / C + G r (C =
        // D / 4 float4 per row, G = 128 / C query groups, R = 16 / G
        // queries each); the loads of one part are independent, so they are
        // in flight together.
        constexpr int C = D / 4, G = kDmSoftmaxThreads / C, R = kDmQ / G;
        const int nseg = last - first + 1;
        const int c4 = tid % C, qg = tid / C;
        float M[R], S[R];
        float4 A[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          M[r] = -CUDART_INF_F;
          S[r] = 0.f;
          A[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll 2
        for (int sgi = 0; sgi < nseg; ++sgi) {
          const int64_t slot_row = static_cast<int64_t>(h + first + sgi) * p.nq;
          float ls[R];
          float4 po[R];
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const int q = qg + G * r;
            ls[r] = -CUDART_INF_F;
            po[r] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (q < p.nq) {
              ls[r] = __ldcg(p.part_lse + slot_row + q);
              po[r] = __ldcg(reinterpret_cast<const float4 *>(p.part_o + (slot_row + q) * D) + c4);
            }
          }
#pragma unroll
          for (int r = 0; r < R; ++r) {
            if (ls[r] == -CUDART_INF_F) continue;  // the part saw no key of the query
            if (ls[r] > M[r]) {
              const float sc = ex2_approx((M[r] - ls[r]) * 1.4426950408889634f);  // 0 at first
              S[r] *= sc;
              A[r].x *= sc; A[r].y *= sc; A[r].z *= sc; A[r].w *= sc;
              M[r] = ls[r];
            }
            const float wgt = ex2_approx((ls[r] - M[r]) * 1.4426950408889634f);
            S[r] += wgt;
            A[r].x = fmaf(wgt, po[r].x, A[r].x);
            A[r].y = fmaf(wgt, po[r].y, A[r].y);
            A[r].z = fmaf(wgt, po[r].z, A[r].z);
            A[r].w = fmaf(wgt, po[r].w, A[r].w);
          }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int q = qg + G * r;
          if (q >= p.nq) continue;
          const float inv = __frcp_rn(S[r]);
          reinterpret_cast<uint2 *>(p.o + (row0 + q) * D)[c4] =
              make_uint2(pack_bf16x2(A[r].x * inv, A[r].y * inv),
                         pack_bf16x2(A[r].z * inv, A[r].w * inv));
          if (c4 == 0) p.lse[row0 + q] = M[r] + lg2_approx(S[r]) * kLn2;
        }
        if (tid == 0) p.counters[h] = 0;  // ready for the next launch
      }
    }
    g = gend;
  }
}

// ------------------------------------------------------------------ kernel

template <int D>
__global__ void __launch_bounds__(kDmThreads, 1)
    attn_decode_mma_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const DecodeMmaParams p) {
  using L = DmSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    const uint32_t b0 = base + L::kBars;
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(b0 + 8 * (L::KV_FULL + s), 1);
      mbar_init(b0 + 8 * (L::KV_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b0 + 8 * (L::Q_FULL + b), 1);
      mbar_init(b0 + 8 * (L::Q_EMPTY + b), 1);
      mbar_init(b0 + 8 * (L::S_FULL + b), 1);
      mbar_init(b0 + 8 * (L::S_EMPTY + b), 4);
      mbar_init(b0 + 8 * (L::P_FULL + b), 4);
      mbar_init(b0 + 8 * (L::P_EMPTY + b), 1);
    }
    mbar_init(b0 + 8 * L::DRAIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kDmMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kDmTmemCols);
    tmem_relinquish_alloc_permit();
  }
  if (warp == kDmLoaderWarp && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.status, p.timeout_ns};
  const int g0 = blockIdx.x * p.per_cta;
  const int g1 = min(p.total, g0 + p.per_cta);
  if (warp < 4) {
    dm_softmax<D>(base, smem, tmem, p, wc, g0, g1, warp, lane);
  } else if (warp == kDmLoaderWarp) {
    if (lane == 0) dm_loader<D>(base, &tm_q, &tm_k, &tm_v, p, wc, g0, g1);
    __syncwarp();
  } else {
    if (lane == 0) dm_mma<D>(base, tmem, p, wc, g0, g1);
    __syncwarp();
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kDmMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kDmTmemCols);
  }
}

}  // namespace attn_b200
