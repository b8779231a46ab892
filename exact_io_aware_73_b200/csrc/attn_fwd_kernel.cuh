// attn_fwd_kernel.cuh -- exact attention forward for B200 (sm_100a).
//
// Computes, per (batch, head), O = softmax(scale * Q K^T [causal mask]) V and
// lse = ln(row sum of exp(scaled scores)), walking key/value tiles with the
// online-softmax recurrence so the N x N score matrix never reaches HBM.
//
// Source cited as [MM]: the marketmaker.cc blog post (Indonesian edition)
// "Apakah Konteks Sehari Penuh Mengalahkan Konteks Sepuluh Menit? Perhatian
// Kilat dan Pertanyaan Panjang Urutan", by section heading.
//
//   * tiles Q_i (128 rows) and K_j, V_j (128 keys) staged on chip, one pass
//     over the key/value blocks per query block  ([MM] "Algoritma Flash
//     Attention");
//   * running max / running sum with retroactive rescaling of the output,
//     normalised once at the end ([MM] "Pengulangan softmax online",
//     "FA2: paralelisme" item 1);
//   * work split over batch x heads x query blocks ([MM] "FA2: paralelisme"
//     item 2); each softmax thread owns one query row, so no cross-warp
//     reduction is needed (item 3);
//   * a loader warp issuing asynchronous tensor copies for the next key/value
//     block while the other warps compute on the current one, and the two
//     GEMMs of one query tile overlapping the softmax of the other
//     ([MM] "FA3: Mekanika hopper" items 1 and 2);
//   * key/value blocks entirely in a query block's future are never loaded
//     or computed ([MM] "Causal masking adalah tempat perdagangan mendapat
//     diskon").
//
// Blackwell mapping (not the pages' Hopper design):
//   * a persistent CTA per SM walks "units" = two 128-row Q tiles of one
//     (batch, head) that share every K/V tile it loads;
//   * warps 0-3 / 4-7: softmax warpgroups for Q tile 0 / 1 (one TMEM lane =
//     one query row per thread); warps 8 and 10: TMA loaders (Q and K, V);
//     warp 9: tcgen05 MMA issuer (one thread) and TMEM owner; at d = 64 and
//     for block-sparse units warp 9 issues for Q tile 0 and warp 11 for
//     Q tile 1;
//   * TMEM (512 columns x 128 lanes x 32 bit): S0 | S1 | O0 | O1.  The
//     softmax writes P (bf16) back over the first 64 columns of its S tile
//     (at d = 64, dense: into 64 columns of its own after O1); the P.V MMA
//     reads it from TMEM as its A operand;
//   * S = Q K^T: tcgen05.mma kind::f16, M=128 N=128 K=d, A and B K-major in
//     128B-swizzled shared memory (exactly the layout the TMA writes);
//     O += P V: M=128 N=d K=128, A from TMEM, B (V) MN-major in shared memory;
//   * the epilogue stages each warp's 32 output rows in shared memory and
//     writes them with TMA tensor stores (whole 128-byte row segments); Q
//     tiles are released by a tcgen05.commit after their last S MMA, so the
//     next unit's Q load overlaps this epilogue;
//   * the row max is rescaled lazily: the output is only corrected when a
//     row's running max grows by more than 2^8 (in exp2 units); P then stays
//     below 256, and O / l is unchanged because m and l always move together;
//   * every wait is bounded in time; a wait that runs out records it in a
//     device status word, the CTA drains its in-flight copies, frees its
//     tensor memory and exits.
//
// FP8 variant (template flag FP8; [MM] "FA3: Mekanika hopper" item 3): Q, K,
// V arrive as E4M3 codes with power-of-two block scales (one per 128-row Q /
// K tile, one per head for V).  Both GEMMs run as tcgen05.mma kind::f8f6f4
// (K = 32 per instruction, 128-byte rows = one swizzle panel at d = 128).  The
// score multiplier scale * log2(e) * q_scale * k_scale changes per K tile;
// a row's base m moves only when its tile maximum exceeds it by more than
// 2^4, and P is carried as 2^(x - m + 4) <= 256, so that every probability
// down to 2^-10 of the row maximum is an E4M3 normal number; P goes to TMEM
// as four E4M3 bytes per column.  The row sum adds the unrounded P; V's
// per-head scale multiplies the output in the epilogue and lse subtracts the
// 2^4 again.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <math_constants.h>

#include "ptx_sm100.cuh"

namespace attn_b200 {

constexpr int kBlockM = 128;   // query rows per Q tile (= TMEM lanes)
constexpr int kBlockN = 128;   // keys per K/V tile
constexpr int kThreads = 384;  // 12 warps = 3 warpgroups
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kVLoaderWarp = 10;
constexpr int kMmaWarp2 = 11;  // tile 1's MMA issuer (see mma_role_tile)
// Register split.  With 12 warps every thread is launched with 168
// registers (an SM sub-partition holds 3 warps of the CTA); warpgroup 2 (the
// loader / MMA / idle warps) hands registers back and the two softmax
// warpgroups take them, so a softmax thread holds its whole score row with
// room for the compiler to keep many exponentials in flight.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 200;
constexpr int kControlRegs = 104;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P <= 2^8
// FP8: a row's base moves when its tile maximum exceeds it by more than
// kFp8Threshold; P = 2^(x - m + kFp8Offset) then stays <= 2^8 (E4M3 holds up
// to 448), and every p >= 2^-(14 - kFp8Threshold) of the row maximum is an
// E4M3 normal number.
constexpr float kFp8Threshold = 4.0f;
constexpr float kFp8Offset = 8.0f - kFp8Threshold;
constexpr float kLn2 = 0.6931471805599453f;

// Device status word bits.
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBounds = 2u;  // debug build: an index check failed
constexpr uint32_t kRoleProducer = 1u << 8;
constexpr uint32_t kRoleMma = 1u << 9;
constexpr uint32_t kRoleSoftmax = 1u << 10;
constexpr uint32_t kRoleEpilogue = 1u << 11;
constexpr uint32_t kRoleDrain = 1u << 12;

// Pairs of exponentials (out of every 8 pairs of a score row) evaluated on the
// FMA pipe by exp2_poly_x2 instead of the MUFU unit; the rest use ex2.approx.
// At d = 64 the MUFU carries twice the exponentials per tensor-core FLOP of
// d = 128, so an eighth of them move to the FMA pipe (a quarter measured best
// before P got TMEM columns of its own; with the next S off the softmax's
// chain the FMA pipe's extra instructions cost more than they save); at
// d = 128 measurement favoured the MUFU alone.
#ifndef ATTN_EXP2_EMU_PER8
#define ATTN_EXP2_EMU_PER8_D64 1
#define ATTN_EXP2_EMU_PER8_D128 0
#else
#define ATTN_EXP2_EMU_PER8_D64 ATTN_EXP2_EMU_PER8
#define ATTN_EXP2_EMU_PER8_D128 ATTN_EXP2_EMU_PER8
#endif
template <int D>
constexpr int kEmuPer8 = (D == 128) ? ATTN_EXP2_EMU_PER8_D128 : ATTN_EXP2_EMU_PER8_D64;
static_assert(kEmuPer8<64> >= 0 && kEmuPer8<64> <= 8 && kEmuPer8<128> >= 0 &&
                  kEmuPer8<128> <= 8,
              "pairs out of 8");

// 2^x for two values at once on the FMA / integer pipes (x <= 8 here).
// Cody-Waite split x = n + f, n = round-to-nearest(x) obtained by adding
// 1.5 * 2^23 (n then sits in the low mantissa bits), f = x - n in [-1/2, 1/2];
// 2^f by a degree-3 polynomial with minimax relative error 7.5e-5, fitted by
// csrc/gen_exp2_poly.py (Remez exchange); 2^n by adding n to the exponent
// field.  x is clamped at -125 so the exponent cannot underflow (2^-125 is
// far below what a bf16 P can add next to the row maximum's weight of >= 1).
__device__ __forceinline__ uint64_t exp2_poly_x2(float x0, float x1) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const uint64_t x = f32x2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = add_f32x2(x, f32x2(kMagic, kMagic));
  const uint64_t n = add_f32x2(t, f32x2(-kMagic, -kMagic));
  const uint64_t f = fma_f32x2(n, f32x2(-1.f, -1.f), x);
  uint64_t q = fma_f32x2(f32x2(0x1.c3f76p-5f, 0x1.c3f76p-5f), f,
                         f32x2(0x1.f0de1ap-3f, 0x1.f0de1ap-3f));
  q = fma_f32x2(q, f, f32x2(0x1.62f31ap-1f, 0x1.62f31ap-1f));
  q = fma_f32x2(q, f, f32x2(0x1.fff692p-1f, 0x1.fff692p-1f));
  float t0, t1, q0, q1;
  f32x2_split(t, t0, t1);
  f32x2_split(q, q0, q1);
  const uint32_t r0 = __float_as_uint(q0) + (__float_as_uint(t0) << 23);
  const uint32_t r1 = __float_as_uint(q1) + (__float_as_uint(t1) << 23);
  return f32x2(__uint_as_float(r0), __uint_as_float(r1));
}

struct FwdParams {
  uint16_t *o;         // [BH, N, D] bf16
  float *lse;          // [BH, N] fp32
  uint32_t *status;    // device status word
  int bh;              // B * H
  int n;               // sequence length
  int num_units;       // bh * ceil(n / 256)
  float c_log2;        // scale * log2(e)
  unsigned long long timeout_ns;
  uint32_t debug_flags;  // bit 0: first CTA skips its first Q copy
  // FP8 variant only: dequantization scales (powers of two)
  const float *q_scale;  // [BH, tiles] one per 128-row Q tile
  const float *k_scale;  // [BH, tiles] one per 128-row K tile
  const float *v_scale;  // [BH] one per head
  int tiles;             // ceil(n / 128)
  // Merge into an accumulator of partial results (attention over disjoint
  // key sets, combined exactly through the log-sum-exp).  kMergeNone: write
  // O (bf16) and lse.  First: write this result to acc_o (fp32 [BH, N, D])
  // and acc_lse.  Into: acc <- merge(acc, this).  Last: O, lse <-
  // merge(acc, this), in bf16 / fp32.
  float *acc_o = nullptr;
  float *acc_lse = nullptr;
  int merge_mode = 0;
  // Non-causal only: units from tail_start on are single Q tiles, unit
  // tail_start + s being tile s % 2 of the pair tail_start + s / 2 (a last
  // round of pairs that would fill few CTAs runs as twice as many single
  // tiles instead).
  int tail_start = 0x7fffffff;
  // Block-sparse variant only: one byte per (Q tile, K tile) pair of a head,
  // row-major [tiles x tiles]; nonzero = the pair is computed.  A head's
  // mask starts mask_head_stride bytes after the previous one's (0: one
  // mask for every head).
  const uint8_t *block_mask = nullptr;
  int64_t mask_head_stride = 0;
};
constexpr int kMergeNone = 0, kMergeFirst = 1, kMergeInto = 2, kMergeLast = 3;

// Pairs of FP8 exponentials (out of 8) evaluated on the FMA pipe.
#ifndef ATTN_EXP2_EMU_PER8_FP8
#define ATTN_EXP2_EMU_PER8_FP8 0
#endif

// Shared-memory map (offsets from a 1024-byte aligned base).  Tiles are
// 128 rows of D elements (2 bytes, or 1 for FP8), in 128-byte-wide panels.
template <int D, bool FP8 = false>
struct Smem {
  static constexpr int kElem = FP8 ? 1 : 2;
  static constexpr int kRowBytes = D * kElem;
  static constexpr int kSub = kRowBytes / 128;                // 128-byte panels
  static constexpr int kPanelElems = 128 / kElem;             // elements per panel row
  static constexpr uint32_t kPanelBytes = kBlockM * 128;      // 128 rows x 128 B
  static constexpr uint32_t kTileBytes = kBlockM * kRowBytes; // one Q/K/V tile
  // Ring depths.  K_j is released as soon as both S MMAs of iteration j are
  // issued, V_j only after both P.V MMAs, so V needs the deeper ring to be
  // refilled a full iteration ahead.
#ifndef ATTN_V_STAGES_D128
#define ATTN_V_STAGES_D128 2
#endif
  static constexpr int kKStages = (kRowBytes == 256) ? 2 : 4;
  static constexpr int kVStages = (kRowBytes == 256) ? ATTN_V_STAGES_D128 : 4;
  static constexpr uint32_t kQ = 0;                           // 2 Q tiles
  static constexpr uint32_t kK = kQ + 2 * kTileBytes;         // K ring
  static constexpr uint32_t kV = kK + kKStages * kTileBytes;  // V ring
  // O staging for the TMA store of the epilogue: one buffer of 32 rows x 64
  // bf16 columns (128-byte rows, 128B-swizzled) per softmax warp
  static constexpr uint32_t kOutWarpBytes = 32 * 128;
  static constexpr uint32_t kOut = kV + kVStages * kTileBytes;
  static constexpr uint32_t kBars = kOut + 8 * kOutWarpBytes;
  // barrier indices
  // P_HALF: the first 64 keys of a tile's P are in TMEM (bf16 only);
  // P_FULL: all of it; S_FREE (d = 64 only): the softmax has read its S
  // tile out of TMEM
  static constexpr int Q_FULL = 0, Q_EMPTY = 2, S_FULL = 4, P_FULL = 6,
                       O_FULL = 8, O_EMPTY = 10, DRAIN = 12, P_HALF = 13,
                       S_FREE = 15,
                       K_FULL = 17, K_EMPTY = K_FULL + kKStages,
                       V_FULL = K_EMPTY + kKStages, V_EMPTY = V_FULL + kVStages,
                       NUM_BARS = V_EMPTY + kVStages;
  static constexpr uint32_t kMisc = kBars + NUM_BARS * 8;  // tmem slot, abort
  // the ring index each K / V slot was last claimed for (see slot_claimed)
  static constexpr uint32_t kSlotPos = kMisc + 16;
  static constexpr uint32_t kBytes = kSlotPos + 4 * (kKStages + kVStages);
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack for alignment
  static_assert(kAlloc <= 232448, "shared memory budget");
};

// One work unit: rows [q0, q0 + 256) of head bh, as two Q tiles; n0 / n1 =
// number of K/V tiles each Q tile visits (0 = tile lies beyond N).  A
// single-tile unit has n1 = 0.
struct Unit {
  int bh, q0, n0, n1;  // n0, n1: K tiles Q tile 0 / 1 computes
  int nu;              // K/V tiles the unit loads (the union of both lists)
};

template <bool CAUSAL>
__device__ __forceinline__ Unit decode_unit(int u, int bh_count, int n,
                                            int tail_start) {
  const int qpairs = (n + 255) >> 8;
  const int tiles = (n + 127) >> 7;
  Unit w;
  int qp;
  if (!CAUSAL && u >= tail_start) {
    // a single Q tile of one of the last pairs; it runs in the first tile's
    // slot (softmax warpgroup 0, S0 / O0)
    const int s = u - tail_start;
    const int pr = tail_start + (s >> 1);
    w.bh = pr / qpairs;
    w.q0 = (pr % qpairs) * 256 + 128 * (s & 1);
    w.n0 = (w.q0 < n) ? tiles : 0;
    w.n1 = 0;
    w.nu = w.n0;
    return w;
  }
  if (CAUSAL) {
    // heaviest units (last query rows) first, heads interleaved
    qp = qpairs - 1 - u / bh_count;
    w.bh = u % bh_count;
  } else {
    // consecutive units share a head's K/V in L2
    w.bh = u / qpairs;
    qp = u % qpairs;
  }
  w.q0 = qp * 256;
  const int qt0 = w.q0 >> 7;
  w.n0 = CAUSAL ? min(tiles, qt0 + 1) : tiles;
  w.n1 = (w.q0 + 128 < n) ? (CAUSAL ? min(tiles, qt0 + 2) : tiles) : 0;
  w.nu = max(w.n0, w.n1);
  return w;
}

// The k-th unit a persistent CTA takes: round-robin over the CTAs, reversed
// in every other round under the causal mask.  Causal units are numbered
// heaviest first, so the reversal (a snake order) gives the CTA that took
// one of the heaviest units of a round one of the lightest of the next; the
// work per CTA then stays within about one unit of the mean, where plain
// round-robin leaves the first CTAs up to a third above it.
template <bool CAUSAL>
__device__ __forceinline__ int unit_at(int k) {
  const int g = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  return k * g + ((CAUSAL && (k & 1)) ? g - 1 - c : c);
}

// Block-sparse units (the block-sparse extension of the tiled algorithm,
// briefgpt.xyz summary page of arXiv 2307.08691, FlashAttention entry): two
// consecutive Q tiles of one (batch, head), like the dense units, each
// computing only the K tiles its mask row marks (and, under the causal mask,
// none past its diagonal).  The unit loads the union of the two lists, in
// order; a K/V tile that only one of the tiles uses is computed by that
// tile alone.  Every role walks the same union with KWalk, so the K/V ring
// stays in step.
__device__ __forceinline__ const uint8_t *sparse_row(const FwdParams &p, int bh, int qt,
                                                    int tiles) {
  return p.block_mask + static_cast<int64_t>(bh) * p.mask_head_stride +
         static_cast<int64_t>(qt) * tiles;
}

// The first computed K tile at or after kj (kend when there is none).
__device__ __forceinline__ int sparse_next(const uint8_t *row, int kj, int kend) {
  while (kj < kend && __ldg(row + kj) == 0) ++kj;
  return kj;
}

template <bool CAUSAL, bool SPARSE>
__device__ __forceinline__ Unit get_unit(int u, const FwdParams &p) {
  if constexpr (!SPARSE) {
    return decode_unit<CAUSAL>(u, p.bh, p.n, p.tail_start);
  } else {
    const int tiles = (p.n + 127) >> 7, pairs = (tiles + 1) >> 1;
    Unit w;
    int pq;
    if (CAUSAL) {  // heaviest pairs (last query rows) first, heads interleaved
      pq = pairs - 1 - u / p.bh;
      w.bh = u % p.bh;
    } else {
      w.bh = u / pairs;
      pq = u % pairs;
    }
    const int qt0 = 2 * pq, qt1 = qt0 + 1;
    w.q0 = qt0 * kBlockM;
    const uint8_t *r0 = sparse_row(p, w.bh, qt0, tiles);
    const uint8_t *r1 = sparse_row(p, w.bh, qt1 < tiles ? qt1 : qt0, tiles);
    const int kend0 = CAUSAL ? qt0 + 1 : tiles;
    const int kend1 = qt1 < tiles ? (CAUSAL ? qt1 + 1 : tiles) : 0;
    int c0 = 0, c1 = 0, cu = 0;
    for (int kj = 0; kj < max(kend0, kend1); ++kj) {
      const bool m0 = kj < kend0 && __ldg(r0 + kj) != 0;
      const bool m1 = kj < kend1 && __ldg(r1 + kj) != 0;
      c0 += m0;
      c1 += m1;
      cu += (m0 || m1);
    }
    w.n0 = c0;
    w.n1 = c1;
    w.nu = cu;
    return w;
  }
}

// The K/V tiles one unit loads, in order: next() steps to the following
// one and returns its K tile index, with bit t of `use` set when Q tile t
// computes it.  Dense units load K tiles 0 .. nu-1, and tile t uses the
// first n_t of them.
template <bool CAUSAL, bool SPARSE>
struct KWalk {
  const uint8_t *r0, *r1;
  int kend0, kend1, kj, n0, n1;
  __device__ __forceinline__ KWalk(const FwdParams &p, const Unit &w)
      : r0(nullptr), r1(nullptr), kend0(0), kend1(0), kj(-1), n0(w.n0), n1(w.n1) {
    if constexpr (SPARSE) {
      const int tiles = (p.n + 127) >> 7, qt0 = w.q0 >> 7, qt1 = qt0 + 1;
      r0 = sparse_row(p, w.bh, qt0, tiles);
      r1 = sparse_row(p, w.bh, qt1 < tiles ? qt1 : qt0, tiles);
      kend0 = CAUSAL ? qt0 + 1 : tiles;
      kend1 = qt1 < tiles ? (CAUSAL ? qt1 + 1 : tiles) : 0;
    }
  }
  __device__ __forceinline__ int next(int &use) {
    ++kj;
    if constexpr (SPARSE) {
      const int kend = max(kend0, kend1);
      for (; kj < kend; ++kj) {
        use = (kj < kend0 && __ldg(r0 + kj) != 0) | ((kj < kend1 && __ldg(r1 + kj) != 0) << 1);
        if (use) return kj;
      }
      use = 0;  // past the end (callers stop after nu steps)
      return kj;
    } else {
      use = (kj < n0) | ((kj < n1) << 1);
      return kj;
    }
  }
};

// Index checks of the debug build (compiled with ATTN_DEBUG_BOUNDS): an index
// the kernel is about to use for a global access must lie in [0, limit);
// when it does not, the status word is flagged and the caller skips the
// access.  In release builds the check is absent and always passes.
#ifdef ATTN_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif
__device__ __forceinline__ bool in_bounds(int64_t i, int64_t limit, uint32_t *status) {
  if constexpr (kDebugBounds) {
    if (i < 0 || i >= limit) {
      atomicOr(status, kStatusBounds);
      return false;
    }
  }
  return true;
}

struct WaitCtx {
  volatile int *abort;
  uint32_t *status;
  unsigned long long timeout_ns;
};

// Bounded wait for the phase of `bar` with parity `parity`.  Returns false
// (after flagging the CTA and the device status word) when the time limit
// runs out, or when another thread of the CTA already gave up.  A waiting
// thread sleeps inside try_wait (up to kSleepHintNs per probe) instead of
// spinning, so it takes no issue slots from the warps sharing its SM
// sub-partition; the abort flag and the clock are looked at between probes.
constexpr uint32_t kSleepHintNs = 20000;

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          const WaitCtx &wc, uint32_t role) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, kSleepHintNs)) return true;
    if (*wc.abort) return false;
    if (global_timer_ns() - t0 > wc.timeout_ns) {
      *wc.abort = 1;
      atomicOr(wc.status, kStatusTimeout | role);
      return false;
    }
  }
}

// Same contract as mbar_wait, for the single MMA-issuing thread: it polls
// without sleeping (it is on the critical path of every tile, and a thread
// woken from a sleeping probe resumes late), looking at the abort flag and
// the clock every 128 probes.
__device__ __forceinline__ bool mbar_wait_spin(uint32_t bar, uint32_t parity,
                                               const WaitCtx &wc, uint32_t role) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 127u) == 0) {
      if (*wc.abort) return false;
      if (global_timer_ns() - t0 > wc.timeout_ns) {
        *wc.abort = 1;
        atomicOr(wc.status, kStatusTimeout | role);
        return false;
      }
    }
  }
}

// With one MMA issuer per Q tile, a tile skips the K/V tiles of its unit
// that only the other tile computes, so it may come to wait on a ring slot
// whose previous occupant has not even landed.  A parity wait is only exact
// for the barrier's current phase or the one before, so the issuer first
// waits until the loader has claimed the slot for ring index `idx` (after
// the slot's previous tile was released, which implies it had landed); the
// FULL barrier is then in the phase for `idx` or past it.  The loader
// publishes the index with release semantics, the issuer reads it with
// acquire semantics; the wait is bounded like mbar_wait_spin.
__device__ __forceinline__ bool slot_claimed(uint32_t pos_addr, int idx, const WaitCtx &wc,
                                             uint32_t role) {
  if (ld_acquire_shared(pos_addr) == idx) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_shared(pos_addr) == idx) return true;
    if ((it & 127u) == 0) {
      if (*wc.abort) return false;
      if (global_timer_ns() - t0 > wc.timeout_ns) {
        *wc.abort = 1;
        atomicOr(wc.status, kStatusTimeout | role);
        return false;
      }
    }
  }
}

// Bounded wait used while draining after an abort: ignores the abort flag.
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity,
                                                const WaitCtx &wc) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait_sleep(bar, parity, kSleepHintNs)) {
    if (global_timer_ns() - t0 > wc.timeout_ns) {
      atomicOr(wc.status, kStatusTimeout | kRoleDrain);
      return;
    }
  }
}

// UMMA shared-memory descriptor, 128-byte swizzle, sm_100 version bits.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr,
                                                    uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  const uint32_t lo = ((addr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
  const uint32_t hi = ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// d = 64 (bf16): the two O accumulators take only 128 of the 512 TMEM
// columns, so each tile's P gets 64 columns of its own instead of
// overwriting S.  A tile's next S then needs only that its softmax has read
// the last S out (S_FREE), not the P.V of it, so it is computed while the
// softmax still works on the current one.  (In block-sparse units the two
// tiles compute different K tiles, and a tile that waited for its next K
// tile before its P.V could wait on a slot the other tile holds until it
// gets that P.V's V slot: there the next S goes ahead only when its K tile
// has already landed.)
template <int D, bool FP8, bool SPARSE>
constexpr bool kSplitP = (D == 64) && !FP8;

// Which MMA role a variant runs.  Where P lies over S (d = 128, FP8) and
// both tiles compute every K tile in step, one thread serves both tiles in
// a fixed order (mma_role): each tile's next S goes out right behind its
// P.V, which keeps the S -> softmax -> P.V chain short; two independent
// issuers there interleave the tiles' MMAs in the tensor pipe and delay
// every S (measured 22 % slower).  The split layout takes S off that chain,
// and block-sparse pairs compute different K tiles, so those run one
// issuing thread per Q tile (mma_role_tile).
template <int D, bool FP8, bool SPARSE>
constexpr bool kPerTileIssuer = SPARSE || kSplitP<D, FP8, SPARSE>;

// ------------------------------------------------------------------ loader

// Two loader threads: one for Q and K, one for V, so that K (released early,
// after the S MMAs) never waits in line behind V (released late, after the
// P.V MMAs).
constexpr int kLoadQK = 1, kLoadV = 2;

template <int D, bool CAUSAL, int MODE, bool FP8, bool SPARSE>
__device__ __forceinline__ void producer_role(uint32_t base,
                                              const CUtensorMap *tq,
                                              const CUtensorMap *tk,
                                              const CUtensorMap *tv,
                                              const FwdParams &p,
                                              const WaitCtx &wc) {
  using L = Smem<D, FP8>;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };
  int qocc[2] = {0, 0};     // non-empty occurrences of each Q tile so far
  int q_issued[2] = {0, 0};
  int k_issued = 0, v_issued = 0;
  bool skip_first_q = (MODE != kLoadV) && (p.debug_flags & 1u) && blockIdx.x == 0;
  bool ok = true;
  const uint64_t pol_kv = policy_evict_last();
  const uint64_t pol_q = policy_evict_first();

  for (int k = 0, u = unit_at<CAUSAL>(0); ok && u < p.num_units; u = unit_at<CAUSAL>(++k)) {
    const Unit w = get_unit<CAUSAL, SPARSE>(u, p);
    const int nt[2] = {w.n0, w.n1};
    KWalk<CAUSAL, SPARSE> walk(p, w);
    for (int t = 0; MODE != kLoadV && t < 2; ++t) {
      if (nt[t] == 0) continue;
      if (qocc[t] > 0) {
        ok = mbar_wait(bar(L::Q_EMPTY + t), (qocc[t] - 1) & 1, wc, kRoleProducer);
        if (!ok) break;
      }
      ++qocc[t];
      if (skip_first_q && t == 0) {  // injected fault: this copy never happens
        skip_first_q = false;
        continue;
      }
      mbar_arrive_expect_tx(bar(L::Q_FULL + t), L::kTileBytes);
      for (int s = 0; s < L::kSub; ++s)
        tma_load_3d_hint(base + L::kQ + t * L::kTileBytes + s * L::kPanelBytes,
                         tq, bar(L::Q_FULL + t), s * L::kPanelElems,
                         w.q0 + kBlockM * t,
                         w.bh, pol_q);
      ++q_issued[t];
    }
    if (!ok) break;
    for (int j = 0; j < w.nu; ++j) {
      int use;
      const int kj = walk.next(use);
      if (MODE != kLoadV) {
        const int ks = k_issued % L::kKStages;
        ok = mbar_wait(bar(L::K_EMPTY + ks), ((k_issued / L::kKStages) & 1) ^ 1,
                       wc, kRoleProducer);
        if (!ok) break;
        if constexpr (kPerTileIssuer<D, FP8, SPARSE>) {
          // the slot's release takes one arrival per Q tile: give the one of
          // a tile that does not compute with this K tile, then publish
          st_release_shared(base + L::kSlotPos + 4 * ks, k_issued);
          if (use != 3) mbar_arrive(bar(L::K_EMPTY + ks));
        }
        mbar_arrive_expect_tx(bar(L::K_FULL + ks), L::kTileBytes);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d_hint(base + L::kK + ks * L::kTileBytes + s * L::kPanelBytes,
                           tk, bar(L::K_FULL + ks), s * L::kPanelElems,
                           kj * kBlockN, w.bh,
                           pol_kv);
        ++k_issued;
      }
      if (MODE != kLoadQK) {
        const int vs = v_issued % L::kVStages;
        ok = mbar_wait(bar(L::V_EMPTY + vs), ((v_issued / L::kVStages) & 1) ^ 1,
                       wc, kRoleProducer);
        if (!ok) break;
        if constexpr (kPerTileIssuer<D, FP8, SPARSE>) {
          st_release_shared(base + L::kSlotPos + 4 * (L::kKStages + vs), v_issued);
          if (use != 3) mbar_arrive(bar(L::V_EMPTY + vs));
        }
        mbar_arrive_expect_tx(bar(L::V_FULL + vs), L::kTileBytes);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d_hint(base + L::kV + vs * L::kTileBytes + s * L::kPanelBytes,
                           tv, bar(L::V_FULL + vs), s * L::kPanelElems,
                           kj * kBlockN, w.bh,
                           pol_kv);
        ++v_issued;
      }
    }
  }

  if (*wc.abort) {
    // Every copy issued must land before the CTA may exit.
    for (int t = 0; t < 2; ++t)
      if (q_issued[t] > 0)
        mbar_wait_drain(bar(L::Q_FULL + t), (q_issued[t] - 1) & 1, wc);
    for (int st = 0; st < L::kKStages; ++st)
      if (k_issued > st) {
        const int last = st + ((k_issued - 1 - st) / L::kKStages) * L::kKStages;
        mbar_wait_drain(bar(L::K_FULL + st), (last / L::kKStages) & 1, wc);
      }
    for (int st = 0; st < L::kVStages; ++st)
      if (v_issued > st) {
        const int last = st + ((v_issued - 1 - st) / L::kVStages) * L::kVStages;
        mbar_wait_drain(bar(L::V_FULL + st), (last / L::kVStages) & 1, wc);
      }
  }
}

// ------------------------------------------------------------------ MMA

template <int D, bool FP8 = false>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem,
                                         uint32_t k_smem) {
  // S[128 x 128] = Q[128 x D] K[128 x D]^T; both K-major, 128B swizzle.  One
  // instruction covers 32 bytes of K (16 bf16 or 32 E4M3 elements).
  constexpr uint32_t idesc = (1u << 4)                           // D: f32
                             | ((FP8 ? 0u : 1u) << 7)            // A: bf16 | e4m3
                             | ((FP8 ? 0u : 1u) << 10)           // B: bf16 | e4m3
                             | ((uint32_t)(kBlockN >> 3) << 17)  // N
                             | ((uint32_t)(kBlockM >> 4) << 24); // M
  // The descriptors are built once; a step adds its byte offset / 16 to the
  // 14-bit address field (shared addresses are below 2^18 and 16-byte
  // aligned, so the field cannot carry), which keeps the issuing thread's
  // instructions between MMAs few.
  const uint64_t qd = smem_desc_sw128(q_smem, 16, 1024);
  const uint64_t kd = smem_desc_sw128(k_smem, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < Smem<D, FP8>::kRowBytes / 32; ++kk) {
    constexpr uint32_t kPanel = Smem<D, FP8>::kPanelBytes;
    const uint64_t off = ((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
    if constexpr (FP8)
      mma_f8_ss(d_tmem, qd + off, kd + off, idesc, kk > 0);
    else
      mma_bf16_ss(d_tmem, qd + off, kd + off, idesc, kk > 0);
  }
}

template <int D, bool FP8 = false, int KK0 = 0, int KK1 = kBlockN / (FP8 ? 32 : 16)>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem,
                                         uint32_t v_smem, bool accumulate) {
  // O[128 x D] (+)= P[128 x 128] V[128 x D]; P in TMEM (K-major: bf16 two per
  // column, or E4M3 four per column), V MN-major (D contiguous) with 128B
  // swizzle: 128-byte-wide D panels are kPanelBytes apart (LBO), 8-key
  // groups 1024 B (SBO).  One instruction covers 16 keys (bf16) or 32 (E4M3):
  // 8 TMEM columns of P and 16 or 32 rows of V.
  constexpr uint32_t idesc = (1u << 4) | ((FP8 ? 0u : 1u) << 7) |
                             ((FP8 ? 0u : 1u) << 10)
                             | (1u << 16)           // B: MN-major
                             | ((uint32_t)(D >> 3) << 17)
                             | ((uint32_t)(kBlockM >> 4) << 24);
  constexpr int kKeys = FP8 ? 32 : 16;
  const uint64_t vd = smem_desc_sw128(v_smem, Smem<D, FP8>::kPanelBytes, 1024);
#pragma unroll
  for (int kk = KK0; kk < KK1; ++kk) {
    const uint64_t bdesc = vd + static_cast<uint64_t>((kk * kKeys * 128) >> 4);
    if constexpr (FP8)
      mma_f8_ts(d_tmem, p_tmem + kk * 8, bdesc, idesc, (accumulate || kk > 0) ? 1u : 0u);
    else
      mma_bf16_ts(d_tmem, p_tmem + kk * 8, bdesc, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D, bool CAUSAL, bool FP8, bool SPARSE>
__device__ __forceinline__ void mma_role(uint32_t base, uint32_t tmem,
                                         const FwdParams &p, const WaitCtx &wc) {
  using L = Smem<D, FP8>;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };
  const uint32_t tS[2] = {tmem + 0, tmem + 128};
  const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};
  const uint32_t sQ[2] = {base + L::kQ, base + L::kQ + L::kTileBytes};
  int qocc[2] = {0, 0}, pcnt[2] = {0, 0}, oocc[2] = {0, 0};
  int kcons = 0, vcons = 0;
  bool ok = true;

  for (int k = 0, u = unit_at<CAUSAL>(0); ok && u < p.num_units; u = unit_at<CAUSAL>(++k)) {
    const Unit w = get_unit<CAUSAL, SPARSE>(u, p);
    const int nt[2] = {w.n0, w.n1};
    const int nmax = max(nt[0], nt[1]);
    if (nmax == 0) continue;  // a single tile beyond N, or no K tile: nothing to compute
    for (int t = 0; t < 2 && ok; ++t)
      if (nt[t] > 0) {
        ok = mbar_wait_spin(bar(L::Q_FULL + t), qocc[t] & 1, wc, kRoleMma);
        ++qocc[t];
      }
    if (!ok) break;
    {  // S_0 for both tiles
      const int ks = kcons % L::kKStages;
      ok = mbar_wait_spin(bar(L::K_FULL + ks), (kcons / L::kKStages) & 1, wc, kRoleMma);
      if (!ok) break;
      tc_fence_after_sync();
      for (int t = 0; t < 2; ++t)
        if (nt[t] > 0) {
          issue_qk<D, FP8>(tS[t], sQ[t], base + L::kK + ks * L::kTileBytes);
          mma_commit(bar(L::S_FULL + t));
          if (nt[t] == 1) mma_commit(bar(L::Q_EMPTY + t));  // last read of Q_t
        }
      mma_commit(bar(L::K_EMPTY + ks));
      ++kcons;
    }
    for (int j = 0; j < nmax && ok; ++j) {
      const int vs = vcons % L::kVStages;
      ok = mbar_wait_spin(bar(L::V_FULL + vs), (vcons / L::kVStages) & 1, wc, kRoleMma);
      if (!ok) break;
      const int ks = kcons % L::kKStages;
      const bool k_next = j + 1 < nmax;  // K_{j+1} exists (waited below)
      bool k_ready = false;
      for (int t = 0; t < 2; ++t) {
        if (j >= nt[t]) continue;
        // bf16: the P.V of the tile's first 64 keys starts while the softmax
        // still computes the second half's probabilities
        ok = mbar_wait_spin(bar((FP8 ? L::P_FULL : L::P_HALF) + t), pcnt[t] & 1, wc,
                            kRoleMma);
        if (!ok) break;
        if (j == 0 && oocc[t] > 0) {
          // previous unit's epilogue must have read O out of TMEM
          ok = mbar_wait_spin(bar(L::O_EMPTY + t), (oocc[t] - 1) & 1, wc, kRoleMma);
          if (!ok) break;
        }
        tc_fence_after_sync();
        const uint32_t vt = base + L::kV + vs * L::kTileBytes;
        if constexpr (FP8) {
          issue_pv<D, FP8>(tO[t], tS[t], vt, j > 0);
        } else {
          issue_pv<D, FP8, 0, 4>(tO[t], tS[t], vt, j > 0);
          ok = mbar_wait_spin(bar(L::P_FULL + t), pcnt[t] & 1, wc, kRoleMma);
          if (!ok) break;
          tc_fence_after_sync();
          issue_pv<D, FP8, 4, 8>(tO[t], tS[t], vt, true);
        }
        ++pcnt[t];
        mma_commit(bar(L::O_FULL + t));
        if (j + 1 < nt[t]) {
          if (!k_ready) {
            ok = mbar_wait_spin(bar(L::K_FULL + ks), (kcons / L::kKStages) & 1, wc,
                          kRoleMma);
            if (!ok) break;
            tc_fence_after_sync();
            k_ready = true;
          }
          // issued after this tile's P.V in the same thread: the tensor pipe
          // reads P before this MMA overwrites the S columns holding it
          issue_qk<D, FP8>(tS[t], sQ[t], base + L::kK + ks * L::kTileBytes);
          mma_commit(bar(L::S_FULL + t));
          if (j + 2 == nt[t]) mma_commit(bar(L::Q_EMPTY + t));  // last read of Q_t
        }
      }
      if (!ok) break;
      mma_commit(bar(L::V_EMPTY + vs));
      ++vcons;
      if (k_next) {
        mma_commit(bar(L::K_EMPTY + ks));
        ++kcons;
      }
    }
    for (int t = 0; t < 2; ++t)
      if (nt[t] > 0) ++oocc[t];
  }
  // All tensor-core work must finish before TMEM is released.
  mma_commit(bar(L::DRAIN));
  mbar_wait_drain(bar(L::DRAIN), 0, wc);
}

// One MMA-issuing thread per Q tile (warp 9 for tile 0, warp 11 for tile 1),
// each walking its own tile's steps in order with blocking waits, so that
// neither tile's MMAs queue behind the other's barriers.  Per K tile j the
// tile issues S_j = Q K_j^T and O += P_j V_j; P_j lies over S_j's columns,
// so S_{j+1} follows P_j V_j in the same thread (the tensor pipe then reads
// P_j before overwriting it), except in the split layout (d = 64), where P
// has columns of its own and S_{j+1} goes out as soon as the softmax has
// read S_j (S_FREE) -- in block-sparse units only if K_{j+1} has landed.
// A K or V slot's EMPTY barrier counts one arrival per Q tile: a
// tcgen05.commit from each tile that computes with it, and one from the
// loader for a tile that does not.
template <int D, bool CAUSAL, bool FP8, bool SPARSE>
__device__ __forceinline__ void mma_role_tile(uint32_t base, uint32_t tmem,
                                              const FwdParams &p, const WaitCtx &wc,
                                              const int t) {
  using L = Smem<D, FP8>;
  constexpr bool kSplit = kSplitP<D, FP8, SPARSE>;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };
  const uint32_t tS = tmem + 128 * t;
  const uint32_t tO = tmem + 256 + D * t;
  const uint32_t tP = kSplit ? tmem + 256 + 2 * D + 64 * t : tS;
  const uint32_t sQ = base + L::kQ + t * L::kTileBytes;
  int qocc = 0, pcnt = 0, oocc = 0, sdone = 0;
  int ring = 0;  // ring index of the unit's first K/V tile
  bool ok = true;

  for (int k = 0, u = unit_at<CAUSAL>(0); ok && u < p.num_units; u = unit_at<CAUSAL>(++k)) {
    const Unit w = get_unit<CAUSAL, SPARSE>(u, p);
    const int n = t ? w.n1 : w.n0;
    if (n == 0) {  // nothing to compute in this unit
      ring += w.nu;
      continue;
    }
    KWalk<CAUSAL, SPARSE> walk(p, w);
    int pos = -1;
    // the place in the unit's K/V list of the next K tile this Q tile computes
    auto step = [&]() {
      int use;
      do {
        walk.next(use);
        ++pos;
      } while (!((use >> t) & 1) && pos < w.nu);
      return pos;
    };
    auto issue_s = [&](int at, int j) -> bool {
      if (kSplit && sdone > 0) {  // the softmax has read the previous S out
        if (!mbar_wait_spin(bar(L::S_FREE + t), (sdone - 1) & 1, wc, kRoleMma)) return false;
      }
      const int ka = ring + at;
      if (!slot_claimed(base + L::kSlotPos + 4 * (ka % L::kKStages), ka, wc, kRoleMma) ||
          !mbar_wait_spin(bar(L::K_FULL + ka % L::kKStages), (ka / L::kKStages) & 1, wc,
                          kRoleMma))
        return false;
      tc_fence_after_sync();
      issue_qk<D, FP8>(tS, sQ, base + L::kK + (ka % L::kKStages) * L::kTileBytes);
      mma_commit(bar(L::S_FULL + t));
      if (j + 1 == n) mma_commit(bar(L::Q_EMPTY + t));  // last read of Q_t
      mma_commit(bar(L::K_EMPTY + ka % L::kKStages));
      ++sdone;
      return true;
    };

    ok = mbar_wait_spin(bar(L::Q_FULL + t), qocc & 1, wc, kRoleMma);
    ++qocc;
    if (!ok) break;
    int at = step(), nat = 0;
    ok = issue_s(at, 0);
    for (int j = 0; j < n && ok; ++j) {
      bool early = false;  // S_{j+1} issued ahead of P_j V_j
      if (kSplit && j + 1 < n) {
        nat = step();
        early = true;
        if constexpr (SPARSE) {
          // only if K_{j+1} has landed: wait for the softmax to read S_j,
          // then look (without waiting) at K_{j+1}'s slot
          ok = mbar_wait_spin(bar(L::S_FREE + t), (sdone - 1) & 1, wc, kRoleMma);
          if (!ok) break;
          const int ka = ring + nat;
          early = ld_acquire_shared(base + L::kSlotPos + 4 * (ka % L::kKStages)) == ka &&
                  mbar_test_wait(bar(L::K_FULL + ka % L::kKStages), (ka / L::kKStages) & 1);
        }
        if (early) {
          ok = issue_s(nat, j + 1);
          if (!ok) break;
        }
      }
      // O += P_j V_j: the first 64 keys once P_HALF, the rest once P_FULL
      // (FP8: all at once); the unit's first P.V also waits for the previous
      // unit's epilogue to read O out of TMEM
      ok = mbar_wait_spin(bar((FP8 ? L::P_FULL : L::P_HALF) + t), pcnt & 1, wc, kRoleMma);
      if (!ok) break;
      const int va = ring + at;
      ok = slot_claimed(base + L::kSlotPos + 4 * (L::kKStages + va % L::kVStages), va, wc,
                        kRoleMma) &&
           mbar_wait_spin(bar(L::V_FULL + va % L::kVStages), (va / L::kVStages) & 1, wc,
                          kRoleMma);
      if (!ok) break;
      if (j == 0 && oocc > 0) {
        ok = mbar_wait_spin(bar(L::O_EMPTY + t), (oocc - 1) & 1, wc, kRoleMma);
        if (!ok) break;
      }
      tc_fence_after_sync();
      const uint32_t vt = base + L::kV + (va % L::kVStages) * L::kTileBytes;
      if constexpr (FP8) {
        issue_pv<D, FP8>(tO, tP, vt, j > 0);
      } else {
        issue_pv<D, FP8, 0, 4>(tO, tP, vt, j > 0);
        ok = mbar_wait_spin(bar(L::P_FULL + t), pcnt & 1, wc, kRoleMma);
        if (!ok) break;
        tc_fence_after_sync();
        issue_pv<D, FP8, 4, 8>(tO, tP, vt, true);
      }
      ++pcnt;
      mma_commit(bar(L::O_FULL + t));
      mma_commit(bar(L::V_EMPTY + va % L::kVStages));
      if (!early && j + 1 < n) {
        if (!kSplit) nat = step();
        ok = issue_s(nat, j + 1);
        if (!ok) break;
      }
      at = nat;
    }
    if (!ok) break;
    ring += w.nu;
    ++oocc;
  }
  // All tensor-core work (both issuers') must finish before TMEM is released.
  mma_commit(bar(L::DRAIN));
  mbar_wait_drain(bar(L::DRAIN), 0, wc);
}

// ------------------------------------------------------------------ softmax

template <int D>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld_32x32b_x32(tO + c * 32, o);
    tmem_wait_ld(o);
#pragma unroll
    for (int i = 0; i < 32; ++i)
      o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
    tmem_st_32x32b_x32(tO + c * 32, o);
  }
}

// Loads this thread's row of S (128 fp32 columns of TMEM) into registers;
// on the last tile of a row applies the mask: keys c > limit are -inf
// (causal diagonal: limit = row; ragged tail: limit = N - 1 - first key).
__device__ __forceinline__ void load_scores(uint32_t tS, uint32_t (&s)[4][32],
                                            bool mask, int limit) {
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tS + c * 32, s[c]);
  tmem_wait_ld(s[0]);
  reg_fence(s[1]);
  reg_fence(s[2]);
  reg_fence(s[3]);
  if (mask) {
#pragma unroll
    for (int c = 0; c < 128; ++c)
      if (c > limit) s[c >> 5][c & 31] = __float_as_uint(-CUDART_INF_F);
  }
}

// Row maximum of the raw scores: 3-input max over pairs, 8 chains.
__device__ __forceinline__ float row_max_raw(const uint32_t (&s)[4][32]) {
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(s[0][i]);
#pragma unroll
  for (int c = 8; c < 128; c += 2)
    mx[(c >> 1) & 7] = max3f(mx[(c >> 1) & 7], __uint_as_float(s[c >> 5][c & 31]),
                             __uint_as_float(s[(c + 1) >> 5][(c + 1) & 31]));
  return max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]),
               fmaxf(mx[6], mx[7]));
}

// p = 2^(s * scale * log2 e - m) for the whole row: one packed FMA per pair,
// the exponential on the MUFU unit or (kEmuPer8 pairs in 8) the FMA pipe,
// packed row sums, bf16x2 packing for the P.V MMA.  Returns the row sum.
template <int D, int HALF, int CC0 = 0, int CC1 = 32>
__device__ __forceinline__ float exp_row(const uint32_t (&s)[4][32], float cl2,
                                         float m, uint32_t (&pk)[32]) {
  // columns 64 HALF .. 64 HALF + 63: pairs c = 32 HALF .. 32 HALF + 31, of
  // which this call computes cc in [CC0, CC1) into pk[cc]
  const uint64_t c2 = f32x2(cl2, cl2);
  const uint64_t nm2 = f32x2(-m, -m);
  uint64_t acc[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
#pragma unroll
  for (int cc = CC0; cc < CC1; ++cc) {
    const int c = 32 * HALF + cc;
    const float s0 = __uint_as_float(s[(2 * c) >> 5][(2 * c) & 31]);
    const float s1 = __uint_as_float(s[(2 * c + 1) >> 5][(2 * c + 1) & 31]);
    const uint64_t x2 = fma_f32x2(f32x2(s0, s1), c2, nm2);
    float x0, x1;
    f32x2_split(x2, x0, x1);
    uint64_t p2;
    if ((c & 7) < kEmuPer8<D>) {
      p2 = exp2_poly_x2(x0, x1);
    } else {
      p2 = f32x2(ex2_approx(x0), ex2_approx(x1));
    }
    acc[c & 1] = add_f32x2(acc[c & 1], p2);
    float p0, p1;
    f32x2_split(p2, p0, p1);
    pk[cc] = pack_bf16x2(p0, p1);
  }
  float a0, a1, b0, b1;
  f32x2_split(acc[0], a0, a1);
  f32x2_split(acc[1], b0, b1);
  return (a0 + a1) + (b0 + b1);
}

// FP8 version of exp_row: p = 2^(s * c - m) (m already lowered by
// kFp8Offset, so p <= 256), row sum of the unrounded p, and four E4M3 codes per 32-bit
// column for the P.V MMA (key 4c in the lowest byte of column c).
__device__ __forceinline__ float exp_row_fp8(const uint32_t (&s)[4][32], float c,
                                             float m, uint32_t (&pk)[32]) {
  const uint64_t c2 = f32x2(c, c);
  const uint64_t nm2 = f32x2(-m, -m);
  uint64_t acc[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    float pv[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int e0 = 4 * q + 2 * h;
      const float s0 = __uint_as_float(s[e0 >> 5][e0 & 31]);
      const float s1 = __uint_as_float(s[(e0 + 1) >> 5][(e0 + 1) & 31]);
      const uint64_t x2 = fma_f32x2(f32x2(s0, s1), c2, nm2);
      float x0, x1;
      f32x2_split(x2, x0, x1);
      uint64_t p2;
      if (((2 * q + h) & 7) < ATTN_EXP2_EMU_PER8_FP8)
        p2 = exp2_poly_x2(x0, x1);
      else
        p2 = f32x2(ex2_approx(x0), ex2_approx(x1));
      acc[h] = add_f32x2(acc[h], p2);
      f32x2_split(p2, pv[2 * h], pv[2 * h + 1]);
    }
    pk[q] = pack_e4m3x4(pv[0], pv[1], pv[2], pv[3]);
  }
  float a0, a1, b0, b1;
  f32x2_split(acc[0], a0, a1);
  f32x2_split(acc[1], b0, b1);
  return (a0 + a1) + (b0 + b1);
}

template <int D, bool CAUSAL, bool FP8, bool SPARSE>
__device__ __forceinline__ void softmax_role(uint32_t base, uint32_t tmem,
                                             const CUtensorMap *tmo,
                                             const FwdParams &p,
                                             const WaitCtx &wc, int warp,
                                             int lane) {
  using L = Smem<D, FP8>;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };
  const int t = warp >> 2;          // which Q tile of the unit
  const int wq = warp & 3;          // TMEM lane quarter of this warp
  const int r = wq * 32 + lane;     // query row within the tile
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  constexpr bool kSplit = kSplitP<D, FP8, SPARSE>;
  const uint32_t tS = lane_base + t * 128;
  const uint32_t tO = lane_base + 256 + t * D;
  // where P goes: over S, or (split layout) its own 64 columns after O1
  const uint32_t tP = kSplit ? lane_base + 256 + 2 * D + t * 64 : tS;
  const float cl2 = p.c_log2;
  int scnt = 0, ocnt = 0;
  bool ok = true;

  for (int k = 0, u = unit_at<CAUSAL>(0); ok && u < p.num_units; u = unit_at<CAUSAL>(++k)) {
    const Unit w = get_unit<CAUSAL, SPARSE>(u, p);
    const int n = t ? w.n1 : w.n0;
    const int qs = w.q0 + kBlockM * t;
    if constexpr (SPARSE) {
      if (n == 0 && qs < p.n) {
        // No K tile computed for these rows: every score is masked, and the
        // output is written as O = 0, lse = -inf (a reading: the softmax of
        // an empty row is undefined).
        const uint32_t buf = base + L::kOut + static_cast<uint32_t>(warp) * L::kOutWarpBytes;
        const int y0 = qs + wq * 32;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          if (lane == 0) bulk_wait_group_read0();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c) st_shared_v4(buf + lane * 128 + c * 16, 0u, 0u, 0u, 0u);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && y0 < p.n) {
            tma_store_3d(tmo, buf, 64 * h, y0, w.bh);
            bulk_commit_group();
          }
        }
        if (qs + r < p.n) p.lse[static_cast<int64_t>(w.bh) * p.n + qs + r] = -CUDART_INF_F;
      }
    }
    if (n == 0) continue;
    const uint8_t *srow = nullptr;
    int kend = 0, kj = -1;  // block-sparse: the K tile of step j
    if constexpr (SPARSE) {
      const int tiles = (p.n + 127) >> 7, qt = qs >> 7;
      srow = sparse_row(p, w.bh, qt, tiles);
      kend = CAUSAL ? qt + 1 : tiles;
    }
    float m_run = -CUDART_INF_F;  // running max, log2 units (x = s * scale * log2 e)
    float l_run = 0.f;            // running sum of exp2(x - m_run)
    // FP8: the Q tile's scale joins the score multiplier; V's is applied at
    // the end (both are powers of two, so these products are exact)
    float cq = cl2, v_mul = 1.f;
    if constexpr (FP8) {
      cq = cl2 * __ldg(p.q_scale + static_cast<int64_t>(w.bh) * p.tiles + (qs >> 7));
      v_mul = __ldg(p.v_scale + w.bh);
    }
    const float* ksc = FP8 ? p.k_scale + static_cast<int64_t>(w.bh) * p.tiles : nullptr;

    for (int j = 0; j < n; ++j) {
      // K tile j's score multiplier, read before the wait hides its latency
      const float c = FP8 ? cq * __ldg(ksc + j) : cl2;
      ok = mbar_wait(bar(L::S_FULL + t), scnt & 1, wc, kRoleSoftmax);
      ++scnt;
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after_sync();

      bool mask;
      int limit;
      if constexpr (SPARSE) {
        // the causal diagonal tile, or the ragged last K tile
        kj = sparse_next(srow, kj + 1, kend);
        const bool diag = CAUSAL && kj == (qs >> 7);
        mask = diag || (kj == ((p.n - 1) >> 7) && (p.n & (kBlockN - 1)));
        limit = diag ? r : (p.n - 1 - kj * kBlockN);
      } else {
        mask = (j == n - 1) && (CAUSAL || (p.n & (kBlockN - 1)));
        limit = CAUSAL ? r : (p.n - 1 - j * kBlockN);
      }
      uint32_t s[4][32];
      load_scores(tS, s, mask, limit);
      if constexpr (kSplit) {
        // S is in registers: its columns may take the next S
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::S_FREE + t));
      }

      // Row max and the lazy base update: the base only moves when some row
      // of the warp gains more than 2^8 (warp-uniform decision, per-row
      // values); P then stays below 256 and O / l is unchanged because m and
      // l always move together.  The first tile of a row sets the base.
      // FP8: the base of a row moves when its own tile maximum exceeds it by
      // more than kFp8Threshold (a per-row decision, so each row's base is a
      // function of that row alone); the warp rescales O when any row moved,
      // the others by exactly 1.
      const float m_tile = row_max_raw(s) * c;
      float alpha = 1.f;
      bool update = false;
      if (j == 0) {
        m_run = m_tile;
      } else if constexpr (FP8) {
        const bool mine = m_tile > m_run + kFp8Threshold;
        update = __any_sync(0xffffffffu, mine);
        if (update) {
          const float m_new = mine ? m_tile : m_run;
          alpha = ex2_approx(m_run - m_new);
          l_run *= alpha;
          m_run = m_new;
        }
      } else {
        update = __any_sync(0xffffffffu, m_tile > m_run + kRescaleThreshold);
        if (update) {
          const float m_new = fmaxf(m_run, m_tile);
          alpha = ex2_approx(m_run - m_new);
          l_run *= alpha;
          m_run = m_new;
        }
      }
      float row_sum;
      if constexpr (FP8) {
        uint32_t pk[32];
        row_sum = exp_row_fp8(s, c, m_run - kFp8Offset, pk);
        tmem_st_32x32b_x32(tS + 0, pk);
      } else {
        // The first half's P is stored while the second half is computed,
        // and announced (P_HALF) a quarter of the way through it, so that the
        // P.V of the first 64 keys overlaps the rest.  O is rescaled before
        // that announcement: the P.V then adds to the rescaled O.  O holds
        // the earlier P.V products only; the S_FULL commit for this tile was
        // issued after the previous P.V, so that MMA has completed.
        // In the split layout this tile's next S may have been issued
        // before the last P.V, so that P.V is awaited here (O_FULL) before
        // P's columns are overwritten or O rescaled.
        uint32_t pk[2][32];
        row_sum = exp_row<D, 0>(s, c, m_run, pk[0]);
        if constexpr (kSplit) {
          if (j > 0) {
            ok = mbar_wait(bar(L::O_FULL + t), ocnt & 1, wc, kRoleSoftmax);
            ++ocnt;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after_sync();
          }
        }
        tmem_st_32x32b_x32(tP + 0, pk[0]);
        if (update) rescale_o<D>(tO, alpha);
        row_sum += exp_row<D, 1, 0, 8>(s, c, m_run, pk[1]);
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::P_HALF + t));
        row_sum += exp_row<D, 1, 8, 32>(s, c, m_run, pk[1]);
        tmem_st_32x32b_x32(tP + 32, pk[1]);
      }
      l_run += row_sum;
      if constexpr (FP8) {
        // O holds the earlier P.V products; the S_FULL commit for this tile
        // was issued after the previous P.V, so that MMA has completed.
        if (update) rescale_o<D>(tO, alpha);
      }
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::P_FULL + t));
    }
    if (!ok) break;

    // ---- epilogue: O / l -> bf16 -> this row of O in HBM; lse
    // (the last P.V's O_FULL phase; the split layout has consumed the others)
    ocnt += kSplit ? 1 : n;
    ok = mbar_wait(bar(L::O_FULL + t), (ocnt - 1) & 1, wc, kRoleEpilogue);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    tc_fence_after_sync();
    const float inv_l = __frcp_rn(l_run) * v_mul;
    int64_t grow = static_cast<int64_t>(w.bh) * p.n + qs + r;
    if constexpr (kDebugBounds) {
      // injected index error (debug builds only): the first row stored by
      // CTA 0 points past the output, which the check below must catch
      if ((p.debug_flags & 4u) && blockIdx.x == 0 && k == 0 && t == 0 && r == 0)
        grow += static_cast<int64_t>(p.bh) * p.n;
    }
    // a row past N is never stored; in the debug build neither is a row
    // whose unit or global index is out of range
    const bool row_ok = qs + r < p.n && in_bounds(w.bh, p.bh, p.status) &&
                        in_bounds(qs, p.n, p.status) &&
                        in_bounds(grow, static_cast<int64_t>(p.bh) * p.n, p.status);
    // this block's log-sum-exp (natural log)
    const float lse_this = (m_run - (FP8 ? kFp8Offset : 0.f) + lg2_approx(l_run)) * kLn2;
    float lse_out = lse_this;
    if (p.merge_mode == kMergeNone) {
      // The row of O leaves TMEM first, so that its columns go back to the
      // next unit's P.V as early as possible.  It then reaches HBM through
      // shared memory: each warp stages its 32 rows x 64 columns in the
      // 128B-swizzled layout of the O tensor map, and one lane issues a TMA
      // tensor store, so the global writes are whole 128-byte row segments
      // rather than 16-byte pieces 2 D bytes apart.  The tensor map clips
      // rows at or past N.
      uint32_t ov[D / 32][32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld_32x32b_x32(tO + c * 32, ov[c]);
      tmem_wait_ld(ov[0]);
#pragma unroll
      for (int c = 1; c < D / 32; ++c) reg_fence(ov[c]);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::O_EMPTY + t));  // O columns reusable
      const uint32_t buf = base + L::kOut + static_cast<uint32_t>(warp) * L::kOutWarpBytes;
      const int y0 = qs + wq * 32;
      int zc = w.bh;
      if constexpr (kDebugBounds) {
        // the injected index error of the debug build (see grow above)
        if ((p.debug_flags & 4u) && blockIdx.x == 0 && k == 0 && t == 0 && wq == 0)
          zc += p.bh;
      }
      const bool store_ok =
          y0 < p.n && in_bounds(zc, p.bh, p.status) && in_bounds(y0, p.n, p.status);
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        uint32_t wv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int col = 64 * h + 2 * i;
          wv[i] = pack_bf16x2(__uint_as_float(ov[col >> 5][col & 31]) * inv_l,
                              __uint_as_float(ov[(col + 1) >> 5][(col + 1) & 31]) * inv_l);
        }
        if (lane == 0) bulk_wait_group_read0();  // the previous store has read the buffer
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(buf + lane * 128 + ((c ^ (lane & 7)) << 4), wv[4 * c],
                       wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && store_ok) {
          tma_store_3d(tmo, buf, 64 * h, y0, zc);
          bulk_commit_group();
        }
      }
    } else {
      // weights of the accumulator and of this block: exp(lse_x - lse_new)
      float wa = 0.f, wp = 1.f;
      if (p.merge_mode != kMergeFirst && row_ok) {
        const float la = p.acc_lse[grow];
        const float mx = fmaxf(la, lse_this);
        wa = (la == -CUDART_INF_F) ? 0.f : ex2_approx((la - mx) * 1.4426950408889634f);
        wp = ex2_approx((lse_this - mx) * 1.4426950408889634f);
        const float tot = wa + wp;
        lse_out = mx + lg2_approx(tot) * kLn2;
        const float it = __frcp_rn(tot);
        wa *= it;
        wp *= it;
      }
      float4 *arow = reinterpret_cast<float4 *>(p.acc_o + grow * D);
      uint4 *orow = reinterpret_cast<uint4 *>(p.o + grow * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tO + c * 32, o);
        tmem_wait_ld(o);
        if (!row_ok) continue;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o[i]) * inv_l * wp;
        if (p.merge_mode != kMergeFirst) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 a4 = arow[c * 8 + i];
            v[4 * i] = fmaf(wa, a4.x, v[4 * i]);
            v[4 * i + 1] = fmaf(wa, a4.y, v[4 * i + 1]);
            v[4 * i + 2] = fmaf(wa, a4.z, v[4 * i + 2]);
            v[4 * i + 3] = fmaf(wa, a4.w, v[4 * i + 3]);
          }
        }
        if (p.merge_mode == kMergeLast) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            orow[c * 4 + i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]),
                                         pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                         pack_bf16x2(v[8 * i + 4], v[8 * i + 5]),
                                         pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            arow[c * 8 + i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::O_EMPTY + t));  // O columns reusable
    }
    if (row_ok) {
      if (p.merge_mode == kMergeFirst || p.merge_mode == kMergeInto)
        p.acc_lse[grow] = lse_out;
      else
        p.lse[grow] = lse_out;
    }
  }
  // every TMA store this warp issued must be complete before the CTA exits
  if (lane == 0) bulk_wait_group0();
}

// ------------------------------------------------------------------ kernel

template <int D, bool CAUSAL, bool FP8 = false, bool SPARSE = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_o,
                          const FwdParams p) {
  using L = Smem<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    const uint32_t b0 = base + L::kBars;
    for (int t = 0; t < 2; ++t) {
      mbar_init(b0 + 8 * (L::Q_FULL + t), 1);
      mbar_init(b0 + 8 * (L::Q_EMPTY + t), 1);
      mbar_init(b0 + 8 * (L::S_FULL + t), 1);
      mbar_init(b0 + 8 * (L::P_FULL + t), 4);
      mbar_init(b0 + 8 * (L::P_HALF + t), 4);
      mbar_init(b0 + 8 * (L::S_FREE + t), 4);
      mbar_init(b0 + 8 * (L::O_FULL + t), 1);
      mbar_init(b0 + 8 * (L::O_EMPTY + t), 4);
    }
    // with one issuer per Q tile, both commit to DRAIN and to every EMPTY
    const uint32_t issuers = kPerTileIssuer<D, FP8, SPARSE> ? 2 : 1;
    mbar_init(b0 + 8 * L::DRAIN, issuers);
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(b0 + 8 * (L::K_FULL + s), 1);
      mbar_init(b0 + 8 * (L::K_EMPTY + s), issuers);
    }
    for (int s = 0; s < L::kVStages; ++s) {
      mbar_init(b0 + 8 * (L::V_FULL + s), 1);
      mbar_init(b0 + 8 * (L::V_EMPTY + s), issuers);
    }
    *abort_flag = 0;
    for (int s = 0; s < L::kKStages + L::kVStages; ++s)
      reinterpret_cast<volatile int *>(smem + L::kSlotPos)[s] = -1;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    if (p.merge_mode == kMergeNone) prefetch_tensormap(&tm_o);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.status, p.timeout_ns};

  if (warp < 8) {
    setmaxnreg_inc<kSoftmaxRegs>();
    softmax_role<D, CAUSAL, FP8, SPARSE>(base, tmem, &tm_o, p, wc, warp, lane);
  } else {
    setmaxnreg_dec<kControlRegs>();
    if (warp == kProducerWarp) {
      if (lane == 0)
        producer_role<D, CAUSAL, kLoadQK, FP8, SPARSE>(base, &tm_q, &tm_k, &tm_v, p, wc);
    } else if (warp == kVLoaderWarp) {
      if (lane == 0)
        producer_role<D, CAUSAL, kLoadV, FP8, SPARSE>(base, &tm_q, &tm_k, &tm_v, p, wc);
    } else if (warp == kMmaWarp) {
      if (lane == 0) {
        if constexpr (kPerTileIssuer<D, FP8, SPARSE>)
          mma_role_tile<D, CAUSAL, FP8, SPARSE>(base, tmem, p, wc, 0);
        else
          mma_role<D, CAUSAL, FP8, SPARSE>(base, tmem, p, wc);
      }
    } else if (warp == kMmaWarp2) {
      if constexpr (kPerTileIssuer<D, FP8, SPARSE>) {
        if (lane == 0) mma_role_tile<D, CAUSAL, FP8, SPARSE>(base, tmem, p, wc, 1);
      }
    }
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn_b200
