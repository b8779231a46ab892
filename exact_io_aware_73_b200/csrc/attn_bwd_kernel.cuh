// attn_bwd_kernel.cuh -- backward pass of exact attention for B200 (sm_100a).
//
// Source cited as [MM]: the marketmaker.cc blog post (Indonesian edition)
// "Apakah Konteks Sehari Penuh Mengalahkan Konteks Sepuluh Menit? Perhatian
// Kilat dan Pertanyaan Panjang Urutan", section "Backward pass: menghitung
// ulang, bukan menyimpan": the backward pass keeps only O and the softmax
// statistics of the forward (here lse = m + ln l) and recomputes the score
// tiles from Q and K instead of storing the N x N probabilities.
//
// Gradients of O = softmax(scale Q K^T [mask]) V for an upstream gradient dO
// (the calculus of the forward definition; the pages give no formulas):
//     P = exp(scale Q K^T - lse)   (recomputed per tile from the saved lse)
//     dV = P^T dO      dP = dO V^T      D_i = sum_t dO_it O_it
//     dS = P * (dP - D)             dQ = scale dS K      dK = scale dS^T Q
//
// Three kernels, all persistent with bounded waits like the forward:
//   attn_bwd_prep_kernel    D_i, one warp per row (bandwidth-bound);
//   attn_bwd_dq_kernel      one 128-row Q tile per unit, loop over K/V tiles:
//                           S = Q K^T and dP = dO V^T (tcgen05, TMEM), the
//                           compute warpgroup forms dS over S, dQ += dS K;
//   attn_bwd_dkdv_kernel    one 128-key K/V tile per unit, loop over Q tiles:
//                           S^T = K Q^T and dP^T = V dO^T, the compute
//                           warpgroup forms P^T and dS^T (lse and D per query
//                           column come from shared memory), dV += P^T dO,
//                           dK += dS^T Q.
// Each tcgen05 MMA has one of the two forms of the forward kernel: A and B
// K-major in shared memory (N = 128), or A from TMEM and B MN-major (N = d).
#pragma once

#include "attn_fwd_kernel.cuh"

namespace attn_b200 {

// Warps 0-7 compute, 8 loader, 9 MMA.  The compute work on a tile is
// elementwise (P from the saved lse, dS from P, dP and D), so the two
// compute warpgroups split its columns: warp w takes TMEM lane quarter w % 4
// (rows 32 (w % 4) ..) and the 64 columns of half w / 4.  Two warps per SM
// sub-partition hide each other's TMEM and MUFU latencies.
constexpr int kBwdComputeWarps = 8;
constexpr int kBwdThreads = 320;
constexpr int kBwdLoaderWarp = 8;
constexpr int kBwdMmaWarp = 9;

// The two compute warps of TMEM lane quarter wq (warps wq and wq + 4) meet
// here between loading their fp32 columns and storing bf16 results: chunk c's
// bf16 values go to columns 16c .. 16c + 15, so the upper half's results
// (c = 2, 3) land on fp32 columns 32 .. 63, which the lower half reads.
__device__ __forceinline__ void bwd_pair_sync(int wq) {
  tc_fence_before_sync();
  asm volatile("barrier.cta.sync %0, 64;" ::"r"(1 + wq) : "memory");
  tc_fence_after_sync();
}

// Pairs of exponentials (out of every 8) that the compute warps evaluate on
// the FMA pipe (exp2_poly_x2) instead of the MUFU unit: at d = 64 the
// exponentials weigh twice as much per tensor-core FLOP as at d = 128, and
// two pairs in eight measured best (the polynomial's relative error, below
// 8e-5, is far inside the bf16 rounding of P).
#ifndef ATTN_BWD_EXP2_EMU_PER8_D64
#define ATTN_BWD_EXP2_EMU_PER8_D64 2
#endif
template <int D>
constexpr int kBwdEmuPer8 = (D == 64) ? ATTN_BWD_EXP2_EMU_PER8_D64 : 0;

// Two exponentials of a pair: the FMA-pipe polynomial for the first
// kBwdEmuPer8<D> pairs of every 8, ex2.approx otherwise.
template <int D>
__device__ __forceinline__ void bwd_exp2_pair(int pair, uint64_t x2, float &p0, float &p1) {
  float x0, x1;
  f32x2_split(x2, x0, x1);
  if ((pair & 7) < kBwdEmuPer8<D>) {
    f32x2_split(exp2_poly_x2(x0, x1), p0, p1);
  } else {
    p0 = ex2_approx(x0);
    p1 = ex2_approx(x1);
  }
}

struct BwdParams {
  const uint16_t *o;     // [BH, N, D] forward output (prep only)
  const uint16_t *dout;  // [BH, N, D] upstream gradient (prep only)
  const float *lse;      // [BH, N] forward log-sum-exp, natural log (prep only)
  // Workspace, rows padded to npad = 128 * tiles so every 128-row TMA tile of
  // these fp32 vectors starts on a 512-byte boundary; padding rows hold 0.
  // Both are stored negated: the compute warps add them (packed f32x2
  // arithmetic has no negated operand).
  float *lse2;           // [BH, npad] -lse * log2(e)
  float *dsum;           // [BH, npad] -D_i, D_i = sum_t dO_it O_it
  uint16_t *dq, *dk, *dv;  // [BH, N, D] outputs
  uint32_t *status;
  int bh, n, npad, tiles, num_units;
  float c_log2;          // scale * log2(e)
  float scale;
  unsigned long long timeout_ns;
};

// ------------------------------------------------------------------ prep

// -D_i (D_i = sum_t dO_it * O_it) and -lse_i * log2(e) for every row, fp32,
// into the padded workspace vectors (0 in padding rows); one warp per row.
template <int D>
__global__ void __launch_bounds__(256)
    attn_bwd_prep_kernel(const BwdParams p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(p.bh) * p.npad;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int64_t prow = warp; prow < rows; prow += nwarps) {
    const int64_t bh = prow / p.npad;
    const int n = static_cast<int>(prow - bh * p.npad);
    float acc = 0.f, l2 = 0.f;
    if (n < p.n) {
      const int64_t row = bh * p.n + n;
      const uint16_t *a = p.o + row * D + lane * (D / 32);
      const uint16_t *b = p.dout + row * D + lane * (D / 32);
#pragma unroll
      for (int t = 0; t < D / 32; ++t)
        acc += __uint_as_float(static_cast<uint32_t>(a[t]) << 16) *
               __uint_as_float(static_cast<uint32_t>(b[t]) << 16);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, off);
      l2 = p.lse[row] * 1.4426950408889634f;
    }
    if (lane == 0) {
      p.dsum[prow] = -acc;
      p.lse2[prow] = -l2;
    }
  }
}

// ------------------------------------------------------------------ dQ

template <int D>
struct BwdDqSmem {
  static constexpr uint32_t kTile = Smem<D>::kTileBytes;
  static constexpr uint32_t kPanel = Smem<D>::kPanelBytes;
  static constexpr int kSub = D / 64;
  static constexpr int kStages = (D == 128) ? 2 : 4;  // K+V ring
  static constexpr uint32_t kQ = 0, kDO = kTile;
  static constexpr uint32_t kK = 2 * kTile;
  static constexpr uint32_t kV = kK + kStages * kTile;
  static constexpr uint32_t kBars = kV + kStages * kTile;
  static constexpr int Q_FULL = 0, Q_EMPTY = 1, S_FULL = 2, DS_FULL = 3,
                       ACC_FULL = 4, ACC_EMPTY = 5, DRAIN = 6, DP_FULL = 7,
                       S_FREE = 8, KV_FULL = 9, KV_EMPTY = KV_FULL + kStages,
                       NUM_BARS = KV_EMPTY + kStages;
  static constexpr uint32_t kMisc = kBars + NUM_BARS * 8;
  static constexpr uint32_t kAlloc = kMisc + 16 + 1024;
  static_assert(kAlloc <= 232448, "shared memory budget");
};

template <bool CAUSAL>
__device__ __forceinline__ void dq_unit(int u, int bh_count, int tiles,
                                        int &bh, int &qt, int &nkv) {
  if (CAUSAL) {  // longest rows first
    qt = tiles - 1 - u / bh_count;
    bh = u % bh_count;
    nkv = qt + 1;
  } else {
    bh = u / tiles;
    qt = u % tiles;
    nkv = tiles;
  }
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const BwdParams p) {
  using L = BwdDqSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };

  if (tid == 0) {
    mbar_init(bar(L::Q_FULL), 1);
    mbar_init(bar(L::Q_EMPTY), 1);
    mbar_init(bar(L::S_FULL), 1);
    mbar_init(bar(L::DP_FULL), 1);
    mbar_init(bar(L::S_FREE), kBwdComputeWarps);
    mbar_init(bar(L::DS_FULL), kBwdComputeWarps);
    mbar_init(bar(L::ACC_FULL), 1);
    mbar_init(bar(L::ACC_EMPTY), kBwdComputeWarps);
    mbar_init(bar(L::DRAIN), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::KV_FULL + s), 1);
      mbar_init(bar(L::KV_EMPTY + s), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.status, p.timeout_ns};
  // TMEM: S (cols 0-127), dP (128-255, dS written over it), dQ (256-256+D)
  const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 256;

  if (warp == kBwdLoaderWarp) {
    if (lane == 0) {
      int uocc = 0, kv_issued = 0;
      bool ok = true;
      for (int k = 0, u = unit_at<CAUSAL>(0); ok && u < p.num_units; u = unit_at<CAUSAL>(++k)) {
        int bh, qt, nkv;
        dq_unit<CAUSAL>(u, p.bh, p.tiles, bh, qt, nkv);
        if (uocc > 0) {
          ok = mbar_wait(bar(L::Q_EMPTY), (uocc - 1) & 1, wc, kRoleProducer);
          if (!ok) break;
        }
        ++uocc;
        mbar_arrive_expect_tx(bar(L::Q_FULL), 2 * L::kTile);
        for (int s = 0; s < L::kSub; ++s) {
          tma_load_3d(base + L::kQ + s * L::kPanel, &tm_q, bar(L::Q_FULL), s * 64,
                      qt * kBlockM, bh);
          tma_load_3d(base + L::kDO + s * L::kPanel, &tm_do, bar(L::Q_FULL),
                      s * 64, qt * kBlockM, bh);
        }
        for (int j = 0; j < nkv; ++j) {
          const int st = kv_issued % L::kStages;
          ok = mbar_wait(bar(L::KV_EMPTY + st), ((kv_issued / L::kStages) & 1) ^ 1,
                         wc, kRoleProducer);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::KV_FULL + st), 2 * L::kTile);
          for (int s = 0; s < L::kSub; ++s) {
            tma_load_3d(base + L::kK + st * L::kTile + s * L::kPanel, &tm_k,
                        bar(L::KV_FULL + st), s * 64, j * kBlockN, bh);
            tma_load_3d(base + L::kV + st * L::kTile + s * L::kPanel, &tm_v,
                        bar(L::KV_FULL + st), s * 64, j * kBlockN, bh);
          }
          ++kv_issued;
        }
      }
      if (*wc.abort) {
        if (uocc > 0) mbar_wait_drain(bar(L::Q_FULL), (uocc - 1) & 1, wc);
        for (int st = 0; st < L::kStages; ++st)
          if (kv_issued > st) {
            const int last = st + ((kv_issued - 1 - st) / L::kStages) * L::kStages;
            mbar_wait_drain(bar(L::KV_FULL + st), (last / L::kStages) & 1, wc);
          }
      }
    }
    __syncwarp();
  } else if (warp == kBwdMmaWarp) {
    if (lane == 0) {
      // Per K/V tile j: S_j and dP_j; the compute warps read S_j (P phase),
      // release it (S_FREE) and form dS_j over dP_j (dS phase).  S_{j+1} is
      // issued as soon as S_j is free, so it runs during the dS phase; dQ_j
      // and dP_{j+1} run during the next P phase.
      int uocc = 0, kv_cons = 0, jcnt = 0;
      bool ok = true;
      for (int k = 0, u = unit_at<CAUSAL>(0); ok && u < p.num_units; u = unit_at<CAUSAL>(++k)) {
        int bh, qt, nkv;
        dq_unit<CAUSAL>(u, p.bh, p.tiles, bh, qt, nkv);
        ok = mbar_wait_spin(bar(L::Q_FULL), uocc & 1, wc, kRoleMma);
        if (!ok) break;
        auto stage_of = [&](int idx) { return idx % L::kStages; };
        auto k_tile = [&](int idx) { return base + L::kK + stage_of(idx) * L::kTile; };
        auto v_tile = [&](int idx) { return base + L::kV + stage_of(idx) * L::kTile; };
        // prologue: S_0, dP_0
        ok = mbar_wait_spin(bar(L::KV_FULL + stage_of(kv_cons)),
                            (kv_cons / L::kStages) & 1, wc, kRoleMma);
        if (!ok) break;
        tc_fence_after_sync();
        issue_qk<D>(tS, base + L::kQ, k_tile(kv_cons));     // S  = Q  K^T
        mma_commit(bar(L::S_FULL));
        issue_qk<D>(tdP, base + L::kDO, v_tile(kv_cons));   // dP = dO V^T
        mma_commit(bar(L::DP_FULL));
        if (nkv == 1) mma_commit(bar(L::Q_EMPTY));  // last read of Q, dO
        for (int j = 0; j < nkv; ++j) {
          const int cur = kv_cons + j;
          const int nxt = cur + 1;
          if (j + 1 < nkv) {
            ok = mbar_wait_spin(bar(L::KV_FULL + stage_of(nxt)),
                                (nxt / L::kStages) & 1, wc, kRoleMma);
            if (!ok) break;
            ok = mbar_wait_spin(bar(L::S_FREE), (jcnt + j) & 1, wc, kRoleMma);
            if (!ok) break;
            tc_fence_after_sync();
            issue_qk<D>(tS, base + L::kQ, k_tile(nxt));
            mma_commit(bar(L::S_FULL));
          }
          ok = mbar_wait_spin(bar(L::DS_FULL), (jcnt + j) & 1, wc, kRoleMma);
          if (!ok) break;
          if (j == 0 && uocc > 0) {
            ok = mbar_wait_spin(bar(L::ACC_EMPTY), (uocc - 1) & 1, wc, kRoleMma);
            if (!ok) break;
          }
          tc_fence_after_sync();
          issue_pv<D>(tdQ, tdP, k_tile(cur), j > 0);   // dQ += dS K
          mma_commit(bar(L::KV_EMPTY + stage_of(cur)));
          if (j + 1 < nkv) {
            // after dQ_j in this thread: dS_j has been read from these columns
            issue_qk<D>(tdP, base + L::kDO, v_tile(nxt));
            mma_commit(bar(L::DP_FULL));
            if (j + 2 == nkv) mma_commit(bar(L::Q_EMPTY));  // last read of Q, dO
          }
        }
        if (!ok) break;
        kv_cons += nkv;
        jcnt += nkv;
        mma_commit(bar(L::ACC_FULL));
        ++uocc;
      }
      mma_commit(bar(L::DRAIN));
      mbar_wait_drain(bar(L::DRAIN), 0, wc);
    }
    __syncwarp();
  } else {
    // compute warpgroups: thread = query row r of the tile, columns of half hc
    const int wq = warp & 3;  // TMEM lane quarter
    const int hc = warp >> 2;  // 64-column half of the tile
    const int r = wq * 32 + lane;
    const uint32_t lb = static_cast<uint32_t>(wq * 32) << 16;
    int s_cnt = 0, uocc = 0;
    bool ok = true;
    for (int k = 0, u = unit_at<CAUSAL>(0); ok && u < p.num_units; u = unit_at<CAUSAL>(++k)) {
      int bh, qt, nkv;
      dq_unit<CAUSAL>(u, p.bh, p.tiles, bh, qt, nkv);
      const int row = qt * kBlockM + r;  // < npad: padded vectors in range
      const bool row_ok = row < p.n;
      const int64_t grow = static_cast<int64_t>(bh) * p.n + row;
      const int64_t prow = static_cast<int64_t>(bh) * p.npad + row;
      const uint64_t nlse2 = f32x2(p.lse2[prow], p.lse2[prow]);  // -lse log2(e)
      const uint64_t ndrow2 = f32x2(p.dsum[prow], p.dsum[prow]);  // -D
      const uint64_t c2 = f32x2(p.c_log2, p.c_log2);
      for (int j = 0; j < nkv; ++j) {
        // ---- P phase: P_j from S_j, kept in registers; S released
        ok = mbar_wait(bar(L::S_FULL), s_cnt & 1, wc, kRoleSoftmax);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after_sync();
        const bool mask = (j == nkv - 1) && (CAUSAL || (p.n & (kBlockN - 1)));
        const int limit = CAUSAL ? r : (p.n - 1 - j * kBlockN);
        float pr[64];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * hc + cc;  // 32-column chunk of the tile
          uint32_t sv[32];
          tmem_ld_32x32b_x32(tS + lb + c * 32, sv);
          tmem_wait_ld(sv);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const uint64_t x2 = fma_f32x2(
                f32x2(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), c2, nlse2);
            bwd_exp2_pair<D>(i >> 1, x2, pr[cc * 32 + i], pr[cc * 32 + i + 1]);
          }
          if (mask) {  // the last K tile only
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i > limit) pr[cc * 32 + i] = 0.f;
          }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::S_FREE));
        // ---- dS phase: dS_j = P_j (dP_j - D) written over dP_j
        ok = mbar_wait(bar(L::DP_FULL), s_cnt & 1, wc, kRoleSoftmax);
        ++s_cnt;
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after_sync();
        uint32_t dv[2][32];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) tmem_ld_32x32b_x32(tdP + lb + (2 * hc + cc) * 32, dv[cc]);
        tmem_wait_ld(dv[0]);
        reg_fence(dv[1]);
        bwd_pair_sync(wq);  // both halves hold their dP before dS overwrites it
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * hc + cc;
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint64_t t2 = add_f32x2(
                f32x2(__uint_as_float(dv[cc][2 * i]), __uint_as_float(dv[cc][2 * i + 1])),
                ndrow2);
            float d0, d1;
            f32x2_split(mul_f32x2(f32x2(pr[cc * 32 + 2 * i], pr[cc * 32 + 2 * i + 1]), t2),
                        d0, d1);
            pk[i] = pack_bf16x2(d0, d1);
          }
          tmem_st_32x32b_x16(tdP + lb + c * 16, pk);  // bf16 dS over dP columns
        }
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::DS_FULL));
      }
      if (!ok) break;
      ok = mbar_wait(bar(L::ACC_FULL), uocc & 1, wc, kRoleEpilogue);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++uocc;
      tc_fence_after_sync();
      uint4 *out = reinterpret_cast<uint4 *>(p.dq + grow * D);
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        const int c = hc * (D / 64) + cc;  // this half's 32-column chunks of dQ
        uint32_t o[32];
        tmem_ld_32x32b_x32(tdQ + lb + c * 32, o);
        tmem_wait_ld(o);
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          h[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * p.scale,
                             __uint_as_float(o[2 * i + 1]) * p.scale);
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            out[c * 4 + i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2],
                                        h[4 * i + 3]);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::ACC_EMPTY));
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ dK, dV

template <int D>
struct BwdDkvSmem {
  static constexpr uint32_t kTile = Smem<D>::kTileBytes;
  static constexpr uint32_t kPanel = Smem<D>::kPanelBytes;
  static constexpr int kSub = D / 64;
  static constexpr int kStages = (D == 128) ? 2 : 4;  // Q+dO+lse+D ring
  // one stage: Q tile, dO tile, 128 lse, 128 D (fp32), 1024-aligned
  static constexpr uint32_t kStage = 2 * kTile + 1024;
  static constexpr uint32_t kK = 0, kV = kTile;
  static constexpr uint32_t kRing = 2 * kTile;
  static constexpr uint32_t kBars = kRing + kStages * kStage;
  static constexpr int KV_FULL = 0, KV_EMPTY = 1, S_FULL = 2, DP_FULL = 3,
                       P_READY = 4, DS_READY = 5, ACC_FULL = 6, ACC_EMPTY = 7,
                       DRAIN = 8, Q_FULL = 9, Q_EMPTY = Q_FULL + kStages,
                       NUM_BARS = Q_EMPTY + kStages;
  static constexpr uint32_t kMisc = kBars + NUM_BARS * 8;
  static constexpr uint32_t kAlloc = kMisc + 16 + 1024;
  static_assert(kAlloc <= 232448, "shared memory budget");
};

template <bool CAUSAL>
__device__ __forceinline__ void dkv_unit(int u, int bh_count, int tiles,
                                         int &bh, int &kt, int &q_first) {
  if (CAUSAL) {  // key tiles seen by the most queries first
    kt = u / bh_count;
    bh = u % bh_count;
    q_first = kt;
  } else {
    bh = u / tiles;
    kt = u % tiles;
    q_first = 0;
  }
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_lse,
                         const __grid_constant__ CUtensorMap tm_dsum,
                         const BwdParams p) {
  using L = BwdDkvSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };

  if (tid == 0) {
    mbar_init(bar(L::KV_FULL), 1);
    mbar_init(bar(L::KV_EMPTY), 1);
    mbar_init(bar(L::S_FULL), 1);
    mbar_init(bar(L::DP_FULL), 1);
    mbar_init(bar(L::P_READY), kBwdComputeWarps);
    mbar_init(bar(L::DS_READY), kBwdComputeWarps);
    mbar_init(bar(L::ACC_FULL), 1);
    mbar_init(bar(L::ACC_EMPTY), kBwdComputeWarps);
    mbar_init(bar(L::DRAIN), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::Q_FULL + s), 1);
      mbar_init(bar(L::Q_EMPTY + s), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.status, p.timeout_ns};
  // TMEM: S^T (0-127, P^T over it), dP^T (128-255, dS^T over it), dV, dK
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256,
                 tdK = tmem + 256 + D;

  if (warp == kBwdLoaderWarp) {
    if (lane == 0) {
      int uocc = 0, q_issued = 0;
      bool ok = true;
      for (int k = 0, u = unit_at<CAUSAL>(0); ok && u < p.num_units; u = unit_at<CAUSAL>(++k)) {
        int bh, kt, q0;
        dkv_unit<CAUSAL>(u, p.bh, p.tiles, bh, kt, q0);
        if (uocc > 0) {
          ok = mbar_wait(bar(L::KV_EMPTY), (uocc - 1) & 1, wc, kRoleProducer);
          if (!ok) break;
        }
        ++uocc;
        mbar_arrive_expect_tx(bar(L::KV_FULL), 2 * L::kTile);
        for (int s = 0; s < L::kSub; ++s) {
          tma_load_3d(base + L::kK + s * L::kPanel, &tm_k, bar(L::KV_FULL), s * 64,
                      kt * kBlockN, bh);
          tma_load_3d(base + L::kV + s * L::kPanel, &tm_v, bar(L::KV_FULL), s * 64,
                      kt * kBlockN, bh);
        }
        for (int i = q0; i < p.tiles; ++i) {
          const int st = q_issued % L::kStages;
          ok = mbar_wait(bar(L::Q_EMPTY + st), ((q_issued / L::kStages) & 1) ^ 1,
                         wc, kRoleProducer);
          if (!ok) break;
          const uint32_t sb = base + L::kRing + st * L::kStage;
          mbar_arrive_expect_tx(bar(L::Q_FULL + st), 2 * L::kTile + 1024);
          for (int s = 0; s < L::kSub; ++s) {
            tma_load_3d(sb + s * L::kPanel, &tm_q, bar(L::Q_FULL + st), s * 64,
                        i * kBlockM, bh);
            tma_load_3d(sb + L::kTile + s * L::kPanel, &tm_do, bar(L::Q_FULL + st),
                        s * 64, i * kBlockM, bh);
          }
          tma_load_2d(sb + 2 * L::kTile, &tm_lse, bar(L::Q_FULL + st), i * kBlockM, bh);
          tma_load_2d(sb + 2 * L::kTile + 512, &tm_dsum, bar(L::Q_FULL + st),
                      i * kBlockM, bh);
          ++q_issued;
        }
      }
      if (*wc.abort) {
        if (uocc > 0) mbar_wait_drain(bar(L::KV_FULL), (uocc - 1) & 1, wc);
        for (int st = 0; st < L::kStages; ++st)
          if (q_issued > st) {
            const int last = st + ((q_issued - 1 - st) / L::kStages) * L::kStages;
            mbar_wait_drain(bar(L::Q_FULL + st), (last / L::kStages) & 1, wc);
          }
      }
    }
    __syncwarp();
  } else if (warp == kBwdMmaWarp) {
    if (lane == 0) {
      // Per Q tile i: S^T_i and dP^T_i; the compute warps form P^T_i over
      // S^T_i (P phase, P_READY), then dS^T_i over dP^T_i (dS phase,
      // DS_READY).  dV_i and S^T_{i+1} run during the dS phase, dK_i and
      // dP^T_{i+1} during the next P phase.  Each MMA that overwrites S^T or
      // dP^T is issued after the one reading P^T or dS^T from those columns.
      int uocc = 0, q_cons = 0, tcnt = 0;
      bool ok = true;
      for (int k = 0, u = unit_at<CAUSAL>(0); ok && u < p.num_units; u = unit_at<CAUSAL>(++k)) {
        int bh, kt, q0;
        dkv_unit<CAUSAL>(u, p.bh, p.tiles, bh, kt, q0);
        ok = mbar_wait_spin(bar(L::KV_FULL), uocc & 1, wc, kRoleMma);
        if (!ok) break;
        auto ring = [&](int idx) {
          return base + L::kRing + (idx % L::kStages) * L::kStage;
        };
        // prologue: S^T and dP^T of the first Q tile
        ok = mbar_wait_spin(bar(L::Q_FULL + q_cons % L::kStages),
                            (q_cons / L::kStages) & 1, wc, kRoleMma);
        if (!ok) break;
        tc_fence_after_sync();
        issue_qk<D>(tS, base + L::kK, ring(q_cons));               // S^T  = K Q^T
        mma_commit(bar(L::S_FULL));
        issue_qk<D>(tdP, base + L::kV, ring(q_cons) + L::kTile);   // dP^T = V dO^T
        mma_commit(bar(L::DP_FULL));
        if (q0 == p.tiles - 1) mma_commit(bar(L::KV_EMPTY));  // last K, V read
        for (int i = q0; i < p.tiles; ++i) {
          const int cur = q_cons + (i - q0);
          const int nxt = cur + 1;
          const int t = tcnt + (i - q0);
          ok = mbar_wait_spin(bar(L::P_READY), t & 1, wc, kRoleMma);
          if (!ok) break;
          if (i == q0 && uocc > 0) {
            ok = mbar_wait_spin(bar(L::ACC_EMPTY), (uocc - 1) & 1, wc, kRoleMma);
            if (!ok) break;
          }
          tc_fence_after_sync();
          issue_pv<D>(tdV, tS, ring(cur) + L::kTile, i > q0);  // dV += P^T dO
          if (i + 1 < p.tiles) {
            ok = mbar_wait_spin(bar(L::Q_FULL + nxt % L::kStages),
                                (nxt / L::kStages) & 1, wc, kRoleMma);
            if (!ok) break;
            tc_fence_after_sync();
            issue_qk<D>(tS, base + L::kK, ring(nxt));
            mma_commit(bar(L::S_FULL));
          }
          ok = mbar_wait_spin(bar(L::DS_READY), t & 1, wc, kRoleMma);
          if (!ok) break;
          tc_fence_after_sync();
          issue_pv<D>(tdK, tdP, ring(cur), i > q0);            // dK += dS^T Q
          mma_commit(bar(L::Q_EMPTY + cur % L::kStages));
          if (i + 1 < p.tiles) {
            issue_qk<D>(tdP, base + L::kV, ring(nxt) + L::kTile);
            mma_commit(bar(L::DP_FULL));
            if (i + 2 == p.tiles) mma_commit(bar(L::KV_EMPTY));  // last K, V read
          }
        }
        if (!ok) break;
        q_cons += p.tiles - q0;
        tcnt += p.tiles - q0;
        mma_commit(bar(L::ACC_FULL));
        ++uocc;
      }
      mma_commit(bar(L::DRAIN));
      mbar_wait_drain(bar(L::DRAIN), 0, wc);
    }
    __syncwarp();
  } else {
    // compute warpgroups: thread = key row r of the tile, query columns of
    // half hc
    const int wq = warp & 3;   // TMEM lane quarter
    const int hc = warp >> 2;  // 64-column half of the tile
    const int r = wq * 32 + lane;
    const uint32_t lb = static_cast<uint32_t>(wq * 32) << 16;
    int s_cnt = 0, uocc = 0, q_cons = 0;
    bool ok = true;
    for (int k = 0, u = unit_at<CAUSAL>(0); ok && u < p.num_units; u = unit_at<CAUSAL>(++k)) {
      int bh, kt, q0;
      dkv_unit<CAUSAL>(u, p.bh, p.tiles, bh, kt, q0);
      for (int i = q0; i < p.tiles; ++i) {
        const int st = q_cons % L::kStages;
        ++q_cons;
        // ---- P phase: P^T_i from S^T_i, kept in fp32 registers, and bf16
        // P^T written over the S^T columns already read
        ok = mbar_wait(bar(L::S_FULL), s_cnt & 1, wc, kRoleSoftmax);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after_sync();
        // the stage's lse / D vectors were written by TMA: acquire them on
        // the stage's own barrier (complete by now: the MMA waited on it)
        ok = mbar_wait(bar(L::Q_FULL + st), ((q_cons - 1) / L::kStages) & 1, wc,
                       kRoleSoftmax);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint32_t vec = base + L::kRing + st * L::kStage + 2 * L::kTile;
        // causal: on the diagonal tile query c < key r is in the key's past
        // of no query (P = 0); on the last tile queries >= N do not exist
        const bool diag = CAUSAL && (i == kt);
        const bool tail = (i == p.tiles - 1) && (p.n & (kBlockM - 1));
        const int qlimit = p.n - 1 - i * kBlockM;
        float pr[64];
        uint32_t sv[2][32];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) tmem_ld_32x32b_x32(tS + lb + (2 * hc + cc) * 32, sv[cc]);
        tmem_wait_ld(sv[0]);
        reg_fence(sv[1]);
        bwd_pair_sync(wq);  // both halves hold their S^T before P^T overwrites it
        const uint64_t c2 = f32x2(p.c_log2, p.c_log2);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * hc + cc;  // 32-column chunk of the tile
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            // -lse log2(e) of four query columns
            const float4 lv = ld_shared_f4(vec + (c * 32 + 4 * g) * 4);
            const uint64_t xa = fma_f32x2(f32x2(__uint_as_float(sv[cc][4 * g]),
                                                __uint_as_float(sv[cc][4 * g + 1])),
                                          c2, f32x2(lv.x, lv.y));
            const uint64_t xb = fma_f32x2(f32x2(__uint_as_float(sv[cc][4 * g + 2]),
                                                __uint_as_float(sv[cc][4 * g + 3])),
                                          c2, f32x2(lv.z, lv.w));
            bwd_exp2_pair<D>(2 * g, xa, pr[cc * 32 + 4 * g], pr[cc * 32 + 4 * g + 1]);
            bwd_exp2_pair<D>(2 * g + 1, xb, pr[cc * 32 + 4 * g + 2], pr[cc * 32 + 4 * g + 3]);
          }
          if (diag || tail) {  // the diagonal and the ragged last Q tile only
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int qc = c * 32 + e;  // query column in the tile
              if ((diag && qc < r) || (tail && qc > qlimit)) pr[cc * 32 + e] = 0.f;
            }
          }
          uint32_t ppk[16];
#pragma unroll
          for (int g = 0; g < 16; ++g)
            ppk[g] = pack_bf16x2(pr[cc * 32 + 2 * g], pr[cc * 32 + 2 * g + 1]);
          tmem_st_32x32b_x16(tS + lb + c * 16, ppk);   // P^T over S^T
        }
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::P_READY));
        // ---- dS phase: dS^T_i = P^T_i (dP^T_i - D) written over dP^T_i
        ok = mbar_wait(bar(L::DP_FULL), s_cnt & 1, wc, kRoleSoftmax);
        ++s_cnt;
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after_sync();
        uint32_t dv[2][32];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) tmem_ld_32x32b_x32(tdP + lb + (2 * hc + cc) * 32, dv[cc]);
        tmem_wait_ld(dv[0]);
        reg_fence(dv[1]);
        bwd_pair_sync(wq);  // both halves hold their dP^T before dS^T overwrites it
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * hc + cc;
          uint32_t dpk[16];
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const float4 dd = ld_shared_f4(vec + 512 + (c * 32 + 4 * g) * 4);  // -D
            const int q4 = cc * 32 + 4 * g;  // index into pr
            const uint64_t ta = add_f32x2(f32x2(__uint_as_float(dv[cc][4 * g]),
                                                __uint_as_float(dv[cc][4 * g + 1])),
                                          f32x2(dd.x, dd.y));
            const uint64_t tb = add_f32x2(f32x2(__uint_as_float(dv[cc][4 * g + 2]),
                                                __uint_as_float(dv[cc][4 * g + 3])),
                                          f32x2(dd.z, dd.w));
            float d0, d1, d2, d3;
            f32x2_split(mul_f32x2(f32x2(pr[q4], pr[q4 + 1]), ta), d0, d1);
            f32x2_split(mul_f32x2(f32x2(pr[q4 + 2], pr[q4 + 3]), tb), d2, d3);
            dpk[2 * g] = pack_bf16x2(d0, d1);
            dpk[2 * g + 1] = pack_bf16x2(d2, d3);
          }
          tmem_st_32x32b_x16(tdP + lb + c * 16, dpk);  // dS^T over dP^T
        }
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::DS_READY));
      }
      if (!ok) break;
      ok = mbar_wait(bar(L::ACC_FULL), uocc & 1, wc, kRoleEpilogue);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++uocc;
      tc_fence_after_sync();
      const int key = kt * kBlockN + r;
      const bool row_ok = key < p.n;
      const int64_t grow = static_cast<int64_t>(bh) * p.n + key;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = which ? tdK : tdV;
        const float mul = which ? p.scale : 1.f;
        uint4 *out = reinterpret_cast<uint4 *>((which ? p.dk : p.dv) + grow * D);
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
          const int c = hc * (D / 64) + cc;  // this half's 32-column chunks
          uint32_t o[32];
          tmem_ld_32x32b_x32(src + lb + c * 32, o);
          tmem_wait_ld(o);
          uint32_t h[16];
#pragma unroll
          for (int i2 = 0; i2 < 16; ++i2)
            h[i2] = pack_bf16x2(__uint_as_float(o[2 * i2]) * mul,
                                __uint_as_float(o[2 * i2 + 1]) * mul);
          if (row_ok) {
#pragma unroll
            for (int i2 = 0; i2 < 4; ++i2)
              out[c * 4 + i2] = make_uint4(h[4 * i2], h[4 * i2 + 1],
                                           h[4 * i2 + 2], h[4 * i2 + 3]);
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::ACC_EMPTY));
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn_b200
