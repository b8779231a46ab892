// attn_decode_kernel.cuh -- split-KV decode attention for B200 (sm_100a).
//
// Source: the briefgpt.xyz summary page of FlashAttention-2 (arXiv
// 2307.08691), entry "LeanAttention": the decode phase of long contexts is
// computed in parallel over the key/value sequence.  The result is exact
// attention for Nq <= 16 new queries (the last Nq positions) against Nk keys:
// with the causal mask query i sees keys 0 .. Nk - Nq + i.
//
// attn_decode runs this kernel when attn_set_decode_kernel(1) selects it; by
// default the tensor-core kernel (attn_decode_mma_kernel.cuh) serves, which
// streamed K/V faster at every Nq and head size measured.  This one keeps P
// in fp32 instead of rounding it to bf16 for a P.V product.
//
// Decode is a matrix-vector product per (batch, head): every key and value
// byte is used for a handful of queries, so the bound is HBM bandwidth, not
// the tensor cores.  One launch serves up to 4 queries per head (their
// state stays in registers with two CTAs per SM); more queries are served in
// groups of 4 by successive launches, each stopping at the last key its
// queries can see.  The kernel therefore streams K/V through shared memory
// with bulk asynchronous copies and does the arithmetic on the CUDA cores:
//   * stream-K split: the B*H*ceil(Nk/K) key tiles of all heads are one
//     sequence (K = 64 keys at d = 128, 128 at d = 64: 16 KB of K either
//     way); CTA c takes tiles [c T, (c+1) T) -- an equal share, which may
//     cross heads -- so every SM streams the same number of bytes whatever
//     B*H is;
//   * per CTA: one producer warp (one elected lane) fills a 3-stage ring of
//     K/V tiles (cp.async.bulk, one copy per K or V tile, completion on an
//     mbarrier); eight compute warps each own a slice of every tile (8 or 16
//     keys) and run their own online softmax over it -- no communication
//     between warps inside a tile:
//       1. scores s[q][key] = (q . k) * scale * log2(e): four lanes per key,
//          each a quarter of the dimensions, reduced by two shuffles;
//       2. p = 2^(s - m) against the warp's running reference m, which
//          moves (with a rescale of l and O) only when a score exceeds it by
//          more than 2^8 -- a warp vote per query, the maximum reduction
//          only when the vote says so; each lane keeps its own part of l;
//       3. O[q] += sum over the slice's keys of p v_key, each lane D/32
//          dimensions (p passed through the warp's slice of shared memory);
//     at the end of a head's share the eight warps' (m, l, O) are combined
//     through shared memory (O in rounds of a few queries);
//   * merge: a CTA that finished part of a head writes the part's (O_s,
//     lse_s); the CTA that completes the head's last part (an atomic counter
//     after a memory fence) combines them exactly,
//     lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s.  No CTA
//     waits for another; a head covered by one CTA is written directly.
// Waits on the ring are bounded like the forward's; a timeout sets the
// device status word, and the compute warps agree at the end of the share
// (a barrier with an AND reduction) to leave without writing.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <math_constants.h>

#include "attn_fwd_kernel.cuh"

namespace attn_b200 {

constexpr int kDecMaxQ = 4;            // queries per (batch, head) and launch
constexpr int kDecComputeWarps = 8;
constexpr int kDecComputeThreads = kDecComputeWarps * 32;
constexpr int kDecThreads = kDecComputeThreads + 32;  // + producer warp
constexpr int kDecMaxCtas = 1024;      // bound on the grid (workspace sizing)
constexpr float kDecLazy = 8.f;        // log2 units: p <= 2^8

template <int D>
struct DecSmem {
  // keys per tile: 16 KB of K (and of V) either way; at d = 64 each lane
  // group takes two keys of its warp's slice, so that every query value it
  // reads from shared memory serves two keys
  static constexpr int kTileKeys = (D == 64) ? 128 : 64;
  static constexpr int kKeysPerLane = kTileKeys / (8 * kDecComputeWarps);  // R
  static constexpr int kSlice = 8 * kKeysPerLane;  // keys of a warp per tile
  static constexpr uint32_t kTileBytes = kTileKeys * D * 2;  // K or V tile
  static constexpr int kStages = 3;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kStages * kTileBytes;
  // the head's queries (fp32 [4][D], pre-scaled; within a query the first
  // halves of all 8-dimension chunks, then the second halves) while a share
  // runs; at its end the same bytes hold the warps' O for a round of kRedQ
  // queries
  static constexpr uint32_t kRedBytes = 8 * 1024;
  static constexpr int kRedQ = kRedBytes / (kDecComputeWarps * D * 4);  // 2 or 4
  static_assert(kDecMaxQ * D * 4 <= kRedBytes, "queries fit the shared region");
  static constexpr uint32_t kQ = kV + kStages * kTileBytes;
  // each warp's probabilities of its current slice, [kSlice keys][4 queries]
  static constexpr uint32_t kP = kQ + kRedBytes;
  static constexpr uint32_t kStat = kP + kDecComputeWarps * kSlice * kDecMaxQ * 4;  // m, l [8][4][2]
  static constexpr uint32_t kBars = kStat + kDecComputeWarps * kDecMaxQ * 8;
  static constexpr int FULL = 0, EMPTY = kStages, NUM_BARS = 2 * kStages;
  static constexpr uint32_t kMisc = kBars + NUM_BARS * 8;         // abort flag, last flag
  static constexpr uint32_t kBytes = kMisc + 16;
  // two CTAs per SM (228 KB, of which 1 KB per CTA is reserved)
  static_assert(2 * (kBytes + 1024) <= 228 * 1024, "two CTAs per SM");
};

struct DecodeParams {
  const uint16_t *q;   // [BH, Nq, D]
  const uint16_t *k;   // [BH, Nk, D]
  const uint16_t *v;   // [BH, Nk, D]
  uint16_t *o;         // [BH, Nq, D]
  float *lse;          // [BH, Nq]
  float *part_o;       // [slots, Nq, D] partial outputs (normalised)
  float *part_lse;     // [slots, Nq]
  int *counters;       // [BH] parts finished per head (zero at launch)
  uint32_t *status;
  int bh, nq, nk;
  int qstride;         // rows per head of q, o, lse (nq unless a group of them)
  int kstride;         // rows per head of k, v (nk unless the keys are cut short)
  int ntiles;          // key tiles per head
  int total;           // bh * ntiles
  int per_cta;         // T: tiles per CTA
  int causal;
  float c_log2;        // scale * log2(e)
  unsigned long long timeout_ns;
  uint32_t debug_flags;  // bit 1: CTA 0's producer skips its first tile
};

// All 256 compute threads meet at named barrier 1 (the producer warp never
// joins it); the result is the AND of their predicates.
__device__ __forceinline__ bool dec_bar_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "n"(kDecComputeThreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void dec_bar() {
  asm volatile("barrier.cta.sync 1, %0;" ::"n"(kDecComputeThreads) : "memory");
}

// Bulk copy of `bytes` (a multiple of 16) from global to shared memory,
// completing on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src,
                                         uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// CTA c's tiles and the parts of heads they form.
__device__ __forceinline__ int dec_first_cta(int h, const DecodeParams &p) {
  return static_cast<int>((static_cast<int64_t>(h) * p.ntiles) / p.per_cta);
}
__device__ __forceinline__ int dec_last_cta(int h, const DecodeParams &p) {
  return static_cast<int>((static_cast<int64_t>(h + 1) * p.ntiles - 1) / p.per_cta);
}

// ------------------------------------------------------------------ producer

// One elected lane: K and V tiles of the CTA's share, in order, into the
// ring (one bulk copy each; the last tile of a head may be short).
template <int D>
__device__ __forceinline__ void dec_producer(uint32_t base, const DecodeParams &p,
                                             const WaitCtx &wc, int g0, int g1) {
  using L = DecSmem<D>;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };
  int issued = 0;
  // injected fault: the first tile's copies are never issued, so the compute
  // warps' wait for it must run out (its stage is then not drained)
  const int skipped = ((p.debug_flags & 2u) && blockIdx.x == 0) ? 0 : -1;
  for (int g = g0; g < g1; ++g) {
    const int h = g / p.ntiles;
    const int j = g - h * p.ntiles;
    const int st = issued % L::kStages;
    if (!mbar_wait(bar(L::EMPTY + st), ((issued / L::kStages) & 1) ^ 1, wc,
                   kRoleProducer))
      break;
    if (issued == skipped) {
      ++issued;
      continue;
    }
    const int rows = min(L::kTileKeys, p.nk - j * L::kTileKeys);
    const uint32_t bytes = static_cast<uint32_t>(rows) * D * 2;
    mbar_arrive_expect_tx(bar(L::FULL + st), 2 * bytes);
    const int64_t off = (static_cast<int64_t>(h) * p.kstride + j * L::kTileKeys) * D;
    bulk_g2s(base + L::kK + st * L::kTileBytes, p.k + off, bytes, bar(L::FULL + st));
    bulk_g2s(base + L::kV + st * L::kTileBytes, p.v + off, bytes, bar(L::FULL + st));
    ++issued;
  }
  if (*wc.abort) {
    // every copy issued must land before the CTA may exit
    for (int st = 0; st < L::kStages; ++st)
      if (issued > st) {
        const int last = st + ((issued - 1 - st) / L::kStages) * L::kStages;
        if (last == skipped) continue;  // nothing was copied for it
        mbar_wait_drain(bar(L::FULL + st), (last / L::kStages) & 1, wc);
      }
  }
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------------------ compute

// One CTA's share of key tiles, head part by head part.  QMAX (the 4
// queries of a launch) bounds the queries so that a lane's per-query state
// stays in registers.
//
// Lane (kl, q4) = (lane / 4, lane % 4) of warp w scores keys
// w * kSlice + kl + 8 r (r < R), a quarter of the dimensions each: the
// 16-byte chunks q4, q4 + 4, ... of the row, visited in the order
// c ^ (kl & 1) so that the two keys read by one quarter-warp fall in
// different banks (rows are 128 or 256 bytes, so the same chunk of two rows
// shares banks).  The queries' matching halves of those chunks lie 16 bytes
// apart in the query layout, so their reads are conflict-free too.
template <int D, int QMAX>
__device__ __forceinline__ void dec_compute(uint32_t base, uint8_t *smem,
                                            const DecodeParams &p, const WaitCtx &wc,
                                            int g0, int g1, int warp, int lane) {
  using L = DecSmem<D>;
  static_assert(QMAX == kDecMaxQ, "one query group per launch");
  constexpr int E = D / 32;        // output dimensions per lane
  constexpr int kChunks = D / 8;   // 16-byte chunks per row
  constexpr int R = L::kKeysPerLane;
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };
  const int tid = warp * 32 + lane;
  const int kl = lane >> 2, q4 = lane & 3;  // key of the warp's slice, quarter
  float *qf = reinterpret_cast<float *>(smem + L::kQ);
  float *red = qf;  // the same bytes once the share's last tile is done
  float *stat = reinterpret_cast<float *>(smem + L::kStat);
  float *pw = reinterpret_cast<float *>(smem + L::kP) + warp * L::kSlice * kDecMaxQ;
  volatile int *last_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
  int cons = 0;
  for (int g = g0; g < g1;) {
    const int h = g / p.ntiles;
    const int gend = min(g1, (h + 1) * p.ntiles);
    dec_bar();  // the previous part's readers of the shared region are done
    const uint16_t *qsrc = p.q + static_cast<int64_t>(h) * p.qstride * D;
    for (int i = tid; i < p.nq * D; i += kDecComputeThreads) {
      // dimension x of query q: chunk x / 8, half (x / 4) & 1, element x & 3
      const int q = i / D, x = i - q * D;
      const int at = q * D + ((x >> 2) & 1) * (D / 2) + (x >> 3) * 4 + (x & 3);
      qf[at] = __uint_as_float(static_cast<uint32_t>(qsrc[i]) << 16) * p.c_log2;
    }
    dec_bar();
    float m_w[QMAX], l_w[QMAX], acc[QMAX][E];
#pragma unroll
    for (int q = 0; q < QMAX; ++q) {
      m_w[q] = -CUDART_INF_F;
      l_w[q] = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[q][e] = 0.f;
    }
    bool ok = true;
    for (int gg = g; gg < gend; ++gg, ++cons) {
      const int j = gg - h * p.ntiles;
      const int st = cons % L::kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::FULL + st), (cons / L::kStages) & 1,
                                             wc, kRoleSoftmax));
      if (!ok) break;
      const int rows = min(L::kTileKeys, p.nk - j * L::kTileKeys);
      const uint8_t *kt = smem + L::kK + st * L::kTileBytes;
      const uint8_t *vt = smem + L::kV + st * L::kTileBytes;
      int key[R];
      bool kvalid[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        key[r] = warp * L::kSlice + kl + 8 * r;  // this lane's keys within the tile
        kvalid[r] = key[r] < rows;
      }
      // 1. scores of the slice's keys
      float s[R][QMAX];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int q = 0; q < QMAX; ++q) s[r][q] = 0.f;
#pragma unroll
      for (int c = 0; c < kChunks / 4; ++c) {
        const int ch = q4 + 4 * (c ^ (kl & 1));
        float kf[R][8];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint4 raw = kvalid[r]
              ? *reinterpret_cast<const uint4 *>(kt + key[r] * D * 2 + ch * 16)
              : make_uint4(0u, 0u, 0u, 0u);
          kf[r][0] = bf16lo(raw.x); kf[r][1] = bf16hi(raw.x);
          kf[r][2] = bf16lo(raw.y); kf[r][3] = bf16hi(raw.y);
          kf[r][4] = bf16lo(raw.z); kf[r][5] = bf16hi(raw.z);
          kf[r][6] = bf16lo(raw.w); kf[r][7] = bf16hi(raw.w);
        }
#pragma unroll
        for (int q = 0; q < QMAX; ++q) {
          if (q >= p.nq) break;
          const float4 a = *reinterpret_cast<const float4 *>(qf + q * D + ch * 4);
          const float4 b = *reinterpret_cast<const float4 *>(qf + q * D + D / 2 + ch * 4);
#pragma unroll
          for (int r = 0; r < R; ++r)
            s[r][q] = fmaf(a.x, kf[r][0], fmaf(a.y, kf[r][1], fmaf(a.z, kf[r][2],
                      fmaf(a.w, kf[r][3], fmaf(b.x, kf[r][4], fmaf(b.y, kf[r][5],
                      fmaf(b.z, kf[r][6], fmaf(b.w, kf[r][7], s[r][q]))))))));
        }
      }
      // 2. the warp's online softmax over its slice (all lanes of a key
      //    hold its score; lanes 4k .. 4k+3 belong to key k)
#pragma unroll
      for (int q = 0; q < QMAX; ++q) {
        if (q >= p.nq) break;  // uniform across the warp
        float smax = -CUDART_INF_F;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          s[r][q] += __shfl_xor_sync(0xffffffffu, s[r][q], 1);
          s[r][q] += __shfl_xor_sync(0xffffffffu, s[r][q], 2);
          const int kabs = j * L::kTileKeys + key[r];
          if (!(kvalid[r] && (!p.causal || kabs <= p.nk - p.nq + q))) s[r][q] = -CUDART_INF_F;
          smax = fmaxf(smax, s[r][q]);
        }
        if (__any_sync(0xffffffffu, smax > m_w[q] + kDecLazy)) {
          float tm = smax;
          tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
          tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
          tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
          const float mn = fmaxf(m_w[q], tm);  // finite: some score beat m
          const float alpha = ex2_approx(m_w[q] - mn);  // 0 while m was -inf
          l_w[q] *= alpha;
#pragma unroll
          for (int e = 0; e < E; ++e) acc[q][e] *= alpha;
          m_w[q] = mn;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          // p <= 2^8; no visible key yet (m = -inf) means p = 0
          const float pk = (m_w[q] == -CUDART_INF_F) ? 0.f : ex2_approx(s[r][q] - m_w[q]);
          l_w[q] += pk;  // each of the key's four lanes adds it: l = sum / 4
          if (q == q4) pw[(kl + 8 * r) * kDecMaxQ + q] = pk;
        }
      }
      __syncwarp();
      // 3. O += p v over the slice's keys, E dimensions per lane
#pragma unroll
      for (int k = 0; k < L::kSlice; ++k) {
        const int krow = warp * L::kSlice + k;
        if (krow >= rows) break;  // uniform across the warp
        float vv[E];
        if constexpr (E == 4) {
          const uint2 w2 = *reinterpret_cast<const uint2 *>(vt + krow * D * 2 + lane * 8);
          vv[0] = bf16lo(w2.x); vv[1] = bf16hi(w2.x); vv[2] = bf16lo(w2.y); vv[3] = bf16hi(w2.y);
        } else {
          const uint32_t w1 = *reinterpret_cast<const uint32_t *>(vt + krow * D * 2 + lane * 4);
          vv[0] = bf16lo(w1); vv[1] = bf16hi(w1);
        }
        const float4 pq = *reinterpret_cast<const float4 *>(pw + k * kDecMaxQ);
        const float pv4[4] = {pq.x, pq.y, pq.z, pq.w};
#pragma unroll
        for (int q = 0; q < QMAX; ++q) {
          if (q >= p.nq) break;
#pragma unroll
          for (int e = 0; e < E; ++e) acc[q][e] = fmaf(pv4[q], vv[e], acc[q][e]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::EMPTY + st));  // K and V of this stage read
    }
    if (!dec_bar_and(ok)) return;  // a wait ran out: every compute thread leaves
#pragma unroll
    for (int q = 0; q < QMAX; ++q) {
      if (q >= p.nq) break;
      float t = l_w[q];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
      l_w[q] = 0.25f * t;  // every key's p was added by its four lanes
    }

    // ---- the eight warps' (m, l, O) combined, then written (whole head) or
    // recorded as a part; O goes through the shared region kRedQ queries at
    // a time.
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < QMAX; ++q)
        if (q < p.nq) {
          stat[(warp * kDecMaxQ + q) * 2] = m_w[q];
          stat[(warp * kDecMaxQ + q) * 2 + 1] = l_w[q];
        }
    }
    const int first = dec_first_cta(h, p), last = dec_last_cta(h, p);
    const bool whole = first == last;
    const int slot = h + static_cast<int>(blockIdx.x);
    const int64_t row0 = static_cast<int64_t>(h) * p.qstride;
    for (int q0 = 0; q0 < p.nq; q0 += L::kRedQ) {
      dec_bar();  // earlier readers of the shared region are done
#pragma unroll
      for (int q = 0; q < QMAX; ++q)
        if (q >= q0 && q < q0 + L::kRedQ && q < p.nq) {
          float *dst = red + (warp * L::kRedQ + (q - q0)) * D + lane * E;
          if constexpr (E == 4)
            *reinterpret_cast<float4 *>(dst) = make_float4(acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
          else
            *reinterpret_cast<float2 *>(dst) = make_float2(acc[q][0], acc[q][1]);
        }
      dec_bar();
      const int nr = min(L::kRedQ, p.nq - q0);
      for (int item = tid; item < nr * (D / 2); item += kDecComputeThreads) {
        const int ql = item / (D / 2), pair = item - ql * (D / 2);
        const int q = q0 + ql;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int w = 0; w < kDecComputeWarps; ++w)
          M = fmaxf(M, stat[(w * kDecMaxQ + q) * 2]);
        float lsum = 0.f, o0 = 0.f, o1 = 0.f;
        if (M != -CUDART_INF_F) {
#pragma unroll
          for (int w = 0; w < kDecComputeWarps; ++w) {
            const float mw = stat[(w * kDecMaxQ + q) * 2];
            if (mw == -CUDART_INF_F) continue;
            const float f = ex2_approx(mw - M);
            lsum = fmaf(f, stat[(w * kDecMaxQ + q) * 2 + 1], lsum);
            const float2 r = *reinterpret_cast<const float2 *>(
                red + (w * L::kRedQ + ql) * D + 2 * pair);
            o0 = fmaf(f, r.x, o0);
            o1 = fmaf(f, r.y, o1);
          }
        }
        const bool any = lsum > 0.f;  // a part may see no key of a causal row
        const float inv = any ? __frcp_rn(lsum) : 0.f;
        const float lse2 = any ? M + lg2_approx(lsum) : -CUDART_INF_F;  // log2 units
        if (whole) {
          reinterpret_cast<uint32_t *>(p.o + (row0 + q) * D)[pair] =
              pack_bf16x2(o0 * inv, o1 * inv);
          if (pair == 0) p.lse[row0 + q] = lse2 * kLn2;
        } else {
          reinterpret_cast<float2 *>(p.part_o + (static_cast<int64_t>(slot) * p.nq + q) * D)[pair] =
              make_float2(o0 * inv, o1 * inv);
          if (pair == 0)
            p.part_lse[static_cast<int64_t>(slot) * p.nq + q] = any ? lse2 * kLn2 : -CUDART_INF_F;
        }
      }
    }
    if (!whole) {
      __threadfence();  // the part is visible device-wide before it is counted
      dec_bar();
      if (tid == 0) *last_flag = (atomicAdd(p.counters + h, 1) == last - first);
      dec_bar();
      if (*last_flag) {
        __threadfence();
        const int nseg = last - first + 1;
        for (int item = tid; item < p.nq * (D / 2); item += kDecComputeThreads) {
          const int q = item / (D / 2), pair = item - q * (D / 2);
          float M = -CUDART_INF_F;
          for (int sgi = 0; sgi < nseg; ++sgi)
            M = fmaxf(M, __ldcg(p.part_lse + static_cast<int64_t>(h + first + sgi) * p.nq + q));
          float sum = 0.f, o0 = 0.f, o1 = 0.f;
          for (int sgi = 0; sgi < nseg; ++sgi) {
            const int64_t r = static_cast<int64_t>(h + first + sgi) * p.nq + q;
            const float ls = __ldcg(p.part_lse + r);
            if (ls == -CUDART_INF_F) continue;
            const float wgt = ex2_approx((ls - M) * 1.4426950408889634f);
            const float2 po = __ldcg(reinterpret_cast<const float2 *>(p.part_o + r * D) + pair);
            sum += wgt;
            o0 = fmaf(wgt, po.x, o0);
            o1 = fmaf(wgt, po.y, o1);
          }
          const float inv = __frcp_rn(sum);
          reinterpret_cast<uint32_t *>(p.o + (row0 + q) * D)[pair] = pack_bf16x2(o0 * inv, o1 * inv);
          if (pair == 0) p.lse[row0 + q] = M + lg2_approx(sum) * kLn2;
        }
        if (tid == 0) p.counters[h] = 0;  // ready for the next launch
      }
    }
    g = gend;
  }
}

// ------------------------------------------------------------------ kernel

template <int D, int QMAX>
__global__ void __launch_bounds__(kDecThreads, 2)
    attn_decode_kernel(const DecodeParams p) {
  using L = DecSmem<D>;
  extern __shared__ __align__(128) uint8_t dsmem[];
  const uint32_t base = smem_u32(dsmem);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(dsmem + L::kMisc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(base + L::kBars + 8u * (L::FULL + s), 1);
      mbar_init(base + L::kBars + 8u * (L::EMPTY + s), kDecComputeWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtx wc{abort_flag, p.status, p.timeout_ns};
  const int g0 = blockIdx.x * p.per_cta;
  const int g1 = min(p.total, g0 + p.per_cta);
  if (warp == kDecComputeWarps) {
    if (lane == 0) dec_producer<D>(base, p, wc, g0, g1);
    __syncwarp();
  } else {
    dec_compute<D, QMAX>(base, dsmem, p, wc, g0, g1, warp, lane);
  }
  __syncthreads();
}

}  // namespace attn_b200
