// attn_decode_kernel.cuh -- split-KV decode attention for B200 (sm_100a).
//
// Source: the briefgpt.xyz summary page of FlashAttention-2 (arXiv
// 2307.08691), entry "LeanAttention": the decode phase of long contexts is
// computed in parallel over the key/value sequence.  The result is exact
// attention for Nq <= 16 new queries (the last Nq positions) against Nk keys:
// with the causal mask query i sees keys 0 .. Nk - Nq + i.
//
// Decode is a matrix-vector product per (batch, head): every key and value
// byte is used for a handful of queries, so the bound is HBM bandwidth, not
// the tensor cores.  The kernel therefore streams K/V through shared memory
// with bulk asynchronous copies and does the arithmetic on the CUDA cores:
//   * stream-K split: the B*H*ceil(Nk/64) key tiles of all heads are one
//     sequence; CTA c takes tiles [c T, (c+1) T) -- an equal share, which may
//     cross heads -- so every SM streams the same number of bytes whatever
//     B*H is;
//   * per CTA: one producer warp (one elected lane) fills a ring of K/V
//     stages (cp.async.bulk, one copy per 64-key K or V tile, completion on
//     an mbarrier); eight compute warps, per tile:
//       1. scores s[q][key] = (q . k) * scale * log2(e): four lanes per key,
//          each a quarter of the dimensions, reduced by two shuffles;
//       2. online softmax, one warp per query: tile max, running max m,
//          p = 2^(s - m), running sum l, rescale factor alpha;
//       3. O[q] = alpha O[q] + sum_key p v_key: one thread per (query group,
//          pair of dimensions);
//   * merge: a CTA that finished part of a head writes the part's (O_s,
//     lse_s); the CTA that completes the head's last part (an atomic counter
//     after a memory fence) combines them exactly,
//     lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s.  No CTA
//     waits for another; a head covered by one CTA is written directly.
// Waits on the ring are bounded like the forward's; a timeout sets the
// device status word and every compute warp leaves together.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <math_constants.h>

#include "attn_fwd_kernel.cuh"

namespace attn_b200 {

constexpr int kDecTileKeys = 64;
constexpr int kDecMaxQ = 16;           // queries per (batch, head)
constexpr int kDecComputeWarps = 8;
constexpr int kDecComputeThreads = kDecComputeWarps * 32;
constexpr int kDecThreads = kDecComputeThreads + 32;  // + producer warp
constexpr int kDecMaxCtas = 1024;      // bound on the grid (workspace sizing)

template <int D>
struct DecSmem {
  static constexpr uint32_t kTileBytes = kDecTileKeys * D * 2;  // K or V tile
  static constexpr int kStages = (D == 128) ? 3 : 6;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kStages * kTileBytes;
  static constexpr uint32_t kQ = kV + kStages * kTileBytes;       // fp32 [16][D]
  // scores, then probabilities, of the current tile: fp32 [16][64].  One
  // buffer suffices: the barrier that opens a tile is reached only after
  // every thread finished the previous tile's P.V step.
  static constexpr uint32_t kS = kQ + kDecMaxQ * D * 4;
  static constexpr uint32_t kAlpha = kS + kDecMaxQ * kDecTileKeys * 4;  // [16]
  static constexpr uint32_t kStat = kAlpha + kDecMaxQ * 4;        // m, l [16][2]
  static constexpr uint32_t kBars = kStat + kDecMaxQ * 8;
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
  int ntiles;          // key tiles per head
  int total;           // bh * ntiles
  int per_cta;         // T: tiles per CTA
  int causal;
  float c_log2;        // scale * log2(e)
  unsigned long long timeout_ns;
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
  for (int g = g0; g < g1; ++g) {
    const int h = g / p.ntiles;
    const int j = g - h * p.ntiles;
    const int st = issued % L::kStages;
    if (!mbar_wait(bar(L::EMPTY + st), ((issued / L::kStages) & 1) ^ 1, wc,
                   kRoleProducer))
      break;
    const int rows = min(kDecTileKeys, p.nk - j * kDecTileKeys);
    const uint32_t bytes = static_cast<uint32_t>(rows) * D * 2;
    mbar_arrive_expect_tx(bar(L::FULL + st), 2 * bytes);
    const int64_t off = (static_cast<int64_t>(h) * p.nk + j * kDecTileKeys) * D;
    bulk_g2s(base + L::kK + st * L::kTileBytes, p.k + off, bytes, bar(L::FULL + st));
    bulk_g2s(base + L::kV + st * L::kTileBytes, p.v + off, bytes, bar(L::FULL + st));
    ++issued;
  }
  if (*wc.abort) {
    // every copy issued must land before the CTA may exit
    for (int st = 0; st < L::kStages; ++st)
      if (issued > st) {
        const int last = st + ((issued - 1 - st) / L::kStages) * L::kStages;
        mbar_wait_drain(bar(L::FULL + st), (last / L::kStages) & 1, wc);
      }
  }
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------------------ compute

// One head's part: write it (whole head in this CTA) or record it and, if it
// is the last part to finish, merge all of the head's parts.
template <int D>
__device__ __forceinline__ void dec_finish_head(uint8_t *smem, const DecodeParams &p,
                                                int h, int tid,
                                                const float (&acc)[kDecMaxQ / (kDecComputeThreads / (D / 2))][2]) {
  using L = DecSmem<D>;
  constexpr int kPairs = D / 2;
  constexpr int kGroups = kDecComputeThreads / kPairs;
  constexpr int kQPer = kDecMaxQ / kGroups;
  const float *stat = reinterpret_cast<const float *>(smem + L::kStat);
  volatile int *last_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
  const int pair = tid % kPairs, grp = tid / kPairs;
  const int first = dec_first_cta(h, p), last = dec_last_cta(h, p);
  const int64_t row0 = static_cast<int64_t>(h) * p.nq;
  if (first == last) {
#pragma unroll
    for (int i = 0; i < kQPer; ++i) {
      const int q = grp + i * kGroups;
      if (q >= p.nq) continue;
      const float m = stat[2 * q], l = stat[2 * q + 1];
      const float inv = __frcp_rn(l);
      reinterpret_cast<uint32_t *>(p.o + (row0 + q) * D)[pair] =
          pack_bf16x2(acc[i][0] * inv, acc[i][1] * inv);
      if (pair == 0) p.lse[row0 + q] = (m + lg2_approx(l)) * kLn2;
    }
    return;
  }
  const int slot = h + static_cast<int>(blockIdx.x);
#pragma unroll
  for (int i = 0; i < kQPer; ++i) {
    const int q = grp + i * kGroups;
    if (q >= p.nq) continue;
    const float m = stat[2 * q], l = stat[2 * q + 1];
    const bool any = l > 0.f;  // a part may see no key of a causal row
    const float inv = any ? __frcp_rn(l) : 0.f;
    float2 *dst = reinterpret_cast<float2 *>(p.part_o + (static_cast<int64_t>(slot) * p.nq + q) * D);
    dst[pair] = make_float2(acc[i][0] * inv, acc[i][1] * inv);
    if (pair == 0)
      p.part_lse[static_cast<int64_t>(slot) * p.nq + q] =
          any ? (m + lg2_approx(l)) * kLn2 : -CUDART_INF_F;
  }
  __threadfence();  // the part is visible device-wide before it is counted
  dec_bar();
  if (tid == 0) *last_flag = (atomicAdd(p.counters + h, 1) == last - first);
  dec_bar();
  if (!*last_flag) return;
  __threadfence();
  const int nseg = last - first + 1;
#pragma unroll
  for (int i = 0; i < kQPer; ++i) {
    const int q = grp + i * kGroups;
    if (q >= p.nq) continue;
    float M = -CUDART_INF_F;
    for (int s = 0; s < nseg; ++s)
      M = fmaxf(M, __ldcg(p.part_lse + static_cast<int64_t>(h + first + s) * p.nq + q));
    float sum = 0.f, o0 = 0.f, o1 = 0.f;
    for (int s = 0; s < nseg; ++s) {
      const int64_t r = static_cast<int64_t>(h + first + s) * p.nq + q;
      const float ls = __ldcg(p.part_lse + r);
      const float w = (ls == -CUDART_INF_F) ? 0.f : ex2_approx((ls - M) * 1.4426950408889634f);
      const float2 po = __ldcg(reinterpret_cast<const float2 *>(p.part_o + r * D) + pair);
      sum += w;
      o0 = fmaf(w, po.x, o0);
      o1 = fmaf(w, po.y, o1);
    }
    const float inv = __frcp_rn(sum);
    reinterpret_cast<uint32_t *>(p.o + (row0 + q) * D)[pair] = pack_bf16x2(o0 * inv, o1 * inv);
    if (pair == 0) p.lse[row0 + q] = M + lg2_approx(sum) * kLn2;
  }
  if (tid == 0) p.counters[h] = 0;  // ready for the next launch
}

template <int D>
__device__ __forceinline__ void dec_compute(uint32_t base, uint8_t *smem,
                                            const DecodeParams &p, const WaitCtx &wc,
                                            int g0, int g1, int warp, int lane) {
  using L = DecSmem<D>;
  constexpr int kPairs = D / 2;
  constexpr int kGroups = kDecComputeThreads / kPairs;  // 4 (d = 128) or 8
  constexpr int kQPer = kDecMaxQ / kGroups;             // queries per thread
  constexpr int kChunks = D / 8;                        // 16-byte chunks per row
  auto bar = [&](int i) { return base + L::kBars + 8u * i; };
  const int tid = warp * 32 + lane;
  const int pair = tid % kPairs, grp = tid / kPairs;
  float *qf = reinterpret_cast<float *>(smem + L::kQ);
  float *sbuf = reinterpret_cast<float *>(smem + L::kS);
  float *alpha_s = reinterpret_cast<float *>(smem + L::kAlpha);
  float *stat = reinterpret_cast<float *>(smem + L::kStat);
  int cons = 0;
  bool ok = true;
  for (int g = g0; ok && g < g1;) {
    const int h = g / p.ntiles;
    const int gend = min(g1, (h + 1) * p.ntiles);
    // this head's queries, scaled into log2 units
    dec_bar();  // the previous part's readers of qf / stat are done
    const uint16_t *qsrc = p.q + static_cast<int64_t>(h) * p.nq * D;
    for (int i = tid; i < p.nq * D; i += kDecComputeThreads)
      qf[i] = __uint_as_float(static_cast<uint32_t>(qsrc[i]) << 16) * p.c_log2;
    float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_run[2] = {0.f, 0.f};
    float acc[kQPer][2];
#pragma unroll
    for (int i = 0; i < kQPer; ++i) acc[i][0] = acc[i][1] = 0.f;
    dec_bar();
    for (int gg = g; gg < gend; ++gg, ++cons) {
      const int j = gg - h * p.ntiles;
      const int st = cons % L::kStages;
      const bool got = mbar_wait(bar(L::FULL + st), (cons / L::kStages) & 1, wc,
                                 kRoleSoftmax);
      ok = dec_bar_and(got);  // every compute thread takes the same branch
      if (!ok) break;
      const int rows = min(kDecTileKeys, p.nk - j * kDecTileKeys);
      const int kb = j * kDecTileKeys;
      const uint8_t *kt = smem + L::kK + st * L::kTileBytes;
      const uint8_t *vt = smem + L::kV + st * L::kTileBytes;
      float *S = sbuf;
      float *al = alpha_s;

      // 1. scores: lane quarter q4 of key `key` takes chunks q4, q4 + 4, ...
      {
        const int key = warp * 8 + (lane >> 2), q4 = lane & 3;
        float part[kDecMaxQ];
#pragma unroll
        for (int q = 0; q < kDecMaxQ; ++q) part[q] = 0.f;
        if (key < rows) {
#pragma unroll
          for (int c = 0; c < kChunks / 4; ++c) {
            const int ch = q4 + 4 * c;
            const uint4 raw = *reinterpret_cast<const uint4 *>(kt + key * D * 2 + ch * 16);
            const float kf[8] = {bf16lo(raw.x), bf16hi(raw.x), bf16lo(raw.y), bf16hi(raw.y),
                                 bf16lo(raw.z), bf16hi(raw.z), bf16lo(raw.w), bf16hi(raw.w)};
#pragma unroll
            for (int q = 0; q < kDecMaxQ; ++q) {
              if (q >= p.nq) break;
              const float4 a = *reinterpret_cast<const float4 *>(qf + q * D + ch * 8);
              const float4 b = *reinterpret_cast<const float4 *>(qf + q * D + ch * 8 + 4);
              part[q] = fmaf(a.x, kf[0], fmaf(a.y, kf[1], fmaf(a.z, kf[2], fmaf(a.w, kf[3],
                        fmaf(b.x, kf[4], fmaf(b.y, kf[5], fmaf(b.z, kf[6], fmaf(b.w, kf[7], part[q]))))))));
            }
          }
        }
#pragma unroll
        for (int q = 0; q < kDecMaxQ; ++q) {
          if (q >= p.nq) break;  // uniform across the warp
          part[q] += __shfl_xor_sync(0xffffffffu, part[q], 1);
          part[q] += __shfl_xor_sync(0xffffffffu, part[q], 2);
          if ((q & 3) == q4) {
            const bool vis = key < rows && (!p.causal || kb + key <= p.nk - p.nq + q);
            S[q * kDecTileKeys + key] = vis ? part[q] : -CUDART_INF_F;
          }
        }
      }
      dec_bar();
      // 2. online softmax: warp w owns queries w and w + 8
#pragma unroll
      for (int qi = 0; qi < 2; ++qi) {
        const int q = warp + 8 * qi;
        if (q >= p.nq) continue;  // uniform across the warp
        const float s0 = S[q * kDecTileKeys + lane], s1 = S[q * kDecTileKeys + lane + 32];
        float tm = fmaxf(s0, s1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, off));
        const float mn = fmaxf(m_run[qi], tm);
        float a = 1.f, p0 = 0.f, p1 = 0.f;
        if (mn != -CUDART_INF_F) {  // some key of the row visible so far
          a = ex2_approx(m_run[qi] - mn);  // 0 while nothing was visible
          p0 = ex2_approx(s0 - mn);
          p1 = ex2_approx(s1 - mn);
        }
        float ps = p0 + p1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l_run[qi] = fmaf(l_run[qi], a, ps);
        m_run[qi] = mn;
        S[q * kDecTileKeys + lane] = p0;
        S[q * kDecTileKeys + lane + 32] = p1;
        if (lane == 0) al[q] = a;
      }
      dec_bar();
      // 3. O[q] = alpha O[q] + sum_key p[q][key] v[key] for this thread's
      //    pair of dimensions and queries grp, grp + kGroups, ...
#pragma unroll
      for (int i = 0; i < kQPer; ++i) {
        const int q = grp + i * kGroups;
        if (q < p.nq) {
          const float a = al[q];
          acc[i][0] *= a;
          acc[i][1] *= a;
        }
      }
      if (grp < p.nq) {
#pragma unroll 8
        for (int key = 0; key < rows; ++key) {
          const uint32_t v2 = *reinterpret_cast<const uint32_t *>(vt + key * D * 2 + pair * 4);
          const float v0 = bf16lo(v2), v1 = bf16hi(v2);
#pragma unroll
          for (int i = 0; i < kQPer; ++i) {
            const int q = grp + i * kGroups;
            if (q < p.nq) {
              const float pk = S[q * kDecTileKeys + key];
              acc[i][0] = fmaf(pk, v0, acc[i][0]);
              acc[i][1] = fmaf(pk, v1, acc[i][1]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::EMPTY + st));  // K and V of this stage read
    }
    if (!ok) break;
    // the part's statistics, from the softmax warps to every thread
    if (lane == 0) {
#pragma unroll
      for (int qi = 0; qi < 2; ++qi) {
        const int q = warp + 8 * qi;
        if (q < p.nq) {
          stat[2 * q] = m_run[qi];
          stat[2 * q + 1] = l_run[qi];
        }
      }
    }
    dec_bar();
    dec_finish_head<D>(smem, p, h, tid, acc);
    g = gend;
  }
}

// ------------------------------------------------------------------ kernel

template <int D>
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
    dec_compute<D>(base, dsmem, p, wc, g0, g1, warp, lane);
  }
  __syncthreads();
}

}  // namespace attn_b200
