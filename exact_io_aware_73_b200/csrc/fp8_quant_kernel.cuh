// fp8_quant_kernel.cuh -- incoherent processing and block quantization of
// Q, K, V to FP8 (E4M3) for the FP8 attention forward on B200 (sm_100a).
//
// Source cited as [MM]: the marketmaker.cc blog post (Indonesian edition)
// "Apakah Konteks Sehari Penuh Mengalahkan Konteks Sepuluh Menit? Perhatian
// Kilat dan Pertanyaan Panjang Urutan", section "FA3: Mekanika hopper",
// item 3: vectors are rotated at random before block quantization so that an
// outlier's magnitude is spread over all coordinates.
//
// The kernel is persistent (one CTA of 512 threads per SM walks the 128-row
// tiles); thread (row, q) of a tile owns coordinates [32 q, 32 q + 32) of
// one row and loads the next tile's share while it works on this one.  Per
// tile:
//   * rotation (Q and K only): each row x becomes x diag(s) H, with s the
//     random +-1 signs (a 128-bit mask, bit t set = negate coordinate t) and
//     H the unscaled d x d Sylvester Hadamard matrix (H H^T = d I), applied as
//     the fast Walsh-Hadamard butterfly in fp64.  Butterflies of span < 32
//     stay in the thread, the two wider ones pair the row's four lanes by
//     shuffle.  bf16 inputs make every partial
//     sum exact in fp64, so the butterfly's order cannot change the result;
//     the row is then rounded to fp32;
//   * block scale: the largest power of two 2^e with amax * 2^e <= 448 (the
//     largest finite E4M3 value), amax over the block; the stored
//     dequantization scale is 2^-e.  Blocks are the tile (Q, K) or the whole
//     head (V: a first pass stores each tile's amax, the second reduces them);
//   * codes: E4M3(x * 2^e), round to nearest even (the scaling is exact).
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"

namespace attn_b200 {

constexpr int kQuantThreads = 512;  // 128 rows x 4 lanes: one tile per pass
constexpr int kQuantRows = 128;
constexpr int kQuantE = 32;          // coordinates per thread (d = 128)

enum QuantMode : int {
  kQuantPerTile = 0,  // scale per 128-row tile, codes written
  kQuantAmaxOnly = 1, // tile amax written, nothing else
  kQuantPerHead = 2,  // scale per head from the stored tile amaxes, codes written
};

struct QuantParams {
  const uint16_t *x;    // [BH, N, D] bf16
  uint8_t *codes;       // [BH, N, D] E4M3
  float *scales;        // per tile: [BH, tiles]; per head: [BH]
  float *tile_amax;     // [BH, tiles] (amax pass writes, per-head pass reads)
  uint64_t sign_lo, sign_hi;  // rotation signs, bit t -> coordinate t
  int bh, n, tiles;
  int rotate;
};

// Largest e (at most 126) with amax * 2^e <= 448; 0 when amax is 0.
__device__ __forceinline__ int e4m3_block_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  int E;
  frexpf(amax, &E);  // amax = f 2^E, f in [0.5, 1)
  int e = 9 - E;     // amax * 2^e < 2^9
  while (ldexpf(amax, e) > 448.f) --e;
  return e > 126 ? 126 : e;
}

// This thread's 32 bf16 values of tile `tile_id` (zeros past N): 4 x 16 B.
__device__ __forceinline__ void quant_load(const QuantParams &p, int tile_id, int row,
                                           int q4, uint4 (&raw)[4]) {
  const int bh = tile_id / p.tiles;
  const int r = (tile_id - bh * p.tiles) * kQuantRows + row;
  if (r < p.n) {
    const uint4 *src = reinterpret_cast<const uint4 *>(
        p.x + (static_cast<int64_t>(bh) * p.n + r) * 128 + q4 * kQuantE);
#pragma unroll
    for (int i = 0; i < 4; ++i) raw[i] = src[i];
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) raw[i] = make_uint4(0, 0, 0, 0);
  }
}

// The rotated (or plain) values of the thread's coordinates, rounded to fp32.
// Every lane of the warp must call this (the shuffles name the full warp).
__device__ __forceinline__ void quant_transform(const QuantParams &p, int q4,
                                                const uint4 (&raw)[4], float (&y)[kQuantE]) {
  constexpr int E = kQuantE;
  if (!p.rotate) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        y[8 * i + 2 * j] = __uint_as_float(w4[j] << 16);
        y[8 * i + 2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
      }
    }
    return;
  }
  double x[E];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[8 * i + 2 * j] = __uint_as_float(w4[j] << 16);
      x[8 * i + 2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
    }
  }
  const uint64_t word = (q4 * E < 64) ? p.sign_lo : p.sign_hi;
  const uint32_t bits = static_cast<uint32_t>(word >> ((q4 * E) & 63));
#pragma unroll
  for (int k = 0; k < E; ++k)
    if ((bits >> k) & 1u) x[k] = -x[k];
  // butterflies of span h < 32 inside the thread
#pragma unroll
  for (int h = 1; h < E; h <<= 1)
#pragma unroll
    for (int k = 0; k < E; ++k)
      if ((k & h) == 0) {
        const double a = x[k], b = x[k + h];
        x[k] = a + b;
        x[k + h] = a - b;
      }
  // spans 32 and 64 pair lane with lane ^ 1, lane ^ 2 of its row: the lane
  // holding the lower coordinate t keeps x_t + x_{t+h}, the other keeps
  // x_t - x_{t+h} seen from its partner (partner - own)
#pragma unroll
  for (int lh = 1; lh < 4; lh <<= 1) {
    const bool upper = (q4 & lh) != 0;
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const double other = __shfl_xor_sync(0xffffffffu, x[k], lh);
      x[k] = upper ? (other - x[k]) : (x[k] + other);
    }
  }
#pragma unroll
  for (int k = 0; k < E; ++k) y[k] = static_cast<float>(x[k]);  // nearest even
}

// Persistent over tiles t = blockIdx.x, blockIdx.x + gridDim.x, ... of all
// heads (t = bh * tiles + tile).  One __syncthreads per tile: the block
// maximum's partial values (and, per head, the head maximum) live in slots
// indexed by the tile's parity, so a slot is rewritten only after every
// thread has passed the next tile's barrier.
template <int D>
__global__ void __launch_bounds__(kQuantThreads, 1)
    fp8_quant_kernel(const QuantParams p, const int mode) {
  static_assert(D == 128, "the FP8 path supports head dimension 128");
  __shared__ float warp_amax[2][kQuantThreads / 32];
  __shared__ float head_amax[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = threadIdx.x >> 2, q4 = threadIdx.x & 3;
  const int total = p.bh * p.tiles;
  uint4 nxt[4];
  int t = blockIdx.x;
  if (t < total) quant_load(p, t, row, q4, nxt);
  for (int it = 0; t < total; t += gridDim.x, ++it) {
    uint4 cur[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
    if (t + static_cast<int>(gridDim.x) < total)
      quant_load(p, t + gridDim.x, row, q4, nxt);  // in flight during this tile
    const int bh = t / p.tiles;
    const int tile = t - bh * p.tiles;
    const int r = tile * kQuantRows + row;
    float y[kQuantE];
    quant_transform(p, q4, cur, y);  // rows past N hold zeros

    const int slot = it & 1;
    if (mode != kQuantPerHead) {
      float a = 0.f;
#pragma unroll
      for (int k = 0; k < kQuantE; ++k) a = fmaxf(a, fabsf(y[k]));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      if (lane == 0) warp_amax[slot][warp] = a;
    } else if (warp == 0) {
      // the head's amax from every tile's (written by the amax pass)
      float a = 0.f;
      for (int i = lane; i < p.tiles; i += 32)
        a = fmaxf(a, p.tile_amax[static_cast<int64_t>(bh) * p.tiles + i]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      if (lane == 0) head_amax[slot] = a;
    }
    __syncthreads();
    float amax;
    if (mode == kQuantPerHead) {
      amax = head_amax[slot];
    } else {
      amax = warp_amax[slot][0];
#pragma unroll
      for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, warp_amax[slot][w]);
    }
    if (mode == kQuantAmaxOnly) {
      if (threadIdx.x == 0) p.tile_amax[t] = amax;
      continue;
    }
    const int e = e4m3_block_exponent(amax);
    if (threadIdx.x == 0) {
      if (mode == kQuantPerTile)
        p.scales[t] = ldexpf(1.f, -e);
      else if (tile == 0)
        p.scales[bh] = ldexpf(1.f, -e);
    }
    if (r < p.n) {
      const float mul = ldexpf(1.f, e);  // exact: a power of two
      uint32_t w[8];
#pragma unroll
      for (int g = 0; g < 8; ++g)
        w[g] = pack_e4m3x4(y[4 * g] * mul, y[4 * g + 1] * mul, y[4 * g + 2] * mul,
                           y[4 * g + 3] * mul);
      uint4 *dst = reinterpret_cast<uint4 *>(
          p.codes + (static_cast<int64_t>(bh) * p.n + r) * 128 + q4 * kQuantE);
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  }
}

}  // namespace attn_b200
