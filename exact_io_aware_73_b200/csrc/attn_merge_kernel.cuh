// attn_merge_kernel.cuh -- exact merge of partial attention results for B200.
//
// Sources: the marketmaker.cc post (Indonesian edition) "Apakah Konteks
// Sehari Penuh Mengalahkan Konteks Sepuluh Menit? ...", section "Backward
// pass: menghitung ulang, bukan menyimpan" (the softmax statistics m, l kept
// per row, here folded into lse = m + ln l), and the briefgpt.xyz summary
// page of FlashAttention-2 (arXiv 2307.08691), entry "BurstAttention"
// (attention distributed over devices along the sequence).
//
// Attention of a row over keys split into disjoint parts s is exactly
//     lse = log sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s,
// where (O_s, lse_s) is the row's attention over part s alone.  These
// kernels fold one part at a time into an fp32 accumulator (O, lse) and
// write the final bf16 output; a part in which the row sees no key has
// lse_s = -inf and weight 0.  Elementwise and HBM-bound: one warp per row,
// coalesced 8- or 16-byte accesses.
#pragma once

#include <cstdint>
#include <math_constants.h>

#include "ptx_sm100.cuh"

namespace attn_b200 {

// acc_o [rows, D] fp32, acc_lse [rows] fp32; part_o [rows, D] bf16,
// part_lse [rows] fp32.  first != 0: the accumulator is initialised from the
// part.  One warp per row (D/32 dimensions per lane): every lane reads the
// row's two log-sum-exps before lane 0 overwrites the accumulator's.
template <int D>
__global__ void __launch_bounds__(256)
    attn_merge_fold_kernel(float *acc_o, float *acc_lse, const uint16_t *part_o,
                           const float *part_lse, int64_t rows, int first) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
       r < rows; r += warps) {
    const float lp = part_lse[r];
    const float la = first ? -CUDART_INF_F : acc_lse[r];
    __syncwarp();
    const float m = fmaxf(la, lp);
    float wa = 0.f, wp = 0.f, lnew = -CUDART_INF_F;
    if (m != -CUDART_INF_F) {  // some part so far sees a key of this row
      wa = (la == -CUDART_INF_F) ? 0.f : __expf(la - m);
      wp = (lp == -CUDART_INF_F) ? 0.f : __expf(lp - m);
      const float t = wa + wp;
      lnew = m + __logf(t);
      wa = __fdividef(wa, t);
      wp = __fdividef(wp, t);
    }
    float pv[E], av[E];
    if constexpr (E == 4) {
      const uint2 raw = reinterpret_cast<const uint2 *>(part_o + r * D)[lane];
      pv[0] = __uint_as_float(raw.x << 16); pv[1] = __uint_as_float(raw.x & 0xFFFF0000u);
      pv[2] = __uint_as_float(raw.y << 16); pv[3] = __uint_as_float(raw.y & 0xFFFF0000u);
      const float4 a4 = first ? make_float4(0.f, 0.f, 0.f, 0.f)
                              : reinterpret_cast<const float4 *>(acc_o + r * D)[lane];
      av[0] = a4.x; av[1] = a4.y; av[2] = a4.z; av[3] = a4.w;
      reinterpret_cast<float4 *>(acc_o + r * D)[lane] =
          make_float4(wa * av[0] + wp * pv[0], wa * av[1] + wp * pv[1],
                      wa * av[2] + wp * pv[2], wa * av[3] + wp * pv[3]);
    } else {
      const uint32_t raw = reinterpret_cast<const uint32_t *>(part_o + r * D)[lane];
      pv[0] = __uint_as_float(raw << 16); pv[1] = __uint_as_float(raw & 0xFFFF0000u);
      const float2 a2 = first ? make_float2(0.f, 0.f)
                              : reinterpret_cast<const float2 *>(acc_o + r * D)[lane];
      av[0] = a2.x; av[1] = a2.y;
      reinterpret_cast<float2 *>(acc_o + r * D)[lane] =
          make_float2(wa * av[0] + wp * pv[0], wa * av[1] + wp * pv[1]);
    }
    if (lane == 0) acc_lse[r] = lnew;
  }
}

// O = bf16(acc_o) [rows, D], lse = acc_lse; one warp per row.
template <int D>
__global__ void __launch_bounds__(256)
    attn_merge_finish_kernel(const float *acc_o, const float *acc_lse, uint16_t *out_o,
                             float *out_lse, int64_t rows) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
       r < rows; r += warps) {
    if constexpr (E == 4) {
      const float4 a = reinterpret_cast<const float4 *>(acc_o + r * D)[lane];
      reinterpret_cast<uint2 *>(out_o + r * D)[lane] =
          make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
    } else {
      const float2 a = reinterpret_cast<const float2 *>(acc_o + r * D)[lane];
      reinterpret_cast<uint32_t *>(out_o + r * D)[lane] = pack_bf16x2(a.x, a.y);
    }
    if (lane == 0) out_lse[r] = acc_lse[r];
  }
}

}  // namespace attn_b200
