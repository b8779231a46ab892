// attn_api.cu -- host side of the C ABI declared in include/attn_b200.h:
// argument validation, TMA descriptor encoding, kernel selection and launch,
// the per-device status word, and the host-buffer (end-to-end) entry point.
//
// The operation and its layouts are defined in the header.  This file makes
// no CUDA call before every argument check has passed.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_b200.h"
#include "attn_bwd_kernel.cuh"
#include "fp8_quant_kernel.cuh"
#include "attn_decode_kernel.cuh"
#include "attn_decode_mma_kernel.cuh"
#include "attn_merge_kernel.cuh"

namespace {

using attn_b200::FwdParams;
using attn_b200::Smem;

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 1000000000ull;

struct DeviceState {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  uint32_t *status = nullptr;  // 4-byte device status word, lazily allocated
  // forward variants: 0-3 bf16 (d, causal), 4-5 E4M3, 6-9 block-sparse bf16
  bool smem_attr_set[10] = {false, false, false, false, false,
                            false, false, false, false, false};
  bool bwd_attr_set[4] = {false, false, false, false};
  bool dec_attr_set[2] = {false, false};  // decode kernel, d = 128 / 64
  bool dm_attr_set[2] = {false, false};   // tensor-core decode kernel, d = 128 / 64
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<uint32_t> g_inject{0};
std::atomic<uint32_t> g_last_bits{0};
std::atomic<int> g_decode_max_ctas{0};
std::atomic<int> g_decode_kernel{0};  // 0 automatic, 1 CUDA cores, 2 tensor cores

// Error code for a nonzero device status word: a wait that ran out of time
// wins over a failed index check of the debug build; any other bit is a
// generic failure.
int status_bits_to_code(uint32_t bits) {
  if (bits & attn_b200::kStatusTimeout) return ATTN_ERR_DEVICE_TIMEOUT;
  if (bits & attn_b200::kStatusBounds) return ATTN_ERR_DEVICE_BOUNDS;
  return ATTN_ERR_CUDA;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t,
                                  void *, const cuuint64_t *, const cuuint64_t *,
                                  const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int get_encode_fn(EncodeTiledFn *out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPointByVersion(
        "cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
      return ATTN_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  *out = g_encode;
  return ATTN_OK;
}

// Current device, checked to be a B200 (compute capability 10.0); allocates
// the device's status word on first use.
int current_device(int *dev_out, DeviceState **st_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ATTN_ERR_UNSUPPORTED_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState &st = g_dev[dev];
  if (!st.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_UNSUPPORTED_DEVICE;
    }
    st.probed = true;
    st.supported = (major == 10 && minor == 0);
    st.sm_count = sms;
  }
  if (!st.supported) return ATTN_ERR_UNSUPPORTED_DEVICE;
  if (!st.status) {
    void *p = nullptr;
    if (cudaMalloc(&p, sizeof(uint32_t)) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    if (cudaMemset(p, 0, sizeof(uint32_t)) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(p);
      return ATTN_ERR_CUDA;
    }
    st.status = static_cast<uint32_t *>(p);
  }
  *dev_out = dev;
  *st_out = &st;
  return ATTN_OK;
}

bool is_device_memory_of(const void *p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) &&
         a.device == dev;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a);
  const uintptr_t y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Shape / pointer checks shared by both entry points (no CUDA calls).
int check_args(const void *q, const void *k, const void *v, const void *o,
               const float *lse, int B, int H, int N, int d, float scale,
               bool check_alignment) {
  if (B < 0 || H < 0 || N < 0) return ATTN_ERR_INVALID_SIZE;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED_HEAD_DIM;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID_SCALE;
  if (B == 0 || H == 0 || N == 0) return ATTN_OK;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL_POINTER;
  const int64_t bh = static_cast<int64_t>(B) * H;
  if (N > ATTN_MAX_SEQ || bh > ATTN_MAX_HEADS) return ATTN_ERR_INVALID_SIZE;
  const int64_t units = bh * ((N + 255) / 256);
  if (units > 0x7fffffffLL) return ATTN_ERR_INVALID_SIZE;
  if (check_alignment) {
    auto al = [](const void *p, uintptr_t a) {
      return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
    };
    if (!al(q, 16) || !al(k, 16) || !al(v, 16) || !al(o, 16) || !al(lse, 4))
      return ATTN_ERR_MISALIGNED;
  }
  const size_t tbytes = static_cast<size_t>(bh) * N * d * 2;
  const size_t lbytes = static_cast<size_t>(bh) * N * 4;
  if (overlaps(o, tbytes, q, tbytes) || overlaps(o, tbytes, k, tbytes) ||
      overlaps(o, tbytes, v, tbytes) || overlaps(lse, lbytes, q, tbytes) ||
      overlaps(lse, lbytes, k, tbytes) || overlaps(lse, lbytes, v, tbytes) ||
      overlaps(lse, lbytes, o, tbytes))
    return ATTN_ERR_ALIAS;
  return ATTN_OK;
}

// [B*H, N, d] bf16 viewed as a 3-D tensor (d innermost); boxes of 64 x 128
// rows (or box_rows), 128-byte swizzle -- the shared-memory layout the UMMA
// descriptors in the kernels expect.  Rows beyond N read as zero.
int encode_map(EncodeTiledFn enc, CUtensorMap *map, const void *ptr, int bh,
               int N, int d, unsigned box_rows = 128) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void *>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_TENSOR_MAP;
}

// E4M3 codes [B*H, N, d] as a 3-D byte tensor; boxes of 128 x 128 rows
// (one 128-byte swizzle panel per row at d = 128).
int encode_map_u8(EncodeTiledFn enc, CUtensorMap *map, const void *ptr, int bh,
                  int N, int d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d),
                           static_cast<cuuint64_t>(N) * d};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr),
                   dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_TENSOR_MAP;
}

template <int D, bool CAUSAL, bool FP8 = false, bool SPARSE = false>
int launch(DeviceState &st, int variant, const CUtensorMap *maps,
           const FwdParams &p, cudaStream_t stream) {
  auto kern = attn_b200::attn_fwd_sm100_kernel<D, CAUSAL, FP8, SPARSE>;
  const uint32_t smem = Smem<D, FP8>::kAlloc;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!st.smem_attr_set[variant]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem)) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      st.smem_attr_set[variant] = true;
    }
  }
  // O (bf16 [B*H, N, D]) as the epilogue's TMA store sees it: boxes of 64
  // columns x 32 rows, one per softmax warp and half row.  The merge modes
  // write through the accumulator instead and leave the map unused.
  CUtensorMap map_o;
  std::memset(&map_o, 0, sizeof map_o);
  if (p.merge_mode == attn_b200::kMergeNone) {
    EncodeTiledFn enc;
    int rc = get_encode_fn(&enc);
    if (rc == ATTN_OK) rc = encode_map(enc, &map_o, p.o, p.bh, p.n, D, 32);
    if (rc != ATTN_OK) return rc;
  }
  // Non-causal units are pairs of Q tiles of equal cost.  When the last
  // round of pairs would fill at most half of the CTAs (or every pair fits
  // in half of them), those pairs run as single Q tiles on twice as many
  // CTAs: a lone tile shares neither the tensor pipe nor the exponential
  // unit, so it takes well under the time of a pair.
  FwdParams q = p;
  if (!CAUSAL && !SPARSE) {
    const int64_t S = st.sm_count, U2 = p.num_units;
    if (2 * U2 <= S) {
      q.tail_start = 0;
      q.num_units = static_cast<int>(2 * U2);
    } else {
      const int64_t G = U2 < S ? U2 : S, R = U2 / G, r = U2 % G;
      if (r > 0 && 2 * r <= G && U2 + r <= 0x7fffffffLL) {
        q.tail_start = static_cast<int>(G * R);
        q.num_units = static_cast<int>(G * R + 2 * r);
      }
    }
  }
  const int grid = q.num_units < st.sm_count ? q.num_units : st.sm_count;
  kern<<<grid, attn_b200::kThreads, smem, stream>>>(maps[0], maps[1], maps[2], map_o, q);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// attn_fwd_host's copy / compute pipeline: three streams and their events,
// created once per device on first use and kept until process exit.
constexpr int kHostChunks = 8;
struct HostPipe {
  bool ready = false;
  std::mutex mu;  // one call enqueues at a time (events are reused)
  cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t in_done[kHostChunks] = {}, k_done[kHostChunks] = {};
};
HostPipe g_pipe[kMaxDevices];

int host_pipe(int dev, HostPipe **out) {
  std::lock_guard<std::mutex> lk(g_mu);
  HostPipe &hp = g_pipe[dev];
  if (!hp.ready) {
    const unsigned fl = cudaStreamNonBlocking;
    bool ok = cudaStreamCreateWithFlags(&hp.h2d, fl) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.comp, fl) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.d2h, fl) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.end, cudaEventDisableTiming) == cudaSuccess;
    for (int c = 0; ok && c < kHostChunks; ++c)
      ok = cudaEventCreateWithFlags(&hp.in_done[c], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.k_done[c], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    hp.ready = true;
  }
  *out = &hp;
  return ATTN_OK;
}

// fp32 vectors [bh, npad] (npad a multiple of 128) as a 2-D tensor with
// 128-entry boxes: row stride npad * 4 bytes and every box start (x = 128 i)
// are 512-byte multiples.
int encode_vec_map(EncodeTiledFn enc, CUtensorMap *map, const void *ptr, int bh,
                   int npad) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(npad), static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(npad) * 4};
  cuuint32_t box[2] = {128, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(ptr),
                   dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_TENSOR_MAP;
}

template <int D, bool CAUSAL>
int launch_bwd(DeviceState &st, int variant, const CUtensorMap *m,
               const attn_b200::BwdParams &p, cudaStream_t stream) {
  using namespace attn_b200;
  auto kdq = attn_bwd_dq_kernel<D, CAUSAL>;
  auto kdkv = attn_bwd_dkdv_kernel<D, CAUSAL>;
  const uint32_t smem_dq = BwdDqSmem<D>::kAlloc;
  const uint32_t smem_dkv = BwdDkvSmem<D>::kAlloc;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!st.bwd_attr_set[variant]) {
      if (cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_dq)) != cudaSuccess ||
          cudaFuncSetAttribute(kdkv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_dkv)) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      st.bwd_attr_set[variant] = true;
    }
  }
  const int64_t prep_rows = static_cast<int64_t>(p.bh) * p.npad;
  const int64_t prep_blocks_needed = (prep_rows + 7) / 8;
  const int prep_blocks = static_cast<int>(
      prep_blocks_needed < st.sm_count * 16 ? prep_blocks_needed : st.sm_count * 16);
  attn_bwd_prep_kernel<D><<<prep_blocks, 256, 0, stream>>>(p);
  const int grid = p.num_units < st.sm_count ? p.num_units : st.sm_count;
  kdq<<<grid, kBwdThreads, smem_dq, stream>>>(m[0], m[1], m[2], m[3], p);
  kdkv<<<grid, kBwdThreads, smem_dkv, stream>>>(m[0], m[1], m[2], m[3], m[4], m[5], p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

// One fp8_quant_kernel launch over every 128-row tile of every head: one
// persistent CTA per SM (or per tile, when there are fewer tiles).
int launch_quant(DeviceState &st, const attn_b200::QuantParams &p, int mode,
                 cudaStream_t stream) {
  const int64_t tiles = static_cast<int64_t>(p.bh) * p.tiles;
  const int grid = static_cast<int>(tiles < st.sm_count ? tiles : st.sm_count);
  attn_b200::fp8_quant_kernel<128><<<grid, attn_b200::kQuantThreads, 0, stream>>>(p, mode);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

template <int D, int QMAX>
int launch_decode(DeviceState &st, int variant, attn_b200::DecodeParams &p,
                  cudaStream_t stream) {
  using L = attn_b200::DecSmem<D>;
  auto kern = attn_b200::attn_decode_kernel<D, QMAX>;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!st.dec_attr_set[variant]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(L::kBytes)) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      st.dec_attr_set[variant] = true;
    }
  }
  // stream-K: an equal share of the key tiles per CTA, two CTAs per SM
  int ctas = g_decode_max_ctas.load();
  if (ctas <= 0) ctas = 2 * st.sm_count;
  if (ctas > attn_b200::kDecMaxCtas) ctas = attn_b200::kDecMaxCtas;
  const int grid0 = p.total < ctas ? p.total : ctas;
  p.per_cta = (p.total + grid0 - 1) / grid0;
  const int grid = (p.total + p.per_cta - 1) / p.per_cta;
  if (cudaMemsetAsync(p.counters, 0, sizeof(int) * static_cast<size_t>(p.bh), stream) !=
      cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  kern<<<grid, attn_b200::kDecThreads, L::kBytes, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

// Which decode kernel serves Nq queries per head at head size d when the
// caller leaves the choice to the library.  Measured on B200 (both kernels
// forced, B=16 H=12 Nk=23400, Nq = 1 .. 16): the tensor-core kernel streams
// K/V faster for every Nq at both head sizes (d = 128: 6412 against 6351
// GB/s at one query; d = 64: 6121 against 5708 at one query, 6098 against
// 4097 at four), so it always serves unless a test forces the other.
bool decode_prefers_mma(int, int) { return true; }

// The tensor-core decode: one CTA per SM, an equal share of the key tiles of
// all heads each (stream-K), the per-head part counters zeroed first.
template <int D>
int launch_decode_mma(DeviceState &st, const CUtensorMap *maps,
                      attn_b200::DecodeMmaParams &p, cudaStream_t stream) {
  using L = attn_b200::DmSmem<D>;
  auto kern = attn_b200::attn_decode_mma_kernel<D>;
  constexpr int variant = D == 128 ? 0 : 1;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!st.dm_attr_set[variant]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(L::kAlloc)) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      st.dm_attr_set[variant] = true;
    }
  }
  int ctas = g_decode_max_ctas.load();
  if (ctas <= 0) ctas = st.sm_count;
  if (ctas > attn_b200::kDmMaxCtas) ctas = attn_b200::kDmMaxCtas;
  const int grid0 = p.total < ctas ? p.total : ctas;
  p.per_cta = (p.total + grid0 - 1) / grid0;
  const int grid = (p.total + p.per_cta - 1) / p.per_cta;
  if (cudaMemsetAsync(p.counters, 0, sizeof(int) * static_cast<size_t>(p.bh), stream) !=
      cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  kern<<<grid, attn_b200::kDmThreads, L::kAlloc, stream>>>(maps[0], maps[1], maps[2], p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

// Size checks shared by the FP8 entries (no CUDA calls).
int check_fp8_sizes(int B, int H, int N, int d) {
  if (B < 0 || H < 0 || N < 0) return ATTN_ERR_INVALID_SIZE;
  if (d != 128) return ATTN_ERR_UNSUPPORTED_HEAD_DIM;
  const int64_t bh = static_cast<int64_t>(B) * H;
  if (N > ATTN_MAX_SEQ || bh > ATTN_MAX_HEADS) return ATTN_ERR_INVALID_SIZE;
  if (bh * ((N + 255) / 256) > 0x7fffffffLL || bh * ((N + 127) / 128) > 0x7fffffffLL)
    return ATTN_ERR_INVALID_SIZE;
  return ATTN_OK;
}

bool aligned(const void *p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

__global__ void exp2_selftest_kernel(const float *x, float *y, int n, int mode) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = (i + 1 < n) ? x[i + 1] : 0.f;
  float y0, y1;
  if (mode == 0) {
    attn_b200::f32x2_split(attn_b200::exp2_poly_x2(x0, x1), y0, y1);
  } else {
    y0 = attn_b200::ex2_approx(x0);
    y1 = attn_b200::ex2_approx(x1);
  }
  y[i] = y0;
  if (i + 1 < n) y[i + 1] = y1;
}

// Head chunks of the host-buffer entries.  The step ends with the last
// chunk's kernel and copies out, after all copies in, so the chunks shrink
// towards the end (for 32 heads: 6, 6, 6, 6, 4, 2, 1, 1) and little work is
// left once the last copy in lands; compute (a few ms) stays well behind the
// copies in.  Problems below 32 MiB per tensor run as one chunk.
int host_chunks(int bh, size_t tensor_bytes, int (&sizes)[kHostChunks]) {
  sizes[0] = bh;
  if (tensor_bytes < (32u << 20) || bh <= 1) return 1;
  if (bh <= kHostChunks) {
    for (int c = 0; c < bh; ++c) sizes[c] = 1;
    return bh;
  }
  const int tail[4] = {bh / 8 > 0 ? bh / 8 : 1, bh / 16 > 0 ? bh / 16 : 1,
                       bh / 32 > 0 ? bh / 32 : 1, bh / 32 > 0 ? bh / 32 : 1};
  const int head = bh - (tail[0] + tail[1] + tail[2] + tail[3]);
  for (int c = 0; c < 4; ++c) sizes[c] = head / 4 + (c < head % 4 ? 1 : 0);
  for (int c = 0; c < 4; ++c) sizes[4 + c] = tail[c];
  return kHostChunks;
}

// The largest head chunk host_chunks gives for B*H heads of N x d.
int host_max_chunk(int bh, int N, int d) {
  int sizes[kHostChunks];
  const int nc = host_chunks(bh, static_cast<size_t>(bh) * N * d * 2, sizes);
  int m = 0;
  for (int c = 0; c < nc; ++c) m = sizes[c] > m ? sizes[c] : m;
  return m;
}

// The copy / compute pipeline shared by the host-buffer entries: chunk i's
// copies in (host -> staging), its computation `chunk(h0, nh, comp stream)`
// and its copies out run on three library-owned streams, so that they
// overlap chunk i+1's copies in and chunk i-1's copies out.  `stream`
// orders the whole call: the streams start after its earlier work and it
// waits for the last copy out.  Staging: dq, dk, dv, dout [bh, N, d] bf16
// and dl [bh, N] fp32 in device memory.
template <typename ChunkFn>
int run_host_pipeline(const void *q, const void *k, const void *v, void *o, float *lse,
                      int bh, int N, int d, uint8_t *dq, uint8_t *dk, uint8_t *dv,
                      uint8_t *dout, float *dl, cudaStream_t s, ChunkFn chunk) {
  int rc, dev;
  DeviceState *st;
  if ((rc = current_device(&dev, &st)) != ATTN_OK) return rc;
  HostPipe *hp = nullptr;
  if ((rc = host_pipe(dev, &hp)) != ATTN_OK) return rc;
  int sizes[kHostChunks];
  const int nchunks = host_chunks(bh, static_cast<size_t>(bh) * N * d * 2, sizes);
  std::lock_guard<std::mutex> lk(hp->mu);
  auto fail = [] { cudaGetLastError(); return ATTN_ERR_CUDA; };
  if (cudaEventRecord(hp->start, s) != cudaSuccess) return fail();
  for (cudaStream_t t : {hp->h2d, hp->comp, hp->d2h})
    if (cudaStreamWaitEvent(t, hp->start, 0) != cudaSuccess) return fail();
  for (int c = 0, h0 = 0; c < nchunks; h0 += sizes[c], ++c) {
    const int nh = sizes[c];
    if (nh <= 0) continue;
    const size_t off = static_cast<size_t>(h0) * N * d * 2;
    const size_t len = static_cast<size_t>(nh) * N * d * 2;
    const size_t loff = static_cast<size_t>(h0) * N, llen = static_cast<size_t>(nh) * N;
    const uint8_t *hq = static_cast<const uint8_t *>(q), *hk = static_cast<const uint8_t *>(k),
                  *hv = static_cast<const uint8_t *>(v);
    if (cudaMemcpyAsync(dq + off, hq + off, len, cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess ||
        cudaMemcpyAsync(dk + off, hk + off, len, cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess ||
        cudaMemcpyAsync(dv + off, hv + off, len, cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess ||
        cudaEventRecord(hp->in_done[c], hp->h2d) != cudaSuccess ||
        cudaStreamWaitEvent(hp->comp, hp->in_done[c], 0) != cudaSuccess)
      return fail();
    rc = chunk(h0, nh, reinterpret_cast<attn_stream_t>(hp->comp));
    if (rc != ATTN_OK) return rc;
    if (cudaEventRecord(hp->k_done[c], hp->comp) != cudaSuccess ||
        cudaStreamWaitEvent(hp->d2h, hp->k_done[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t *>(o) + off, dout + off, len,
                        cudaMemcpyDeviceToHost, hp->d2h) != cudaSuccess ||
        cudaMemcpyAsync(lse + loff, dl + loff, llen * 4, cudaMemcpyDeviceToHost,
                        hp->d2h) != cudaSuccess)
      return fail();
  }
  if (cudaEventRecord(hp->end, hp->d2h) != cudaSuccess ||
      cudaStreamWaitEvent(s, hp->end, 0) != cudaSuccess)
    return fail();
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
             int B, int H, int N, int d, int causal, float scale,
             attn_stream_t stream) {
  int rc = check_args(q, k, v, o, lse, B, H, N, d, scale, true);
  if (rc != ATTN_OK || B == 0 || H == 0 || N == 0) return rc;

  int dev;
  DeviceState *st;
  if ((rc = current_device(&dev, &st)) != ATTN_OK) return rc;
  if (!is_device_memory_of(q, dev) || !is_device_memory_of(k, dev) ||
      !is_device_memory_of(v, dev) || !is_device_memory_of(o, dev) ||
      !is_device_memory_of(lse, dev))
    return ATTN_ERR_NOT_DEVICE_MEMORY;

  EncodeTiledFn enc;
  if ((rc = get_encode_fn(&enc)) != ATTN_OK) return rc;
  const int bh = B * H;
  CUtensorMap maps[3];
  if ((rc = encode_map(enc, &maps[0], q, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[1], k, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[2], v, bh, N, d)) != ATTN_OK) return rc;

  FwdParams p;
  p.o = static_cast<uint16_t *>(o);
  p.lse = lse;
  p.status = st->status;
  p.bh = bh;
  p.n = N;
  p.num_units = bh * ((N + 255) / 256);
  p.c_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.timeout_ns = g_timeout_ns.load();
  p.debug_flags = g_inject.load() & 5u;  // bits 0 and 2 concern this kernel

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? launch<128, true>(*st, 0, maps, p, s)
                  : launch<128, false>(*st, 1, maps, p, s);
  return causal ? launch<64, true>(*st, 2, maps, p, s)
                : launch<64, false>(*st, 3, maps, p, s);
}

int attn_fwd_block_sparse(const void *q, const void *k, const void *v, void *o,
                          float *lse, int B, int H, int N, int d, int causal,
                          float scale, const uint8_t *block_mask,
                          int mask_per_head, attn_stream_t stream) {
  int rc = check_args(q, k, v, o, lse, B, H, N, d, scale, true);
  if (rc != ATTN_OK || B == 0 || H == 0 || N == 0) return rc;
  if (!block_mask) return ATTN_ERR_NULL_POINTER;
  const int bh = B * H;
  const int tiles = (N + 127) / 128;
  const int64_t units = static_cast<int64_t>(bh) * ((tiles + 1) / 2);
  if (units > 0x7fffffffLL) return ATTN_ERR_INVALID_SIZE;
  const size_t mask_bytes = static_cast<size_t>(mask_per_head ? bh : 1) * tiles * tiles;
  const size_t tb = static_cast<size_t>(bh) * N * d * 2, lb = static_cast<size_t>(bh) * N * 4;
  if (overlaps(o, tb, block_mask, mask_bytes) || overlaps(lse, lb, block_mask, mask_bytes))
    return ATTN_ERR_ALIAS;

  int dev;
  DeviceState *st;
  if ((rc = current_device(&dev, &st)) != ATTN_OK) return rc;
  if (!is_device_memory_of(q, dev) || !is_device_memory_of(k, dev) ||
      !is_device_memory_of(v, dev) || !is_device_memory_of(o, dev) ||
      !is_device_memory_of(lse, dev) || !is_device_memory_of(block_mask, dev))
    return ATTN_ERR_NOT_DEVICE_MEMORY;

  EncodeTiledFn enc;
  if ((rc = get_encode_fn(&enc)) != ATTN_OK) return rc;
  CUtensorMap maps[3];
  if ((rc = encode_map(enc, &maps[0], q, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[1], k, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[2], v, bh, N, d)) != ATTN_OK) return rc;

  FwdParams p;
  p.o = static_cast<uint16_t *>(o);
  p.lse = lse;
  p.status = st->status;
  p.bh = bh;
  p.n = N;
  p.num_units = static_cast<int>(units);  // two consecutive Q tiles per unit
  p.c_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.timeout_ns = g_timeout_ns.load();
  p.debug_flags = 0;
  p.block_mask = block_mask;
  p.mask_head_stride = mask_per_head ? static_cast<int64_t>(tiles) * tiles : 0;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? launch<128, true, false, true>(*st, 6, maps, p, s)
                  : launch<128, false, false, true>(*st, 7, maps, p, s);
  return causal ? launch<64, true, false, true>(*st, 8, maps, p, s)
                : launch<64, false, false, true>(*st, 9, maps, p, s);
}

int attn_fwd_merge(const void *q, const void *k, const void *v, float *acc_o,
                   float *acc_lse, void *o, float *lse, int B, int H, int N, int d,
                   int causal, float scale, int mode, attn_stream_t stream) {
  if (mode != attn_b200::kMergeFirst && mode != attn_b200::kMergeInto &&
      mode != attn_b200::kMergeLast)
    return ATTN_ERR_INVALID_SIZE;
  const bool last = mode == attn_b200::kMergeLast;
  // the bf16 outputs are checked as attn_fwd's when they are written; the
  // accumulator takes their place otherwise (same alignment rules)
  int rc = check_args(q, k, v, last ? o : static_cast<void *>(acc_o),
                      last ? lse : acc_lse, B, H, N, d, scale, true);
  if (rc != ATTN_OK || B == 0 || H == 0 || N == 0) return rc;
  if (!acc_o || !acc_lse) return ATTN_ERR_NULL_POINTER;
  if (!aligned(acc_o, 16) || !aligned(acc_lse, 4)) return ATTN_ERR_MISALIGNED;
  const size_t rows = static_cast<size_t>(B) * H * N;
  const size_t tb = rows * d * 2, ab = rows * d * 4, lb = rows * 4;
  const void *ins[3] = {q, k, v};
  for (const void *in : ins)
    if (overlaps(acc_o, ab, in, tb) || overlaps(acc_lse, lb, in, tb)) return ATTN_ERR_ALIAS;
  if (overlaps(acc_o, ab, acc_lse, lb)) return ATTN_ERR_ALIAS;
  if (last && (overlaps(o, tb, acc_o, ab) || overlaps(o, tb, acc_lse, lb) ||
               overlaps(lse, lb, acc_o, ab) || overlaps(lse, lb, acc_lse, lb)))
    return ATTN_ERR_ALIAS;
  int dev;
  DeviceState *st;
  if ((rc = current_device(&dev, &st)) != ATTN_OK) return rc;
  const void *all[5] = {q, k, v, acc_o, acc_lse};
  for (const void *ptr : all)
    if (!is_device_memory_of(ptr, dev)) return ATTN_ERR_NOT_DEVICE_MEMORY;
  if (last && (!is_device_memory_of(o, dev) || !is_device_memory_of(lse, dev)))
    return ATTN_ERR_NOT_DEVICE_MEMORY;
  EncodeTiledFn enc;
  if ((rc = get_encode_fn(&enc)) != ATTN_OK) return rc;
  const int bh = B * H;
  CUtensorMap maps[3];
  if ((rc = encode_map(enc, &maps[0], q, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[1], k, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[2], v, bh, N, d)) != ATTN_OK) return rc;
  FwdParams p;
  p.o = last ? static_cast<uint16_t *>(o) : nullptr;
  p.lse = last ? lse : nullptr;
  p.acc_o = acc_o;
  p.acc_lse = acc_lse;
  p.merge_mode = mode;
  p.status = st->status;
  p.bh = bh;
  p.n = N;
  p.num_units = bh * ((N + 255) / 256);
  p.c_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.timeout_ns = g_timeout_ns.load();
  p.debug_flags = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? launch<128, true>(*st, 0, maps, p, s)
                  : launch<128, false>(*st, 1, maps, p, s);
  return causal ? launch<64, true>(*st, 2, maps, p, s)
                : launch<64, false>(*st, 3, maps, p, s);
}

size_t attn_fwd_host_workspace_bytes(int B, int H, int N, int d) {
  if (B < 0 || H < 0 || N < 0 || (d != 64 && d != 128)) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  return 4 * round256(rows * d * 2) + round256(rows * 4);
}

int attn_fwd_host(const void *q, const void *k, const void *v, void *o,
                  float *lse, int B, int H, int N, int d, int causal,
                  float scale, void *workspace, size_t workspace_bytes,
                  attn_stream_t stream) {
  int rc = check_args(q, k, v, o, lse, B, H, N, d, scale, false);
  if (rc != ATTN_OK || B == 0 || H == 0 || N == 0) return rc;
  const size_t need = attn_fwd_host_workspace_bytes(B, H, N, d);
  if (!workspace || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255) != 0)
    return ATTN_ERR_WORKSPACE;
  const int bh = B * H;
  const size_t rows = static_cast<size_t>(bh) * N;
  const size_t tbr = round256(rows * d * 2);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint8_t *dq = ws, *dk = ws + tbr, *dv = ws + 2 * tbr, *dout = ws + 3 * tbr;
  float *dl = reinterpret_cast<float *>(ws + 4 * tbr);
  return run_host_pipeline(
      q, k, v, o, lse, bh, N, d, dq, dk, dv, dout, dl,
      reinterpret_cast<cudaStream_t>(stream), [&](int h0, int nh, attn_stream_t cs) {
        const size_t off = static_cast<size_t>(h0) * N * d * 2;
        return attn_fwd(dq + off, dk + off, dv + off, dout + off,
                        dl + static_cast<size_t>(h0) * N, 1, nh, N, d, causal, scale, cs);
      });
}

size_t attn_bwd_workspace_bytes(int B, int H, int N) {
  if (B < 0 || H < 0 || N < 0) return 0;
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  return 2 * round256(static_cast<size_t>(B) * H * npad * 4);
}

int attn_bwd(const void *q, const void *k, const void *v, const void *o,
             const void *dout, const float *lse, void *dq, void *dk, void *dv,
             void *workspace, size_t workspace_bytes, int B, int H, int N,
             int d, int causal, float scale, attn_stream_t stream) {
  if (B < 0 || H < 0 || N < 0) return ATTN_ERR_INVALID_SIZE;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED_HEAD_DIM;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID_SCALE;
  if (B == 0 || H == 0 || N == 0) return ATTN_OK;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv)
    return ATTN_ERR_NULL_POINTER;
  const int64_t bh64 = static_cast<int64_t>(B) * H;
  if (N > ATTN_MAX_SEQ || bh64 > ATTN_MAX_HEADS) return ATTN_ERR_INVALID_SIZE;
  const int64_t tiles = (N + 127) / 128;
  if (bh64 * tiles > 0x7fffffffLL) return ATTN_ERR_INVALID_SIZE;
  auto al = [](const void *ptr, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0;
  };
  if (!al(q, 16) || !al(k, 16) || !al(v, 16) || !al(o, 16) || !al(dout, 16) ||
      !al(dq, 16) || !al(dk, 16) || !al(dv, 16) || !al(lse, 4))
    return ATTN_ERR_MISALIGNED;
  const size_t need = attn_bwd_workspace_bytes(B, H, N);
  if (!workspace || workspace_bytes < need || !al(workspace, 256))
    return ATTN_ERR_WORKSPACE;
  const size_t tb = static_cast<size_t>(bh64) * N * d * 2;
  const size_t lb = static_cast<size_t>(bh64) * N * 4;
  const void *ins[6] = {q, k, v, o, dout, lse};
  const size_t in_bytes[6] = {tb, tb, tb, tb, tb, lb};
  void *outs[4] = {dq, dk, dv, workspace};
  const size_t out_bytes[4] = {tb, tb, tb, need};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 6; ++b)
      if (overlaps(outs[a], out_bytes[a], ins[b], in_bytes[b])) return ATTN_ERR_ALIAS;
    for (int b = a + 1; b < 4; ++b)
      if (overlaps(outs[a], out_bytes[a], outs[b], out_bytes[b])) return ATTN_ERR_ALIAS;
  }
  int rc, dev;
  DeviceState *st;
  if ((rc = current_device(&dev, &st)) != ATTN_OK) return rc;
  const void *all[10] = {q, k, v, o, dout, lse, dq, dk, dv, workspace};
  for (const void *ptr : all)
    if (!is_device_memory_of(ptr, dev)) return ATTN_ERR_NOT_DEVICE_MEMORY;
  EncodeTiledFn enc;
  if ((rc = get_encode_fn(&enc)) != ATTN_OK) return rc;
  const int bh = B * H;
  const int npad = static_cast<int>(tiles * 128);
  float *lse2 = static_cast<float *>(workspace);
  float *dsum = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                          round256(static_cast<size_t>(bh) * npad * 4));
  CUtensorMap maps[6];
  if ((rc = encode_map(enc, &maps[0], q, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[1], dout, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[2], k, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[3], v, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_vec_map(enc, &maps[4], lse2, bh, npad)) != ATTN_OK) return rc;
  if ((rc = encode_vec_map(enc, &maps[5], dsum, bh, npad)) != ATTN_OK) return rc;
  attn_b200::BwdParams p;
  p.o = static_cast<const uint16_t *>(o);
  p.dout = static_cast<const uint16_t *>(dout);
  p.lse = lse;
  p.lse2 = lse2;
  p.dsum = dsum;
  p.dq = static_cast<uint16_t *>(dq);
  p.dk = static_cast<uint16_t *>(dk);
  p.dv = static_cast<uint16_t *>(dv);
  p.status = st->status;
  p.bh = bh;
  p.n = N;
  p.npad = npad;
  p.tiles = static_cast<int>(tiles);
  p.num_units = static_cast<int>(bh64 * tiles);
  p.c_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.scale = scale;
  p.timeout_ns = g_timeout_ns.load();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? launch_bwd<128, true>(*st, 0, maps, p, s)
                  : launch_bwd<128, false>(*st, 1, maps, p, s);
  return causal ? launch_bwd<64, true>(*st, 2, maps, p, s)
                : launch_bwd<64, false>(*st, 3, maps, p, s);
}

int attn_fp8_quantize(const void *x, void *x8, float *scales, float *tile_amax,
                      int B, int H, int N, int d, int rotate, uint64_t sign_lo,
                      uint64_t sign_hi, int per_head, attn_stream_t stream) {
  int rc = check_fp8_sizes(B, H, N, d);
  if (rc != ATTN_OK || B == 0 || H == 0 || N == 0) return rc;
  if (!x || !x8 || !scales || (per_head && !tile_amax)) return ATTN_ERR_NULL_POINTER;
  if (!aligned(x, 16) || !aligned(x8, 16) || !aligned(scales, 4) ||
      (tile_amax && !aligned(tile_amax, 4)))
    return ATTN_ERR_MISALIGNED;
  const int64_t bh = static_cast<int64_t>(B) * H;
  const int tiles = (N + 127) / 128;
  const size_t xb = static_cast<size_t>(bh) * N * d * 2, cb = xb / 2;
  const size_t sb = static_cast<size_t>(per_head ? bh : bh * tiles) * 4;
  const size_t ab = static_cast<size_t>(bh) * tiles * 4;
  if (overlaps(x8, cb, x, xb) || overlaps(scales, sb, x, xb) ||
      overlaps(scales, sb, x8, cb) ||
      (per_head && (overlaps(tile_amax, ab, x, xb) || overlaps(tile_amax, ab, x8, cb) ||
                    overlaps(tile_amax, ab, scales, sb))))
    return ATTN_ERR_ALIAS;
  int dev;
  DeviceState *st;
  if ((rc = current_device(&dev, &st)) != ATTN_OK) return rc;
  if (!is_device_memory_of(x, dev) || !is_device_memory_of(x8, dev) ||
      !is_device_memory_of(scales, dev) ||
      (per_head && !is_device_memory_of(tile_amax, dev)))
    return ATTN_ERR_NOT_DEVICE_MEMORY;
  attn_b200::QuantParams p;
  p.x = static_cast<const uint16_t *>(x);
  p.codes = static_cast<uint8_t *>(x8);
  p.scales = scales;
  p.tile_amax = tile_amax;
  p.sign_lo = sign_lo;
  p.sign_hi = sign_hi;
  p.bh = static_cast<int>(bh);
  p.n = N;
  p.tiles = tiles;
  p.rotate = rotate ? 1 : 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!per_head) return launch_quant(*st, p, attn_b200::kQuantPerTile, s);
  if ((rc = launch_quant(*st, p, attn_b200::kQuantAmaxOnly, s)) != ATTN_OK) return rc;
  return launch_quant(*st, p, attn_b200::kQuantPerHead, s);
}

int attn_fwd_fp8_quantized(const void *q8, const float *q_scale,
                           const void *k8, const float *k_scale,
                           const void *v8, const float *v_scale, void *o,
                           float *lse, int B, int H, int N, int d, int causal,
                           float scale, attn_stream_t stream) {
  int rc = check_fp8_sizes(B, H, N, d);
  if (rc != ATTN_OK) return rc;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID_SCALE;
  if (B == 0 || H == 0 || N == 0) return ATTN_OK;
  if (!q8 || !q_scale || !k8 || !k_scale || !v8 || !v_scale || !o || !lse)
    return ATTN_ERR_NULL_POINTER;
  if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v8, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(q_scale, 4) || !aligned(k_scale, 4) ||
      !aligned(v_scale, 4))
    return ATTN_ERR_MISALIGNED;
  const int64_t bh64 = static_cast<int64_t>(B) * H;
  const int tiles = (N + 127) / 128;
  const size_t cb = static_cast<size_t>(bh64) * N * d;
  const size_t ob = cb * 2, lb = static_cast<size_t>(bh64) * N * 4;
  const size_t tsb = static_cast<size_t>(bh64) * tiles * 4, vsb = bh64 * 4;
  const void *ins[6] = {q8, k8, v8, q_scale, k_scale, v_scale};
  const size_t in_bytes[6] = {cb, cb, cb, tsb, tsb, vsb};
  for (int a = 0; a < 6; ++a)
    if (overlaps(o, ob, ins[a], in_bytes[a]) || overlaps(lse, lb, ins[a], in_bytes[a]))
      return ATTN_ERR_ALIAS;
  if (overlaps(o, ob, lse, lb)) return ATTN_ERR_ALIAS;
  int dev;
  DeviceState *st;
  if ((rc = current_device(&dev, &st)) != ATTN_OK) return rc;
  const void *all[8] = {q8, k8, v8, q_scale, k_scale, v_scale, o, lse};
  for (const void *ptr : all)
    if (!is_device_memory_of(ptr, dev)) return ATTN_ERR_NOT_DEVICE_MEMORY;
  EncodeTiledFn enc;
  if ((rc = get_encode_fn(&enc)) != ATTN_OK) return rc;
  const int bh = B * H;
  CUtensorMap maps[3];
  if ((rc = encode_map_u8(enc, &maps[0], q8, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map_u8(enc, &maps[1], k8, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map_u8(enc, &maps[2], v8, bh, N, d)) != ATTN_OK) return rc;
  FwdParams p;
  p.o = static_cast<uint16_t *>(o);
  p.lse = lse;
  p.status = st->status;
  p.bh = bh;
  p.n = N;
  p.num_units = bh * ((N + 255) / 256);
  p.c_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.timeout_ns = g_timeout_ns.load();
  p.debug_flags = 0;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.tiles = tiles;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return causal ? launch<128, true, true>(*st, 4, maps, p, s)
                : launch<128, false, true>(*st, 5, maps, p, s);
}

size_t attn_fwd_fp8_workspace_bytes(int B, int H, int N, int d) {
  if (check_fp8_sizes(B, H, N, d) != ATTN_OK) return 0;
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t tiles = (static_cast<size_t>(N) + 127) / 128;
  return 3 * round256(bh * N * d) + 3 * round256(bh * tiles * 4) + round256(bh * 4);
}

int attn_fwd_fp8(const void *q, const void *k, const void *v, void *o,
                 float *lse, int B, int H, int N, int d, int causal,
                 float scale, int rotate, uint64_t sign_lo, uint64_t sign_hi,
                 void *workspace, size_t workspace_bytes, attn_stream_t stream) {
  int rc = check_fp8_sizes(B, H, N, d);
  if (rc != ATTN_OK) return rc;
  if ((rc = check_args(q, k, v, o, lse, B, H, N, d, scale, true)) != ATTN_OK) return rc;
  if (B == 0 || H == 0 || N == 0) return ATTN_OK;
  const size_t need = attn_fwd_fp8_workspace_bytes(B, H, N, d);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
    return ATTN_ERR_WORKSPACE;
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t tb = bh * N * d * 2, lb = bh * N * 4;
  const void *bufs[5] = {q, k, v, o, lse};
  const size_t bytes[5] = {tb, tb, tb, tb, lb};
  for (int a = 0; a < 5; ++a)
    if (overlaps(workspace, need, bufs[a], bytes[a])) return ATTN_ERR_ALIAS;
  const size_t tiles = (static_cast<size_t>(N) + 127) / 128;
  const size_t cbr = round256(bh * N * d), tsr = round256(bh * tiles * 4);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint8_t *q8 = ws, *k8 = ws + cbr, *v8 = ws + 2 * cbr;
  float *qs = reinterpret_cast<float *>(ws + 3 * cbr);
  float *ks = reinterpret_cast<float *>(ws + 3 * cbr + tsr);
  float *vamax = reinterpret_cast<float *>(ws + 3 * cbr + 2 * tsr);
  float *vs = reinterpret_cast<float *>(ws + 3 * cbr + 3 * tsr);
  if ((rc = attn_fp8_quantize(q, q8, qs, nullptr, B, H, N, d, rotate, sign_lo,
                              sign_hi, 0, stream)) != ATTN_OK ||
      (rc = attn_fp8_quantize(k, k8, ks, nullptr, B, H, N, d, rotate, sign_lo,
                              sign_hi, 0, stream)) != ATTN_OK ||
      (rc = attn_fp8_quantize(v, v8, vs, vamax, B, H, N, d, 0, 0, 0, 1, stream)) !=
          ATTN_OK)
    return rc;
  // unscaled Hadamard: (Q D H)(K D H)^T = d Q K^T
  const float scale_qk = rotate ? scale / static_cast<float>(d) : scale;
  return attn_fwd_fp8_quantized(q8, qs, k8, ks, v8, vs, o, lse, B, H, N, d, causal,
                                scale_qk, stream);
}

size_t attn_fwd_fp8_host_workspace_bytes(int B, int H, int N, int d) {
  if (check_fp8_sizes(B, H, N, d) != ATTN_OK) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  const int maxc = host_max_chunk(B * H, N, d);
  return 4 * round256(rows * d * 2) + round256(rows * 4) +
         attn_fwd_fp8_workspace_bytes(1, maxc > 0 ? maxc : 1, N, d);
}

int attn_fwd_fp8_host(const void *q, const void *k, const void *v, void *o, float *lse,
                      int B, int H, int N, int d, int causal, float scale, int rotate,
                      uint64_t sign_lo, uint64_t sign_hi, void *workspace,
                      size_t workspace_bytes, attn_stream_t stream) {
  int rc = check_fp8_sizes(B, H, N, d);
  if (rc != ATTN_OK) return rc;
  if ((rc = check_args(q, k, v, o, lse, B, H, N, d, scale, false)) != ATTN_OK) return rc;
  if (B == 0 || H == 0 || N == 0) return ATTN_OK;
  const size_t need = attn_fwd_fp8_host_workspace_bytes(B, H, N, d);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
    return ATTN_ERR_WORKSPACE;
  const int bh = B * H;
  const size_t rows = static_cast<size_t>(bh) * N;
  const size_t tbr = round256(rows * d * 2);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint8_t *dq = ws, *dk = ws + tbr, *dv = ws + 2 * tbr, *dout = ws + 3 * tbr;
  float *dl = reinterpret_cast<float *>(ws + 4 * tbr);
  // the FP8 codes and scales of one chunk at a time: chunks run one after
  // another on the compute stream, so they share this area
  uint8_t *fws = ws + 4 * tbr + round256(rows * 4);
  const size_t fneed = need - (4 * tbr + round256(rows * 4));
  return run_host_pipeline(
      q, k, v, o, lse, bh, N, d, dq, dk, dv, dout, dl,
      reinterpret_cast<cudaStream_t>(stream), [&](int h0, int nh, attn_stream_t cs) {
        const size_t off = static_cast<size_t>(h0) * N * d * 2;
        return attn_fwd_fp8(dq + off, dk + off, dv + off, dout + off,
                            dl + static_cast<size_t>(h0) * N, 1, nh, N, d, causal, scale,
                            rotate, sign_lo, sign_hi, fws, fneed, cs);
      });
}

size_t attn_decode_workspace_bytes(int B, int H, int Nq, int Nk, int d) {
  if (B < 0 || H < 0 || Nq < 0 || Nq > ATTN_DECODE_MAX_Q || Nk < 0 ||
      (d != 64 && d != 128))
    return 0;
  // a tensor-core launch holds a part for every query; the CUDA-core
  // launches serve at most 4 queries per head each, one after another on the
  // stream, and reuse the same slots
  static_assert(attn_b200::kDmMaxCtas <= attn_b200::kDecMaxCtas, "slot bound");
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t slots = bh + attn_b200::kDecMaxCtas;
  const size_t g = static_cast<size_t>(Nq);
  return round256(slots * g * d * 4) + round256(slots * g * 4) + round256(bh * 4);
}

int attn_decode(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int H, int Nq, int Nk, int d, int causal, float scale,
                void *workspace, size_t workspace_bytes, attn_stream_t stream) {
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_SIZE;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED_HEAD_DIM;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID_SCALE;
  if (Nq > ATTN_DECODE_MAX_Q || (Nq > 0 && Nk == 0) || (causal && Nq > Nk))
    return ATTN_ERR_INVALID_SIZE;
  if (B == 0 || H == 0 || Nq == 0) return ATTN_OK;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL_POINTER;
  const int64_t bh64 = static_cast<int64_t>(B) * H;
  if (Nk > ATTN_MAX_DECODE_KEYS || bh64 > ATTN_MAX_HEADS) return ATTN_ERR_INVALID_SIZE;
  const int tile_keys = d == 128 ? attn_b200::DecSmem<128>::kTileKeys
                                  : attn_b200::DecSmem<64>::kTileKeys;
  const int64_t ntiles = (Nk + tile_keys - 1) / tile_keys;
  if (bh64 * ntiles > 0x7fffffffLL) return ATTN_ERR_INVALID_SIZE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4))
    return ATTN_ERR_MISALIGNED;
  const size_t need = attn_decode_workspace_bytes(B, H, Nq, Nk, d);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
    return ATTN_ERR_WORKSPACE;
  const size_t qb = static_cast<size_t>(bh64) * Nq * d * 2;
  const size_t kb = static_cast<size_t>(bh64) * Nk * d * 2;
  const size_t lb = static_cast<size_t>(bh64) * Nq * 4;
  const void *ins[3] = {q, k, v};
  const size_t in_bytes[3] = {qb, kb, kb};
  void *outs[3] = {o, lse, workspace};
  const size_t out_bytes[3] = {qb, lb, need};
  for (int a = 0; a < 3; ++a) {
    for (int b = 0; b < 3; ++b)
      if (overlaps(outs[a], out_bytes[a], ins[b], in_bytes[b])) return ATTN_ERR_ALIAS;
    for (int b = a + 1; b < 3; ++b)
      if (overlaps(outs[a], out_bytes[a], outs[b], out_bytes[b])) return ATTN_ERR_ALIAS;
  }
  int rc, dev;
  DeviceState *st;
  if ((rc = current_device(&dev, &st)) != ATTN_OK) return rc;
  const void *all[6] = {q, k, v, o, lse, workspace};
  for (const void *ptr : all)
    if (!is_device_memory_of(ptr, dev)) return ATTN_ERR_NOT_DEVICE_MEMORY;
  const size_t slots = static_cast<size_t>(bh64) + attn_b200::kDecMaxCtas;
  constexpr int kGroup = attn_b200::kDecMaxQ;  // queries per CUDA-core launch
  const int choice = g_decode_kernel.load();
  const bool mma = choice == 2 || (choice == 0 && decode_prefers_mma(Nq, d));
  const size_t g = static_cast<size_t>(Nq);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (mma) {
    EncodeTiledFn enc;
    if ((rc = get_encode_fn(&enc)) != ATTN_OK) return rc;
    CUtensorMap maps[3];
    const int bhi = static_cast<int>(bh64);
    if ((rc = encode_map(enc, &maps[0], q, bhi, Nq, d, attn_b200::kDmQ)) != ATTN_OK ||
        (rc = encode_map(enc, &maps[1], k, bhi, Nk, d)) != ATTN_OK ||
        (rc = encode_map(enc, &maps[2], v, bhi, Nk, d)) != ATTN_OK)
      return rc;
    const int tile = d == 128 ? attn_b200::DmSmem<128>::kKeys : attn_b200::DmSmem<64>::kKeys;
    const int64_t nt = (Nk + tile - 1) / tile;
    attn_b200::DecodeMmaParams p;
    p.o = static_cast<uint16_t *>(o);
    p.lse = lse;
    p.part_o = reinterpret_cast<float *>(ws);
    p.part_lse = reinterpret_cast<float *>(ws + round256(slots * g * d * 4));
    p.counters = reinterpret_cast<int *>(ws + round256(slots * g * d * 4) +
                                         round256(slots * g * 4));
    p.status = st->status;
    p.bh = bhi;
    p.nq = Nq;
    p.nk = Nk;
    p.ntiles = static_cast<int>(nt);
    p.total = static_cast<int>(bh64 * nt);
    p.per_cta = 1;
    p.causal = causal ? 1 : 0;
    p.c_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.timeout_ns = g_timeout_ns.load();
    p.debug_flags = g_inject.load();
    return d == 128 ? launch_decode_mma<128>(*st, maps, p, s)
                    : launch_decode_mma<64>(*st, maps, p, s);
  }
  // groups of up to 4 queries, one launch each; under the causal mask a
  // group's last query sees keys 0 .. Nk - Nq + q0 + m - 1, so its launch
  // stops there (same visibility rule with Nk' = that count, Nq' = m)
  for (int q0 = 0; q0 < Nq; q0 += kGroup) {
    const int m = (Nq - q0 < kGroup) ? (Nq - q0) : kGroup;
    const int nk = causal ? Nk - Nq + q0 + m : Nk;
    const int64_t ntiles = (nk + tile_keys - 1) / tile_keys;
    attn_b200::DecodeParams p;
    p.q = static_cast<const uint16_t *>(q) + static_cast<int64_t>(q0) * d;
    p.k = static_cast<const uint16_t *>(k);
    p.v = static_cast<const uint16_t *>(v);
    p.o = static_cast<uint16_t *>(o) + static_cast<int64_t>(q0) * d;
    p.lse = lse + q0;
    p.part_o = reinterpret_cast<float *>(ws);
    p.part_lse = reinterpret_cast<float *>(ws + round256(slots * g * d * 4));
    p.counters = reinterpret_cast<int *>(ws + round256(slots * g * d * 4) +
                                         round256(slots * g * 4));
    p.status = st->status;
    p.bh = static_cast<int>(bh64);
    p.nq = m;
    p.nk = nk;
    p.qstride = Nq;
    p.kstride = Nk;
    p.ntiles = static_cast<int>(ntiles);
    p.total = static_cast<int>(bh64 * ntiles);
    p.per_cta = 1;
    p.causal = causal ? 1 : 0;
    p.c_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.timeout_ns = g_timeout_ns.load();
    p.debug_flags = q0 == 0 ? g_inject.load() : 0u;
    rc = d == 128 ? launch_decode<128, 4>(*st, 0, p, s) : launch_decode<64, 4>(*st, 1, p, s);
    if (rc != ATTN_OK) return rc;
  }
  return ATTN_OK;
}

void attn_set_decode_max_ctas(int n) { g_decode_max_ctas.store(n > 0 ? n : 0); }

void attn_set_decode_kernel(int which) {
  g_decode_kernel.store(which == 1 || which == 2 ? which : 0);
}

int attn_decode_kernel_for(int Nq, int d) {
  const int choice = g_decode_kernel.load();
  if (choice != 0) return choice;
  return decode_prefers_mma(Nq, d) ? 2 : 1;
}

int attn_merge_fold(float *acc_o, float *acc_lse, const void *part_o,
                    const float *part_lse, int64_t rows, int d, int first,
                    attn_stream_t stream) {
  if (rows < 0) return ATTN_ERR_INVALID_SIZE;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED_HEAD_DIM;
  if (rows == 0) return ATTN_OK;
  if (!acc_o || !acc_lse || !part_o || !part_lse) return ATTN_ERR_NULL_POINTER;
  if (!aligned(acc_o, 16) || !aligned(part_o, 16) || !aligned(acc_lse, 4) ||
      !aligned(part_lse, 4))
    return ATTN_ERR_MISALIGNED;
  const size_t ob = static_cast<size_t>(rows) * d * 4, lb = static_cast<size_t>(rows) * 4;
  if (overlaps(acc_o, ob, part_o, ob / 2) || overlaps(acc_o, ob, part_lse, lb) ||
      overlaps(acc_lse, lb, part_o, ob / 2) || overlaps(acc_lse, lb, part_lse, lb) ||
      overlaps(acc_o, ob, acc_lse, lb))
    return ATTN_ERR_ALIAS;
  int rc, dev;
  DeviceState *st;
  if ((rc = current_device(&dev, &st)) != ATTN_OK) return rc;
  const void *all[4] = {acc_o, acc_lse, part_o, part_lse};
  for (const void *ptr : all)
    if (!is_device_memory_of(ptr, dev)) return ATTN_ERR_NOT_DEVICE_MEMORY;
  const int64_t want = (rows + 7) / 8;
  const int blocks = static_cast<int>(want < st->sm_count * 16 ? want : st->sm_count * 16);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t *po = static_cast<const uint16_t *>(part_o);
  if (d == 128)
    attn_b200::attn_merge_fold_kernel<128><<<blocks, 256, 0, s>>>(acc_o, acc_lse, po, part_lse, rows, first);
  else
    attn_b200::attn_merge_fold_kernel<64><<<blocks, 256, 0, s>>>(acc_o, acc_lse, po, part_lse, rows, first);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

int attn_merge_finish(const float *acc_o, const float *acc_lse, void *o, float *lse,
                      int64_t rows, int d, attn_stream_t stream) {
  if (rows < 0) return ATTN_ERR_INVALID_SIZE;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED_HEAD_DIM;
  if (rows == 0) return ATTN_OK;
  if (!acc_o || !acc_lse || !o || !lse) return ATTN_ERR_NULL_POINTER;
  if (!aligned(acc_o, 16) || !aligned(o, 16) || !aligned(acc_lse, 4) || !aligned(lse, 4))
    return ATTN_ERR_MISALIGNED;
  const size_t ob = static_cast<size_t>(rows) * d * 4, lb = static_cast<size_t>(rows) * 4;
  if (overlaps(o, ob / 2, acc_o, ob) || overlaps(o, ob / 2, acc_lse, lb) ||
      overlaps(lse, lb, acc_o, ob) || overlaps(lse, lb, o, ob / 2) ||
      (lse != acc_lse && overlaps(lse, lb, acc_lse, lb)))
    return ATTN_ERR_ALIAS;
  int rc, dev;
  DeviceState *st;
  if ((rc = current_device(&dev, &st)) != ATTN_OK) return rc;
  const void *all[4] = {acc_o, acc_lse, o, lse};
  for (const void *ptr : all)
    if (!is_device_memory_of(ptr, dev)) return ATTN_ERR_NOT_DEVICE_MEMORY;
  const int64_t want = (rows + 7) / 8;
  const int blocks = static_cast<int>(want < st->sm_count * 16 ? want : st->sm_count * 16);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint16_t *oo = static_cast<uint16_t *>(o);
  if (d == 128)
    attn_b200::attn_merge_finish_kernel<128><<<blocks, 256, 0, s>>>(acc_o, acc_lse, oo, lse, rows);
  else
    attn_b200::attn_merge_finish_kernel<64><<<blocks, 256, 0, s>>>(acc_o, acc_lse, oo, lse, rows);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

int attn_status(attn_stream_t stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ATTN_ERR_UNSUPPORTED_DEVICE;
  }
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  uint32_t *word;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    word = g_dev[dev].status;
  }
  if (!word) return ATTN_OK;
  uint32_t bits = 0;
  if (cudaMemcpy(&bits, word, sizeof bits, cudaMemcpyDeviceToHost) !=
      cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  if (bits == 0) return ATTN_OK;
  g_last_bits.store(bits);
  if (cudaMemset(word, 0, sizeof bits) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return status_bits_to_code(bits);
}

uint32_t attn_last_status_bits(void) { return g_last_bits.load(); }

int attn_selftest_exp2(const float *x, float *y, int n, int mode,
                       attn_stream_t stream) {
  if (n < 0) return ATTN_ERR_INVALID_SIZE;
  if (mode != 0 && mode != 1) return ATTN_ERR_INVALID_SCALE;
  if (n == 0) return ATTN_OK;
  if (!x || !y) return ATTN_ERR_NULL_POINTER;
  const int pairs = (n + 1) / 2;
  exp2_selftest_kernel<<<(pairs + 255) / 256, 256, 0,
                         reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n, mode);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

const char *attn_strerror(int code) {
  switch (code) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_NULL_POINTER: return "a required pointer is NULL";
    case ATTN_ERR_INVALID_SIZE: return "B, H or N negative or beyond the supported limits";
    case ATTN_ERR_UNSUPPORTED_HEAD_DIM: return "head dimension must be 64 or 128";
    case ATTN_ERR_MISALIGNED: return "q/k/v/o must be 16-byte aligned and lse 4-byte aligned";
    case ATTN_ERR_INVALID_SCALE: return "scale must be finite and > 0";
    case ATTN_ERR_ALIAS: return "o or lse overlaps an input or each other";
    case ATTN_ERR_UNSUPPORTED_DEVICE: return "no CUDA device, or the current device is not a B200 (compute capability 10.0)";
    case ATTN_ERR_CUDA: return "a CUDA runtime call or the kernel launch failed";
    case ATTN_ERR_TENSOR_MAP: return "TMA tensor-map encoding failed";
    case ATTN_ERR_NOT_DEVICE_MEMORY: return "a buffer is not device memory of the current device";
    case ATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case ATTN_ERR_NOALLOC_TOO_LARGE: return "problem needs more device scratch than the static ATTN_NOALLOC_SCRATCH_BYTES array of attn_fwd_host_noalloc";
    case ATTN_ERR_DEVICE_TIMEOUT: return "a pipeline wait in the kernel ran out of time; outputs are invalid";
    case ATTN_ERR_DEVICE_BOUNDS: return "an index check of the debug build failed; the access was skipped and outputs are invalid";
    default: return "unknown error code";
  }
}

void attn_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns ? ns : kDefaultTimeoutNs);
}

void attn_set_fault_injection(uint32_t flags) { g_inject.store(flags & 7u); }

}  // extern "C"

// ------------------------------------------------------------------------
// attn_fwd_host_noalloc: the host-buffer path with its device scratch in a
// static array instead of caller- or library-allocated memory.
// ------------------------------------------------------------------------
namespace {

// [0, 256): device status word of these calls; [256, end): q | k | v | o |
// lse staging, laid out as attn_fwd_host lays out its workspace.
static __device__ __align__(256) uint8_t g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];
constexpr size_t kNoallocStatusBytes = 256;

struct NoallocState {
  bool ready = false;
  uint8_t *base = nullptr;  // device address of g_noalloc_scratch
};
NoallocState g_noalloc[kMaxDevices];

// Current device checked to be a B200, without touching the lazily
// allocated status word of attn_fwd (so nothing is allocated here); looks up
// the scratch array's device address once per device.
int noalloc_device(int *dev_out, DeviceState **st_out, uint8_t **base_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ATTN_ERR_UNSUPPORTED_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState &st = g_dev[dev];
  if (!st.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_UNSUPPORTED_DEVICE;
    }
    st.probed = true;
    st.supported = (major == 10 && minor == 0);
    st.sm_count = sms;
  }
  if (!st.supported) return ATTN_ERR_UNSUPPORTED_DEVICE;
  NoallocState &na = g_noalloc[dev];
  if (!na.ready) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    na.base = static_cast<uint8_t *>(p);
    na.ready = true;
  }
  *dev_out = dev;
  *st_out = &st;
  *base_out = na.base;
  return ATTN_OK;
}

}  // namespace

extern "C" int attn_fwd_host_noalloc(const void *q, const void *k,
                                     const void *v, void *o, float *lse, int B,
                                     int H, int N, int d, int causal,
                                     float scale, attn_stream_t stream) {
  int rc = check_args(q, k, v, o, lse, B, H, N, d, scale, false);
  if (rc != ATTN_OK || B == 0 || H == 0 || N == 0) return rc;
  const size_t need = attn_fwd_host_workspace_bytes(B, H, N, d);
  if (need > ATTN_NOALLOC_SCRATCH_BYTES - kNoallocStatusBytes)
    return ATTN_ERR_NOALLOC_TOO_LARGE;

  int dev;
  DeviceState *st;
  uint8_t *base;
  if ((rc = noalloc_device(&dev, &st, &base)) != ATTN_OK) return rc;
  uint32_t *status = reinterpret_cast<uint32_t *>(base);
  uint8_t *ws = base + kNoallocStatusBytes;
  const size_t rows = static_cast<size_t>(B) * H * N;
  const size_t tb = rows * d * 2, tbr = round256(tb);
  void *dq = ws, *dk = ws + tbr, *dv = ws + 2 * tbr, *dout = ws + 3 * tbr;
  float *dl = reinterpret_cast<float *>(ws + 4 * tbr);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // The array keeps the previous call's contents: the status word must
  // start at zero; the staging area is fully overwritten below.
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess ||
      cudaMemcpyAsync(dq, q, tb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dk, k, tb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dv, v, tb, cudaMemcpyHostToDevice, s) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  EncodeTiledFn enc;
  if ((rc = get_encode_fn(&enc)) != ATTN_OK) return rc;
  const int bh = B * H;
  CUtensorMap maps[3];
  if ((rc = encode_map(enc, &maps[0], dq, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[1], dk, bh, N, d)) != ATTN_OK) return rc;
  if ((rc = encode_map(enc, &maps[2], dv, bh, N, d)) != ATTN_OK) return rc;
  FwdParams p;
  p.o = static_cast<uint16_t *>(dout);
  p.lse = dl;
  p.status = status;
  p.bh = bh;
  p.n = N;
  p.num_units = bh * ((N + 255) / 256);
  p.c_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.timeout_ns = g_timeout_ns.load();
  p.debug_flags = g_inject.load() & 5u;  // bits 0 and 2 concern this kernel
  if (d == 128)
    rc = causal ? launch<128, true>(*st, 0, maps, p, s)
                : launch<128, false>(*st, 1, maps, p, s);
  else
    rc = causal ? launch<64, true>(*st, 2, maps, p, s)
                : launch<64, false>(*st, 3, maps, p, s);
  if (rc != ATTN_OK) return rc;
  uint32_t bits = 0;
  if (cudaMemcpyAsync(o, dout, tb, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(lse, dl, rows * 4, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(&bits, status, sizeof bits, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  if (bits != 0) {
    g_last_bits.store(bits);
    return status_bits_to_code(bits);
  }
  return ATTN_OK;
}
