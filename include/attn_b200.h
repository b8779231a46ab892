/*
 * attn_b200.h -- C ABI of the B200 (sm_100a) exact attention forward pass.
 *
 * Operation (marketmaker.cc post "Apakah Konteks Sehari Penuh Mengalahkan
 * Konteks Sepuluh Menit? Perhatian Kilat dan Pertanyaan Panjang Urutan",
 * sections "Mengapa perhatian terikat pada memori" and "Algoritma Flash
 * Attention"; causal mask as in "Causal masking adalah tempat perdagangan
 * mendapat diskon" and "Integrasinya delapan baris"):
 *
 *   for every batch b < B and head h < H, with S = scale * Q K^T (N x N):
 *     S[i][j] = -inf when causal != 0 and j > i   (key j in query i's future)
 *     O   = softmax_rows(S) V                     (bf16 output, fp32 math)
 *     lse[i] = ln( sum_j exp(S[i][j]) )           (fp32; the saved softmax
 *                                                  statistics (m, l) of the
 *                                                  section "Backward pass",
 *                                                  folded into m + ln l)
 *
 * S is never written to memory: the kernel walks key/value tiles with the
 * online-softmax recurrence ("Pengulangan softmax online"), which is exact
 * up to rounding.
 *
 * Layouts.  q, k, v, o: contiguous row-major bf16 [B, H, N, d] (d innermost,
 * then the sequence, then heads, then batch) -- the (batch, heads, seq,
 * head_dim) layout of the post's SDPA call.  lse: contiguous fp32 [B, H, N].
 * Q and K/V have the same sequence length N (self-attention).
 *
 * Ownership.  The caller allocates and owns every buffer.  attn_fwd does not
 * allocate per call; the first call on a device allocates one 4-byte device
 * status word for that device, kept until process exit (so make the first
 * call outside any CUDA-graph capture).  o and lse must not overlap q, k, v
 * or each other.
 *
 * Concurrency.  Calls are asynchronous on `stream` (no host synchronisation).
 * Concurrent calls on different streams are safe; they share the device
 * status word, so a timeout reported by attn_status may belong to any of
 * them.
 *
 * Errors.  Every function returns 0 (ATTN_OK) or a positive code below.
 * Argument errors are detected before any CUDA call, so nothing is launched
 * and the CUDA context is untouched.  Device-side failures (a pipeline wait
 * that exceeded its time limit) are reported later by attn_status.
 */
#ifndef ATTN_B200_H_
#define ATTN_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle (cudaStream_t / CUstream); NULL = legacy
 * default stream. */
typedef struct CUstream_st *attn_stream_t;

enum {
  ATTN_OK = 0,
  ATTN_ERR_NULL_POINTER = 1,     /* a required pointer is NULL */
  ATTN_ERR_INVALID_SIZE = 2,     /* B, H or N negative or beyond the limits */
  ATTN_ERR_UNSUPPORTED_HEAD_DIM = 3, /* d is not 64 or 128 */
  ATTN_ERR_MISALIGNED = 4,       /* q/k/v/o not 16-byte or lse not 4-byte aligned */
  ATTN_ERR_INVALID_SCALE = 5,    /* scale not finite or not > 0 */
  ATTN_ERR_ALIAS = 6,            /* o or lse overlaps an input or each other */
  ATTN_ERR_UNSUPPORTED_DEVICE = 7, /* no CUDA device, or not compute 10.0 (B200) */
  ATTN_ERR_CUDA = 8,             /* a CUDA runtime call or the launch failed */
  ATTN_ERR_TENSOR_MAP = 9,       /* TMA descriptor encoding failed */
  ATTN_ERR_NOT_DEVICE_MEMORY = 10, /* q/k/v/o/lse not device memory of the
                                      current device */
  ATTN_ERR_WORKSPACE = 11,       /* attn_fwd_host workspace NULL or too small */
  ATTN_ERR_NOALLOC_TOO_LARGE = 12, /* attn_fwd_host_noalloc: problem needs more
                                      than ATTN_NOALLOC_SCRATCH_BYTES */
  ATTN_ERR_DEVICE_TIMEOUT = 16,  /* (attn_status) a pipeline wait in the
                                    kernel ran past its time limit; the kernel
                                    stopped early and its outputs are invalid */
  ATTN_ERR_DEVICE_BOUNDS = 17    /* (attn_status, debug build only) an index
                                    check in the kernel failed; the access was
                                    skipped and the outputs are invalid */
};

/* Size limits (inclusive).  N <= ATTN_MAX_SEQ; B * H <= ATTN_MAX_HEADS. */
#define ATTN_MAX_SEQ (1 << 24)
#define ATTN_MAX_HEADS (1 << 24)

/*
 * attn_fwd -- exact attention forward on device buffers.
 *
 *   q, k, v  device pointers, bf16 [B, H, N, d], 16-byte aligned.
 *   o        device pointer, bf16 [B, H, N, d], 16-byte aligned (output).
 *   lse      device pointer, fp32 [B, H, N], 4-byte aligned (output): natural
 *            log of each row's softmax denominator over the scaled, masked
 *            scores.
 *   B, H, N  batch, heads, sequence length; any of them 0 is a valid empty
 *            problem (nothing is launched, ATTN_OK).
 *   d        head dimension: 64 or 128.
 *   causal   nonzero: key j is hidden from query i when j > i (the diagonal
 *            stays visible, so no row is ever fully masked).
 *   scale    multiplier of Q K^T, finite and > 0 (1/sqrt(d) for the usual
 *            attention).
 *   stream   CUDA stream the work is queued on.
 *
 * The current CUDA device must be a B200 (compute capability 10.0) and all
 * pointers must be its device memory.  Returns ATTN_OK once the kernel is
 * queued; runtime timeouts surface through attn_status.
 */
int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
             int B, int H, int N, int d, int causal, float scale,
             attn_stream_t stream);

/*
 * attn_fwd_host -- the same operation on HOST buffers, end to end.
 *
 * Copies q, k, v from the host into `workspace`, runs the attn_fwd kernel on
 * the copies, and copies o and lse back into the host buffers.  Problems of
 * 32 MiB or more per tensor are split by heads into up to 8 chunks that
 * shrink towards the end (for 32 heads 6, 6, 6, 6, 4, 2, 1, 1), whose
 * copies in, kernels and copies out overlap on three library-owned streams
 * (created on the device's first call, kept until process exit; make that
 * first call outside any stream capture).  The whole call is ordered on
 * `stream`: it starts after work already queued there, and work queued
 * there afterwards starts after its last copy out.  Returns once queued; the
 * host outputs are valid after `stream` is synchronised.  For asynchronous,
 * overlapping copies the host buffers must be page-locked (cudaHostAlloc /
 * pinned); pageable buffers work but the copies then block the calling
 * thread.  Calls on one device enqueue one at a time (a library mutex).
 *
 *   workspace        device memory of at least attn_fwd_host_workspace_bytes
 *                    (B, H, N, d) bytes, 256-byte aligned, caller-owned.
 *   workspace_bytes  its size.
 * Other arguments as attn_fwd; q, k, v, o, lse are host pointers here.
 */
int attn_fwd_host(const void *q, const void *k, const void *v, void *o,
                  float *lse, int B, int H, int N, int d, int causal,
                  float scale, void *workspace, size_t workspace_bytes,
                  attn_stream_t stream);

/* Workspace bytes attn_fwd_host needs for this problem (0 on bad sizes):
 * q, k, v, o (each B*H*N*d*2 bytes) and lse (B*H*N*4 bytes), each rounded up
 * to 256 bytes. */
size_t attn_fwd_host_workspace_bytes(int B, int H, int N, int d);

/*
 * attn_status -- synchronise `stream`, then read and clear the current
 * device's status word.  Returns ATTN_OK, ATTN_ERR_DEVICE_TIMEOUT when a
 * kernel launched since the last call stopped on a wait time limit, or
 * ATTN_ERR_CUDA when the synchronisation itself failed.
 */
int attn_status(attn_stream_t stream);

/* Raw status bits of the last attn_status that reported a device error
 * (which pipeline role gave up), for diagnostics; 0 when none. */
uint32_t attn_last_status_bits(void);

/*
 * attn_bwd -- backward pass of attn_fwd (gradients of O with respect to
 * q, k, v), by recomputation: the marketmaker.cc post's section "Backward
 * pass: menghitung ulang, bukan menyimpan" keeps only the forward's output
 * and softmax statistics and recomputes the score tiles from Q and K.
 *
 *   q, k, v  the forward's inputs; o, lse its outputs (attn_fwd with the
 *            same B, H, N, d, causal, scale); dout = dL/dO.  All bf16
 *            [B, H, N, d] device buffers (16-byte aligned) except lse, fp32
 *            [B, H, N] (4-byte aligned).
 *   dq, dk, dv  outputs, bf16 [B, H, N, d] (16-byte aligned), written in
 *            full: dq = scale * dS k, dk = scale * dS^T q, dv = P^T dout with
 *            P = softmax(scale q k^T [mask]) and
 *            dS = P * (dout v^T - rowsum(dout * o)).
 *   workspace  device memory of at least attn_bwd_workspace_bytes(B, H, N)
 *            bytes, 256-byte aligned, caller-owned, scratch for this call.
 *
 * Queued on `stream` like attn_fwd; device timeouts surface in attn_status.
 * Outputs and workspace must not overlap any input or each other.
 */
int attn_bwd(const void *q, const void *k, const void *v, const void *o,
             const void *dout, const float *lse, void *dq, void *dk, void *dv,
             void *workspace, size_t workspace_bytes, int B, int H, int N,
             int d, int causal, float scale, attn_stream_t stream);

/* Workspace bytes attn_bwd needs (0 on bad sizes): two fp32 vectors of
 * B * H * (N rounded up to 128) entries, each rounded up to 256 bytes. */
size_t attn_bwd_workspace_bytes(int B, int H, int N);

/*
 * attn_selftest_exp2 -- test hook for the kernel's exponentials.  For n
 * device floats x, writes y[i] = 2^x[i] as the attention kernel evaluates
 * it: mode 0 = the FMA-pipe polynomial (Cody-Waite split + degree-3 minimax,
 * inputs below -125 clamped to -125), mode 1 = the ex2.approx instruction.
 * x and y are 4-byte aligned device pointers of the current device; the work
 * is queued on `stream`.  Returns ATTN_ERR_NULL_POINTER, ATTN_ERR_INVALID_SIZE
 * (n < 0) or ATTN_ERR_INVALID_SCALE (mode not 0 or 1) before any CUDA call.
 */
int attn_selftest_exp2(const float *x, float *y, int n, int mode,
                       attn_stream_t stream);

/* Size of the static device scratch array behind attn_fwd_host_noalloc:
 * 256 bytes of status followed by the q, k, v, o, lse staging area. */
#define ATTN_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * attn_fwd_host_noalloc -- attn_fwd_host for callers that cannot allocate
 * device memory.  The pages have no counterpart: this is a deployment
 * variant of the host-buffer entry point.
 *
 * Who needs it: a host program that holds only host buffers and has no
 * device allocator of its own -- or runs in a process whose device memory
 * belongs to another allocator that must not see untracked cudaMalloc
 * calls, or cannot afford the device-wide synchronisation cudaMalloc and
 * cudaFree may imply.  It allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.  Its device scratch is one static array of
 * ATTN_NOALLOC_SCRATCH_BYTES (32 MiB) compiled into this library; every GPU
 * that loads the library holds that array until the process exits.
 *
 * Arguments as attn_fwd_host (q, k, v, o, lse are host pointers; pinned
 * memory makes the copies asynchronous) minus the workspace.  The call
 * queues the copies in, the kernel and the copies out on `stream`, then
 * synchronises `stream` and returns: the outputs are in o and lse on return,
 * and the return value already includes the kernel's device status
 * (ATTN_ERR_DEVICE_TIMEOUT if a pipeline wait ran out), so attn_status is
 * not needed for it.
 *
 * Limits: attn_fwd_host_workspace_bytes(B, H, N, d) must not exceed
 * ATTN_NOALLOC_SCRATCH_BYTES - 256, else ATTN_ERR_NOALLOC_TOO_LARGE is
 * returned and nothing is queued (for d = 64, B*H*N up to about 65,000 rows;
 * for d = 128, about 32,700).
 *
 * Set-up: the first call on each device looks up the device address of the
 * scratch array (cudaGetSymbolAddress) with that device current.  Sharing:
 * every call on a device uses the same array, which keeps the last call's
 * contents (the status word is cleared at the start of every call).  Calls
 * that overlap on the GPU -- from different host threads or on different
 * streams -- race on the array and corrupt each other's results; serialise
 * them.
 */
int attn_fwd_host_noalloc(const void *q, const void *k, const void *v,
                          void *o, float *lse, int B, int H, int N, int d,
                          int causal, float scale, attn_stream_t stream);

/*
 * FP8 forward with incoherent processing -- the marketmaker.cc post's
 * section "FA3: Mekanika hopper", item 3: naive FP8 attention is spoiled by
 * outliers, so Q and K are rotated at random before block quantization,
 * spreading an outlier's magnitude over all coordinates.
 *
 * Definitions used by the three entries below:
 *   E4M3       OCP FP8 E4M3 ("fn": largest finite 448, no infinities),
 *              round to nearest even, saturating.
 *   rotation   x -> x diag(s) H for every row x of length d: s_t = -1 where
 *              bit t of the 128-bit sign mask (sign_lo bits 0-63, sign_hi
 *              bits 64-127) is set, else +1; H the unscaled d x d Sylvester
 *              Hadamard matrix, H[a][t] = (-1)^popcount(a & t), H H^T = d I.
 *              Computed in fp64 (exact for bf16 rows), then rounded to fp32.
 *   block      one scale per block of rows: the largest 2^e (e <= 126) with
 *              amax * 2^e <= 448, amax = the block's largest |value| after
 *              rotation; codes = E4M3(value * 2^e); stored scale = 2^-e (the
 *              dequantization multiplier).  Q and K: blocks of 128 rows
 *              (scales [B, H, ceil(N/128)]); V: one block per head (scales
 *              [B, H]).
 *   attention  O = softmax(scale_qk * Qhat Khat^T [causal mask]) Vhat on the
 *              dequantized operands (Qhat = codes * scale, ...), computed as
 *              the blocked online softmax in 128-key blocks with a running
 *              base m (log2 units) per row that moves to the block maximum
 *              only when that exceeds it by more than 4: P = 2^(x - m + 4)
 *              <= 256 is rounded to E4M3 for the P.V product (every
 *              probability down to 2^-10 of the row maximum is then an E4M3
 *              normal number), the row sum adds the unrounded P, and
 *              lse = ln(sum_j exp(scale_qk Qhat_i . Khat_j)) (fp32, natural
 *              log) -- independent of the rounding of P.
 * The three entries exist for head dimension d = 128 only (at d = 64 the
 * exponentials, not the tensor cores, bound the forward, and FP8 buys
 * nothing); other d give ATTN_ERR_UNSUPPORTED_HEAD_DIM.
 */

/*
 * attn_fp8_quantize -- block-quantize one bf16 tensor x [B, H, N, 128] to
 * E4M3 codes x8 [B, H, N, 128] (1 byte each) and fp32 scales.
 *   rotate     nonzero: rotate every row with the sign mask first (Q, K).
 *   per_head   0: one scale per 128-row tile, scales [B, H, ceil(N/128)];
 *              nonzero: one per head, scales [B, H], and tile_amax must
 *              point to B * H * ceil(N/128) floats of device scratch (the
 *              first of the two launches stores each tile's amax there).
 *              tile_amax may be NULL when per_head is 0.
 * x and x8 16-byte aligned, scales and tile_amax 4-byte aligned, all device
 * memory of the current device; x8, scales and tile_amax must not overlap x
 * or each other.  Queued on `stream`.
 */
int attn_fp8_quantize(const void *x, void *x8, float *scales, float *tile_amax,
                      int B, int H, int N, int d, int rotate, uint64_t sign_lo,
                      uint64_t sign_hi, int per_head, attn_stream_t stream);

/*
 * attn_fwd_fp8_quantized -- the FP8 attention on quantized operands.
 *   q8, k8, v8     E4M3 codes [B, H, N, 128], 16-byte aligned.
 *   q_scale, k_scale  fp32 [B, H, ceil(N/128)] per-tile scales;
 *   v_scale        fp32 [B, H] per-head scales.  Scales must be powers of
 *                  two (as attn_fp8_quantize writes them).
 *   scale          scale_qk of the definition above: the softmax scale of
 *                  the problem the codes encode (for rotated Q and K that is
 *                  the original scale / d, because H is unscaled).
 *   o, lse         outputs as attn_fwd's: bf16 [B, H, N, 128], fp32 [B, H, N].
 * Same launch, error and status behaviour as attn_fwd.
 */
int attn_fwd_fp8_quantized(const void *q8, const float *q_scale,
                           const void *k8, const float *k_scale,
                           const void *v8, const float *v_scale, void *o,
                           float *lse, int B, int H, int N, int d, int causal,
                           float scale, attn_stream_t stream);

/*
 * attn_fwd_fp8 -- the whole FP8 path from bf16 inputs: quantize Q and K
 * (rotated when `rotate` is nonzero, per 128-row tile) and V (per head)
 * into `workspace`, then attn_fwd_fp8_quantized with scale / d (rotated) or
 * scale (not rotated).  q, k, v, o, lse as attn_fwd (d = 128); workspace:
 * device memory of at least attn_fwd_fp8_workspace_bytes(B, H, N, d) bytes,
 * 256-byte aligned, caller-owned scratch for this call, not overlapping any
 * other argument.  Four kernels are queued on `stream` (two for V).
 */
int attn_fwd_fp8(const void *q, const void *k, const void *v, void *o,
                 float *lse, int B, int H, int N, int d, int causal,
                 float scale, int rotate, uint64_t sign_lo, uint64_t sign_hi,
                 void *workspace, size_t workspace_bytes, attn_stream_t stream);

/* Workspace bytes attn_fwd_fp8 needs (0 on bad sizes or d != 128): three
 * code tensors of B*H*N*d bytes and four fp32 vectors of scales and tile
 * maxima, each rounded up to 256 bytes. */
size_t attn_fwd_fp8_workspace_bytes(int B, int H, int N, int d);

/*
 * attn_fwd_fp8_host -- attn_fwd_fp8 on HOST buffers, end to end: the FP8
 * counterpart of attn_fwd_host.  q, k, v, o (bf16 [B, H, N, 128]) and lse
 * (fp32 [B, H, N]) are host memory, ideally page-locked; the bf16 inputs are
 * copied to the device, rotated and quantized there, attended with the FP8
 * kernel, and O and lse copied back.  Problems of 32 MiB or more per tensor
 * are split by heads into the same shrinking chunks as attn_fwd_host, whose
 * copies in, FP8 computation and copies out overlap on the library's three
 * streams; the result equals attn_fwd_fp8's bit for bit (the block scales
 * are per head and tile, so splitting by heads changes none of them).
 * workspace: device memory of at least attn_fwd_fp8_host_workspace_bytes
 * bytes, 256-byte aligned (bf16 staging of q, k, v, o, lse and the codes and
 * scales of one chunk).  Queued on `stream` like attn_fwd_host; the host
 * outputs are valid after `stream` is synchronised.  Errors as
 * attn_fwd_fp8, plus ATTN_ERR_WORKSPACE.
 */
int attn_fwd_fp8_host(const void *q, const void *k, const void *v, void *o, float *lse,
                      int B, int H, int N, int d, int causal, float scale, int rotate,
                      uint64_t sign_lo, uint64_t sign_hi, void *workspace,
                      size_t workspace_bytes, attn_stream_t stream);

/* Workspace bytes attn_fwd_fp8_host needs (0 on bad sizes). */
size_t attn_fwd_fp8_host_workspace_bytes(int B, int H, int N, int d);

/*
 * attn_decode -- split-KV decode attention: Nq new queries against Nk keys
 * per (batch, head), after the briefgpt.xyz summary page of FlashAttention-2
 * (arXiv 2307.08691), entry "LeanAttention" (the decode phase of long
 * contexts, computed in parallel over the key/value sequence).
 *
 *   q      bf16 [B, H, Nq, d], the queries of the last Nq positions;
 *   k, v   bf16 [B, H, Nk, d], the whole key/value sequence;
 *   o      bf16 [B, H, Nq, d]; lse fp32 [B, H, Nq] (natural log);
 *   O = softmax(scale q k^T [mask]) v exactly; with causal != 0 query i
 *   sees keys 0 .. Nk - Nq + i (the queries are the latest positions).
 * Limits: 1 <= Nq <= ATTN_DECODE_MAX_Q (Nq = 0 is a no-op), Nk >= 1,
 * Nq <= Nk when causal, d in {64, 128}, Nk <= ATTN_MAX_DECODE_KEYS.
 * q, k, v, o 16-byte aligned, lse 4-byte aligned, all device memory of the
 * current device.  workspace: at least attn_decode_workspace_bytes(...)
 * bytes, 256-byte aligned, caller-owned scratch for this call (partial
 * outputs of split heads and one counter per head, zeroed by the call).
 * Outputs and workspace must not overlap the inputs or each other.
 *
 * The key tiles of all heads are split into equal contiguous shares, one per
 * CTA; a head split over several CTAs is combined exactly by the CTA that
 * finishes its last share.  Two kernels (see attn_decode_kernel_for):
 *   - tensor cores, the default: one launch for all queries (S^T = K Q^T and
 *     O^T = V^T P^T with tcgen05, one CTA per SM), K/V read once.  P is
 *     rounded to bf16 for the P.V product, as in attn_fwd;
 *   - CUDA cores, when attn_set_decode_kernel(1) asks for it: two CTAs per
 *     SM, up to 4 queries per head and launch, more in groups of 4 by
 *     successive launches (each reading K/V again); P stays fp32.
 * Queued on `stream`; a wait that runs out of time shows in attn_status
 * (outputs are then invalid).
 */
#define ATTN_DECODE_MAX_Q 16
#define ATTN_MAX_DECODE_KEYS (1 << 26)
int attn_decode(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int H, int Nq, int Nk, int d, int causal, float scale,
                void *workspace, size_t workspace_bytes, attn_stream_t stream);

/* Workspace bytes attn_decode needs (0 on bad sizes): partial outputs and
 * log-sum-exps of Nq queries for B*H + 1024 parts, and B*H counters, each
 * rounded up to 256 bytes. */
size_t attn_decode_workspace_bytes(int B, int H, int Nq, int Nk, int d);

/* Test hook: cap the number of CTAs attn_decode launches (0 = two per SM
 * for the CUDA-core kernel, one per SM for the tensor-core one), so that
 * small problems can be split over many CTAs.  Process-wide. */
void attn_set_decode_max_ctas(int n);

/* Test hook: which decode kernel attn_decode runs, for launches made after
 * the call (process-wide): 1 = the CUDA-core kernel (groups of 4 queries),
 * 2 = the tensor-core kernel (one launch for all queries), anything else =
 * the library's choice (the default; currently the tensor-core kernel for
 * every Nq and d).  Both give the same result up to the bf16 rounding of P
 * in the tensor-core kernel. */
void attn_set_decode_kernel(int which);

/* The decode kernel attn_decode runs for Nq queries per head at head size d
 * under the current setting of attn_set_decode_kernel: 1 = CUDA cores,
 * 2 = tensor cores.  No CUDA calls. */
int attn_decode_kernel_for(int Nq, int d);

/*
 * attn_fwd_block_sparse -- attn_fwd restricted to the (query tile, key tile)
 * blocks a mask selects: the block-sparse extension of the tiled exact
 * algorithm (briefgpt.xyz summary page of FlashAttention-2, arXiv
 * 2307.08691, FlashAttention entry: the method "extends to block-sparse
 * attention"; the entry on sparse FlashAttention for key/query dropping).
 *
 *   S[i, j] = -inf when block_mask[i / 128][j / 128] == 0 (and, if causal,
 *             when j > i); O = softmax_rows(S) V; lse[i] = ln sum_j exp S[i, j].
 *   A row whose every score is masked gets O = 0 and lse = -inf (the softmax
 *   of an empty row is undefined; this is the reading taken).
 *
 * q, k, v, o, lse: as attn_fwd (device memory, [B, H, N, d] bf16 and
 * [B, H, N] fp32, the same alignment and aliasing rules).  block_mask: device
 * bytes, row-major [T, T] with T = ceil(N / 128), one byte per pair of a
 * 128-row query tile and a 128-key key tile, nonzero = computed; shared by
 * every head (mask_per_head = 0) or one [T, T] mask per head in [B, H] order
 * (mask_per_head != 0; B * H * T * T bytes).  Owned by the caller, only read.
 * Under the causal mask, blocks above the diagonal are never computed
 * whatever their mask byte.  Work is one query tile per CTA step over the
 * selected key tiles only, so time scales with the number of selected
 * blocks.  Errors as attn_fwd, plus ATTN_ERR_NULL_POINTER for a NULL mask
 * and ATTN_ERR_NOT_DEVICE_MEMORY for a mask outside the current device.
 * Asynchronous on `stream`.
 */
int attn_fwd_block_sparse(const void *q, const void *k, const void *v, void *o,
                          float *lse, int B, int H, int N, int d, int causal,
                          float scale, const uint8_t *block_mask,
                          int mask_per_head, attn_stream_t stream);

/*
 * Merging partial attention results -- the softmax statistics kept per row
 * (the marketmaker.cc post's section "Backward pass", folded into lse) make
 * attention over disjoint key sets exactly combinable:
 *     lse = log sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.
 * This is what sequence-sharded attention over several devices needs (the
 * briefgpt.xyz summary page of FlashAttention-2, arXiv 2307.08691, entry
 * "BurstAttention"): each device attends its queries to one shard of the
 * keys at a time and folds the result in.
 *
 * attn_merge_fold: fold one part (part_o bf16 [rows, d], part_lse fp32
 * [rows], as attn_fwd writes them) into the accumulator (acc_o fp32 [rows, d],
 * acc_lse fp32 [rows]); first != 0 initialises the accumulator from the part.
 * A row that sees no key in a part must have part_lse = -inf there.
 * attn_merge_finish: o = bf16(acc_o), lse = acc_lse (lse may equal acc_lse).
 * rows = B * H * N_queries; d in {64, 128}; acc_o, part_o, o 16-byte
 * aligned, the lse arrays 4-byte aligned, device memory of the current
 * device, outputs not overlapping inputs.  Queued on `stream`.
 */
/*
 * attn_fwd_merge -- attn_fwd with its result folded into an accumulator in
 * the kernel's epilogue (no separate merge pass, no bf16 rounding of parts):
 *   mode 1 (first): acc_o = O of this call (fp32), acc_lse = its lse;
 *   mode 2 (into):  (acc_o, acc_lse) = merge(accumulator, this call);
 *   mode 3 (last):  o (bf16), lse = merge(accumulator, this call); the
 *                   accumulator is only read.
 * acc_o fp32 [B, H, N, d] (16-byte aligned), acc_lse fp32 [B, H, N]; o and
 * lse as attn_fwd's, used by mode 3 only (may be NULL otherwise).  Every
 * call of a sequence of folds must cover the same queries (q is the same
 * shape; k, v are another disjoint part of the keys, same length N).
 */
int attn_fwd_merge(const void *q, const void *k, const void *v, float *acc_o,
                   float *acc_lse, void *o, float *lse, int B, int H, int N, int d,
                   int causal, float scale, int mode, attn_stream_t stream);

int attn_merge_fold(float *acc_o, float *acc_lse, const void *part_o,
                    const float *part_lse, int64_t rows, int d, int first,
                    attn_stream_t stream);
int attn_merge_finish(const float *acc_o, const float *acc_lse, void *o, float *lse,
                      int64_t rows, int d, attn_stream_t stream);

/* Human-readable text for an error code (static string, never NULL). */
const char *attn_strerror(int code);

/*
 * attn_set_wait_timeout_ns -- time limit of every pipeline wait inside the
 * kernel, for launches made after the call (process-wide).  0 restores the
 * default of 1e9 ns (one second).  A wait that runs out sets the device
 * status word, and the kernel drains its in-flight copies, frees its tensor
 * memory and exits.
 */
void attn_set_wait_timeout_ns(uint64_t ns);

/*
 * attn_set_fault_injection -- test hook.  Bit 0: in later attn_fwd launches
 * the first CTA's loader never issues its first Q-tile copy, so the MMA
 * warp's wait on it runs out after the wait time limit.  Bit 1: in later
 * attn_decode launches the first CTA's producer never issues its first K/V
 * tile, so the compute warps' wait runs out.  Either launch then ends with
 * ATTN_ERR_DEVICE_TIMEOUT in attn_status (outputs invalid) and the CUDA
 * context stays usable.  Bit 2, honoured only by the debug build
 * (libattn_b200_debug.so, compiled with ATTN_DEBUG_BOUNDS, whose kernels check
 * every global row index before they use it): in later attn_fwd launches the
 * first row that CTA 0 stores gets an index past the output; the check
 * catches it, the store is skipped and attn_status returns
 * ATTN_ERR_DEVICE_BOUNDS.  flags = 0 (the default) turns all off; other bits
 * are ignored.
 */
void attn_set_fault_injection(uint32_t flags);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H_ */
