/*
 * q4gsw.h - C ABI of the q4gsw 4-bit group-symmetric weight-quantized linear
 * layer for NVIDIA B200 (sm_100a).
 *
 * Sources of the definitions (three web pages):
 *   [P2] "[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward kernel (4-bit
 *        input-grad)", pytorch/executorch pull request #20943, PR description:
 *        the input gradient d_x[M,K] = d_out[M,N] @ dequant(W)[N,K] contracting
 *        over N; dequant(W[n,k]) = (code - 8) * scale; "Key changes": even-N
 *        code in the low nibble, odd-N code in the high nibble, [num_groups, N]
 *        scales, one prepack shared by forward and backward; "Constraints":
 *        N, K, group_size multiples of 4, fp32.
 *   [P3] "[ExecuTorch][WebGPU] Replace broad QKV fusion with BK64 kernel",
 *        pytorch/executorch pull request #21650, description of #21131: the
 *        Q/K/V projection triple fused over one packing of the constant
 *        weights and scales, scattered into three distinct outputs; outside the
 *        accepted shapes the ordinary routes run.
 *   [P1] "Upstream the Gemma 4 Vulkan support we carry on our ExecuTorch fork",
 *        software-mansion/react-native-executorch issue #1361: the fork's
 *        shader list (linear_q4gsw, linear_dq8ca_q4gsw,
 *        linear_fp32_scale_dq_acc, embedding_q4gsw) and the comment of Oct 20,
 *        2026: fp16 weight scales.
 *
 * Notation: M tokens, K input features, N output features, gs = group_size,
 * G = K / gs.  code[n,k] in 0..15, scale[g,n] fp16,
 *     w[n,k] = (code[n,k] - 8) * scale[k / gs, n].
 *
 * Conventions for every entry point
 *   - Every pointer argument is a DEVICE pointer on the current CUDA device,
 *     except where stated.  The caller allocates and owns every buffer; the
 *     library allocates no device memory when called (its one fixed array, the
 *     1 MiB of q4gsw_adapter_fwd_noalloc, is part of its device image).  Its
 *     state: per host thread, the
 *     route string (q4gsw_last_route) and the debug route pins
 *     (q4gsw_debug_pin_routes); per device, one status word shared by every
 *     stream and thread (see q4gsw_device_error_check) and caches of kernel
 *     attributes and occupancy, filled on first use.
 *   - Dense operands are contiguous row-major.  fp16 values are passed as
 *     uint16_t bit patterns; outputs are fp32.
 *   - Device pointers must be 16-byte aligned (Q4GSW_ERR_ALIGN otherwise).
 *   - Calls enqueue work on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and return without waiting, except q4gsw_prepack (see there).
 *   - Arguments are checked on the host before anything is enqueued; on an
 *     error nothing is enqueued and outputs are untouched.  A launch failure
 *     reported by the CUDA runtime returns Q4GSW_ERR_CUDA.
 *   - No CPU fallback exists: every result is computed by this library's
 *     CUDA kernels.  Results are deterministic: every reduction (warp slices,
 *     split-K CTAs of a cluster) runs in a fixed order, so a call repeated on
 *     the same inputs and route returns the same bits.  Calls may be made from several host threads at once
 *     (first-use caches are filled under std::call_once or atomics).
 *   - The compute calls launch with programmatic dependent launch: a call may
 *     start while the previous kernel on `stream` is still finishing.  It waits
 *     for that kernel before reading activations or writing outputs, but the
 *     packed weight is treated as a constant and may be read earlier.  So a
 *     packed blob must not be written by the kernel enqueued immediately before
 *     a call that reads it (q4gsw_prepack returns only after its own work is
 *     done, so a blob it produced is always safe).
 *   - Shapes accepted: N > 0, N % 8 == 0; K > 0, K % 64 == 0; gs a power of
 *     two with 16 <= gs <= K (so K % gs == 0).  [P2]'s own constraints
 *     (multiples of 4) are a superset; the tighter ones come from the packed
 *     layout (64-byte blocks) and from 16-byte TMA strides.  M == 0 is an empty
 *     batch: nothing is enqueued and Q4GSW_OK is returned.
 */
#ifndef Q4GSW_H
#define Q4GSW_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define Q4GSW_API __attribute__((visibility("default")))
#else
#define Q4GSW_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *q4gsw_stream_t;   /* same type as cudaStream_t */

typedef enum {
  Q4GSW_OK = 0,
  Q4GSW_ERR_NULL = 1,         /* a required pointer is NULL */
  Q4GSW_ERR_SHAPE = 2,        /* negative or zero sizes, [P2] multiple-of-4 rule, Q/K/V split mismatch */
  Q4GSW_ERR_ALIGN = 3,        /* pointer not 16-byte aligned, N % 8 or K % 64 != 0 */
  Q4GSW_ERR_UNSUPPORTED = 4,  /* group size not a power of two in [16, K] */
  Q4GSW_ERR_CODE_RANGE = 5,   /* q4gsw_prepack saw a code > 15 */
  Q4GSW_ERR_CUDA = 6,         /* the CUDA runtime reported an error */
  Q4GSW_ERR_SIZE = 7,         /* a byte count passed in is too small */
  Q4GSW_ERR_TIMEOUT = 8,      /* a kernel's bounded wait ran out (q4gsw_device_error_check) */
  Q4GSW_ERR_INDEX = 9         /* q4gsw_embedding saw an index outside [0, N) (q4gsw_device_error_check) */
} q4gsw_status;

/* Version of the packed-weight byte layout written by q4gsw_prepack. */
Q4GSW_API int q4gsw_layout_version(void);

/*
 * Bytes of the packed weight for (N, K, gs); 0 if the shape is not accepted.
 * Layout version 1 (all offsets from the start of the blob):
 *   codes   [0, N/2*K): for pair p = n/2 and column k, the byte
 *           code[2p,k] | code[2p+1,k] << 4  ([P2] nibble rule) at
 *           p*K + 64*(k/64) + 4*(4*t + i) + slot[e],  where k%64 = 16 i + 4 t + e
 *           and slot = {0, 2, 1, 3}.
 *   scales  at round_up(N/2*K, 256): fp16 [G][N] row-major ([P2] "[num_groups, N]").
 *   trailer at round_up(scales end, 256), 64 bytes of little-endian uint32:
 *           "Q4GS", version, N, K, gs, range flag, then zeros.
 */
Q4GSW_API size_t q4gsw_packed_bytes(int N, int K, int group_size);

/*
 * One-time packer ([P2] "Key changes": the prepack shared by forward and
 * backward; [P3]: the constant weights and scales are packed once).
 *   codes   uint8 [N, K], one code per byte, each in 0..15
 *   scales  fp16  [K/gs, N]
 *   packed  output, packed_bytes >= q4gsw_packed_bytes(N, K, gs)
 * Writes the whole blob (codes, scales, trailer; padding zeroed).  It then
 * waits for `stream` once, to read the range flag back: a code above 15
 * returns Q4GSW_ERR_CODE_RANGE (the blob content is then unspecified).
 */
Q4GSW_API q4gsw_status q4gsw_prepack(const uint8_t *codes, const uint16_t *scales,
                           int N, int K, int group_size,
                           void *packed, size_t packed_bytes,
                           q4gsw_stream_t stream);

/*
 * Forward: y[m,n] = sum_k x[m,k] * w[n,k], fp32 accumulation.
 *   packed  a blob from q4gsw_prepack for the same (N, K, gs)
 *   x       fp16 [M, K];   y  fp32 [M, N] (overwritten)
 * Route (q4gsw_last_route()): M <= 16 a tensor-core GEMV over the streamed
 * packed weight; 16 < M <= 512 a tcgen05 GEMM whose weight tile is
 * dequantised into tensor memory; larger M a tcgen05 GEMM that dequantises
 * into shared memory.
 */
Q4GSW_API q4gsw_status q4gsw_linear_fwd(const void *packed, int N, int K, int group_size,
                              const uint16_t *x, int M, float *y,
                              q4gsw_stream_t stream);

/*
 * Input gradient of the frozen base ([P2]):
 *   d_x[m,k] = sum_n d_out[m,n] * w[n,k]   (contracts over N)
 *   d_out fp16 [M, N];   d_x  fp32 [M, K] (overwritten)
 * Reads the same packed blob as the forward (no re-pack, [P2]).
 */
Q4GSW_API q4gsw_status q4gsw_linear_bwd_input(const void *packed, int N, int K, int group_size,
                                    const uint16_t *d_out, int M, float *d_x,
                                    q4gsw_stream_t stream);

/*
 * Fused Q/K/V forward ([P3]).  packed_qkv is q4gsw_prepack of the
 * row-concatenated codes [Nq+Nk+Nv, K] and scales [G, Nq+Nk+Nv].
 *   y_q fp32 [M, Nq], y_k fp32 [M, Nk], y_v fp32 [M, Nv]: three distinct buffers.
 * Nq, Nk, Nv > 0 and multiples of 8.
 */
Q4GSW_API q4gsw_status q4gsw_qkv_fwd(const void *packed_qkv, int Nq, int Nk, int Nv,
                           int K, int group_size,
                           const uint16_t *x, int M,
                           float *y_q, float *y_k, float *y_v,
                           q4gsw_stream_t stream);

/*
 * Embedding rows gathered from a packed q4gsw weight used as a table of N
 * rows of K features ("[ExecuTorch][WebGPU] Replace broad QKV fusion with
 * BK64 kernel", description of #21483: the Q4 embedding reads the linear
 * weight's nibble layout, is_linear_weight):
 *   out[t, k] = (code[idx[t], k] - 8) * s[k / gs, idx[t]]   for t < T, k < K,
 * each element the exact fp32 product (as q4gsw_dequant's w32).
 *   packed   a blob from q4gsw_prepack for (N, K, gs)
 *   indices  int32 [T] on the device, each in [0, N)
 *   out      fp32 [T, K] (overwritten)
 * T = 0 enqueues nothing.  An index outside [0, N) cannot be seen on the host:
 * its row is written as zeros and q4gsw_device_error_check then returns
 * Q4GSW_ERR_INDEX.
 */
Q4GSW_API q4gsw_status q4gsw_embedding(const void *packed, int N, int K, int group_size,
                             const int32_t *indices, int T, float *out,
                             q4gsw_stream_t stream);

/* ------------------------------------------------------------------------
 * fp32-scale variant (packed layout version 2)
 *
 * "Upstream the Gemma 4 Vulkan support we carry on our ExecuTorch fork",
 * issue #1361: the fork carries an fp32-scale dequantise-and-accumulate shader
 * helper (linear_fp32_scale_dq_acc) beside the fp16-scale q4gsw path; the
 * Oct 20 comment reports no measurable accuracy gain from it.  The pages name
 * it only; this library's reading:
 *   - layout version 2 = the version 1 codes region unchanged, the scales as
 *     fp32 [G][N] (4 bytes each) at the same 256-byte-aligned offset, then the
 *     64-byte trailer with version word 2;
 *   - the dequantised weight is w32[n,k] = fp32_RNE((code[n,k] - 8) * s32[k/gs, n]),
 *     one rounding (the product of a 4-bit integer and a 24-bit significand
 *     needs up to 27 bits);
 *   - the tensor-core GEMMs and the input-gradient GEMVs take fp16_RNE(w32) as
 *     their operand and accumulate in fp32; the forward GEMVs (M <= 16)
 *     multiply the fp32 partial sum of each group by s32 in fp32, so they never
 *     round the weight;
 *   - every output is fp32 and satisfies the same bound as the fp16-scale path.
 * The functions below take the same arguments, checks and routes as their
 * fp16-scale counterparts; a version-1 blob must not be passed to them, nor a
 * version-2 blob to the fp16-scale functions (the blob's trailer records its
 * version; the compute calls do not read it).
 * ---------------------------------------------------------------------- */

/* Bytes of a version-2 blob for (N, K, gs); 0 if the shape is not accepted. */
Q4GSW_API size_t q4gsw_packed_bytes_f32s(int N, int K, int group_size);

/* One-time packer for fp32 scales: codes uint8 [N, K] (0..15), scales fp32
 * [K/gs, N] -> version-2 blob.  Same checks, single wait and range-flag
 * behaviour as q4gsw_prepack. */
Q4GSW_API q4gsw_status q4gsw_prepack_f32s(const uint8_t *codes, const float *scales,
                                int N, int K, int group_size,
                                void *packed, size_t packed_bytes,
                                q4gsw_stream_t stream);

/* Forward, input gradient and fused Q/K/V forward on a version-2 blob. */
Q4GSW_API q4gsw_status q4gsw_linear_fwd_f32s(const void *packed, int N, int K, int group_size,
                                   const uint16_t *x, int M, float *y,
                                   q4gsw_stream_t stream);
Q4GSW_API q4gsw_status q4gsw_linear_bwd_input_f32s(const void *packed, int N, int K, int group_size,
                                         const uint16_t *d_out, int M, float *d_x,
                                         q4gsw_stream_t stream);
Q4GSW_API q4gsw_status q4gsw_qkv_fwd_f32s(const void *packed_qkv, int Nq, int Nk, int Nv,
                                int K, int group_size,
                                const uint16_t *x, int M,
                                float *y_q, float *y_k, float *y_v,
                                q4gsw_stream_t stream);

/* Embedding rows from a version-2 blob: out[t, k] = w32[idx[t], k]. */
Q4GSW_API q4gsw_status q4gsw_embedding_f32s(const void *packed, int N, int K, int group_size,
                                  const int32_t *indices, int T, float *out,
                                  q4gsw_stream_t stream);

/* Debug export: w32 and w16 = fp16_RNE(w32) of a version-2 blob. */
Q4GSW_API q4gsw_status q4gsw_dequant_f32s(const void *packed, int N, int K, int group_size,
                                float *w32, uint16_t *w16, q4gsw_stream_t stream);

/* ------------------------------------------------------------------------
 * Frozen-base low-rank adapter step
 *
 * "[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward kernel (4-bit
 * input-grad)", PR description: the input gradient of the frozen 4-bit base
 * exists for on-device adapter training.  The page does not define the
 * adapter; this library's reading is a rank-r low-rank adapter beside the
 * frozen q4gsw base, with no scaling factor (fold one into B):
 *   forward         y   = x dequant(W)^T + (x A^T) B^T
 *   input gradient  d_x = d_out dequant(W) + (d_out B) A    (its adjoint)
 *   a  fp16 [r, K] row-major,  b  fp16 [N, r] row-major,  8 <= r <= 64, r % 8 == 0
 * Two launches on `stream`: the intermediate u = x A^T (or v = d_out B) is
 * accumulated in fp32, rounded to fp16 and written to `workspace` as rows of
 * 64 halves; then the tensor-memory GEMM of the base adds u B^T (or v A) to
 * its fp32 accumulator as one more 64-deep contraction stage, so the output
 * is written once.  Every token count takes the tensor-memory GEMM route.
 * Error bound per output element: 4e-3 * (sum |x||w| + sum_j (sum_k |x||A_jk|) |B_nj|)
 * (the second term covers the fp16 rounding of the intermediate, which must
 * stay within the fp16 range).
 *   workspace  device, at least q4gsw_adapter_workspace_bytes(M, r) bytes,
 *              owned by the caller, overwritten; calls that share one
 *              workspace must be ordered on the GPU.
 * Only layout-version-1 blobs (fp16 scales).  Same checks and statuses as
 * q4gsw_linear_fwd, plus Q4GSW_ERR_SHAPE for a rank outside the rule and
 * Q4GSW_ERR_SIZE for a workspace that is too small.
 * ---------------------------------------------------------------------- */

/* Workspace bytes of one adapter call (M * 128); 0 for a rank outside the rule. */
Q4GSW_API size_t q4gsw_adapter_workspace_bytes(int M, int r);

Q4GSW_API q4gsw_status q4gsw_adapter_fwd(const void *packed, int N, int K, int group_size,
                               const uint16_t *a, const uint16_t *b, int r,
                               const uint16_t *x, int M, float *y,
                               void *workspace, size_t workspace_bytes,
                               q4gsw_stream_t stream);

Q4GSW_API q4gsw_status q4gsw_adapter_bwd_input(const void *packed, int N, int K, int group_size,
                                     const uint16_t *a, const uint16_t *b, int r,
                                     const uint16_t *d_out, int M, float *d_x,
                                     void *workspace, size_t workspace_bytes,
                                     q4gsw_stream_t stream);

/*
 * q4gsw_adapter_fwd without a workspace argument: the same result, with the
 * intermediate kept in a fixed scratch array inside this library instead of
 * memory the caller allocates.  (The web pages describe no such call; it is
 * this library's own addition.)
 *
 * For callers that cannot allocate device memory when they make the call:
 * code on a latency-critical path where cudaMalloc (which may synchronise the
 * whole device) is not acceptable, plugins hosted by a runtime that owns all
 * device memory and forbids allocations of their own, or programs whose device
 * memory is fixed up front.  The call itself allocates nothing: no cudaMalloc,
 * cudaFree or allocating library routine.  The caller still passes the inputs
 * and the output y.
 *
 * Limit: M <= 8192 tokens (the array holds 1 MiB = 8192 rows of 64 halves);
 * a larger M returns Q4GSW_ERR_SIZE before anything is enqueued.  Every GPU
 * that loads the library holds that 1 MiB until the process exits.
 * Set-up: the first call on a device looks up the array's address on that
 * device (cudaGetSymbolAddress), once; make that first call before any stream
 * capture.  A failed look-up returns Q4GSW_ERR_CUDA.
 * Sharing: all calls on a device use the same array, and it keeps the last
 * call's contents (nothing read by a call depends on them: each call writes
 * every byte it reads).  Calls whose work overlaps on the GPU (different
 * streams, or threads without ordering) race on the array and give wrong
 * results; order them on one stream or with events.
 * Other arguments, checks and statuses as q4gsw_adapter_fwd.
 */
Q4GSW_API q4gsw_status q4gsw_adapter_fwd_noalloc(const void *packed, int N, int K, int group_size,
                                       const uint16_t *a, const uint16_t *b, int r,
                                       const uint16_t *x, int M, float *y,
                                       q4gsw_stream_t stream);

/* ------------------------------------------------------------------------
 * linear_dq8ca_q4gsw: int8 dynamically quantised activations x q4gsw weight
 *
 * "Upstream the Gemma 4 Vulkan support we carry on our ExecuTorch fork",
 * issue #1361: the fork's shader list carries linear_dq8ca_q4gsw beside
 * linear_q4gsw; the page gives only the name.  This library's reading
 * (asymmetric per-token int8 activations, every step an IEEE fp32 operation
 * rounding to nearest even):
 *   lo = min(0, min_k x[m,k]),  hi = max(0, max_k x[m,k]),
 *   a_s[m] = (hi - lo) / 255  (1 when hi == lo),
 *   a_z[m] = clamp(rint(-128 - lo / a_s), -128, 127),
 *   q[m,k] = clamp(rint(x[m,k] / a_s) + a_z, -128, 127),
 *   y[m,n] = a_s[m] * sum_g s[g,n] * sum_{k in g} (q[m,k] - a_z[m]) * (code[n,k] - 8),
 * the inner sums exact (int8 tensor-core MMAs into int32), the outer ones fp32.
 * Error bound per element: 4e-3 * a_s * sum_g |s| * sum |q - a_z| |code - 8|
 * (relative to the quantised activations, which this call defines).
 *
 * Workspace (device, caller-owned, q4gsw_dq8ca_workspace_bytes(M, K) bytes):
 *   q    int8 [M][K] at 0, in the packed codes' order: inside each 64-column
 *        block the 16 bytes at 16 t (t = 0..3) hold columns 4 t + 16 i +
 *        (0, 2, 1, 3) for i = 0..3;
 *   a_s  fp32 [M]  at round_up(M*K, 256);
 *   a_z  int32 [M] at that + round_up(4*M, 256).
 * Two launches on `stream` (quantise, then the product); calls that share a
 * workspace must be ordered on the GPU.  gs must lie in [32, 65536]
 * (Q4GSW_ERR_UNSUPPORTED otherwise); other checks as q4gsw_linear_fwd, plus
 * Q4GSW_ERR_SIZE for a workspace that is too small.  Layout-version-1 blobs.
 * ---------------------------------------------------------------------- */
Q4GSW_API size_t q4gsw_dq8ca_workspace_bytes(int M, int K);
Q4GSW_API q4gsw_status q4gsw_linear_dq8ca_fwd(const void *packed, int N, int K, int group_size,
                                    const uint16_t *x, int M, float *y,
                                    void *workspace, size_t workspace_bytes,
                                    q4gsw_stream_t stream);
/* The quantiser alone (the first launch of q4gsw_linear_dq8ca_fwd), for tests
 * and for callers that reuse the quantised activations. */
Q4GSW_API q4gsw_status q4gsw_dq8ca_quantize(const uint16_t *x, int M, int K,
                                  void *workspace, size_t workspace_bytes,
                                  q4gsw_stream_t stream);

/*
 * Kernel health check.  Every wait inside this library's kernels is bounded
 * (one second of wall-clock time); a wait that runs out makes its kernel stop
 * early, leaving its outputs partly or wholly unwritten, and record the event
 * in the device's status word instead of hanging.  The word is one per device,
 * shared by every stream and host thread.  This call swaps it with zero in one
 * atomic operation, ordered after the work already enqueued on `stream`, then
 * waits for `stream`: events recorded later (by kernels of other streams) stay
 * in the word for the next check.  Q4GSW_ERR_TIMEOUT means the outputs of the
 * calls on this device since the previous check cannot be trusted;
 * Q4GSW_ERR_INDEX that an embedding index was out of range (a timeout takes
 * precedence).  Returns Q4GSW_OK otherwise.
 */
Q4GSW_API q4gsw_status q4gsw_device_error_check(q4gsw_stream_t stream);

/* Debug export: codes uint8 [N, K] back out of a packed blob. */
Q4GSW_API q4gsw_status q4gsw_unpack(const void *packed, int N, int K, int group_size,
                          uint8_t *codes, q4gsw_stream_t stream);

/*
 * Debug export: the dequantised weight [N, K] as the kernels see it.
 *   w32  fp32, (code - 8) * scale computed exactly (may be NULL)
 *   w16  fp16 bits, the tensor-core operand fp16_RNE((code - 8) * scale)
 *        (may be NULL; at least one of w32 / w16 must be given)
 */
Q4GSW_API q4gsw_status q4gsw_dequant(const void *packed, int N, int K, int group_size,
                           float *w32, uint16_t *w16, q4gsw_stream_t stream);

/*
 * Debug export (tests and tuning): pins the kernel route of the calls this
 * host thread makes from now on.
 *   gemv  calls with M <= 16:  0 automatic, 1 register-fed GEMV, 2 TMA-ring GEMV,
 *         3 TMA-ring GEMV whose forward stages the activations in the ring too
 *         (the input gradient has no TMA-ring/register choice other than these two)
 *   gemm  calls with M > 16:   0 automatic, 1 tensor-memory GEMM, 2 shared-memory
 *         GEMM (accumulators per CTA chosen), 3 shared-memory GEMM with one
 *         128-token accumulator, 4 with two
 * Every pinned route computes the same function (within the output bound).
 * Values outside these ranges return Q4GSW_ERR_SHAPE and change nothing.
 */
Q4GSW_API q4gsw_status q4gsw_debug_pin_routes(int gemv, int gemm);

/*
 * Debug export (test of the failure path, no fault involved): enqueues one
 * thread block whose single waiting thread waits, through the same bounded wait
 * the compute kernels use, on a barrier that nothing completes.  After
 * limit_us microseconds (1 .. 1000000) the wait gives up, records a time-out
 * in the device status word and the kernel returns, so the following
 * q4gsw_device_error_check returns Q4GSW_ERR_TIMEOUT.  Other limits return
 * Q4GSW_ERR_SHAPE.
 */
Q4GSW_API q4gsw_status q4gsw_debug_wait_timeout(unsigned int limit_us, q4gsw_stream_t stream);

/* Thread-local description of the kernel route the last call on this thread
 * enqueued (for example "gemv_fwd nt=1 splitk=8"); never NULL. */
Q4GSW_API const char *q4gsw_last_route(void);

/* Static text for a status code; never NULL. */
Q4GSW_API const char *q4gsw_status_str(q4gsw_status status);

#ifdef __cplusplus
}
#endif

#endif /* Q4GSW_H */
