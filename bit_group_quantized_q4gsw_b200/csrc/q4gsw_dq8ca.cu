// q4gsw_dq8ca.cu - int8 dynamically quantised activations times the q4gsw
// weight (linear_dq8ca_q4gsw of the shader list in "Upstream the Gemma 4
// Vulkan support we carry on our ExecuTorch fork", issue #1361; the page gives
// only the name).  Reading:
//   per token m:  lo = min(0, min_k x), hi = max(0, max_k x),
//                 a_s = (hi - lo) / 255 (1 when hi == lo),
//                 a_z = clamp(rint(-128 - lo / a_s), -128, 127),
//                 q[k] = clamp(rint(x[k] / a_s) + a_z, -128, 127)   (fp32, ties to even)
//   y[m, n] = a_s[m] sum_g s[g, n] sum_{k in g} (q[m, k] - a_z[m]) (code[n, k] - 8).
//
// This file holds the quantiser: one CTA per token writes q (int8, in the
// packed codes' order: inside each 64-column block the 16 bytes at 16 t hold
// columns 4 t + 16 i + (0, 2, 1, 3), i = 0..3, so that one 16-byte load gives a
// lane its operand of a 64-column block), a_s and a_z into the caller's
// workspace.  The product streams the weight through a TMA ring
// (q4gsw_dq8ca_tma.cuh).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "q4gsw_common.cuh"
#include "q4gsw_internal.h"

namespace q4gsw {
namespace dq {

constexpr int kQThreads = 1024;
constexpr int kQVec = 4;   // 16-byte vectors a thread keeps in registers (K <= 32768 in one pass)

// Workspace map for M tokens of K features (offsets in bytes).
__host__ __device__ inline size_t off_as(int M, int K) { return round_up((size_t)M * K, 256); }
__host__ __device__ inline size_t off_az(int M, int K) { return off_as(M, K) + round_up((size_t)4 * M, 256); }
__host__ __device__ inline size_t ws_bytes(int M, int K) { return off_az(M, K) + round_up((size_t)4 * M, 256); }

// q of one value: rint of the correctly rounded quotient v / a_s, plus a_z,
// clamped.  The quotient is taken as v times the rounded reciprocal inv of a_s;
// for |v / a_s| <= 256 that product lies within 2^-14 of the correctly rounded
// quotient (three roundings of at most 2^-24 relative each), so wherever it
// is farther than 1e-4 from a half-integer both round to the same integer, and
// only near a tie is the quotient divided out exactly.
__device__ __forceinline__ uint32_t quant_byte(float v, float as, float inv, int az) {
  float r = v * inv;
  if (fabsf(fabsf(r - rintf(r)) - 0.5f) < 1e-4f) r = __fdiv_rn(v, as);
  int qv = (int)rintf(r) + az;
  qv = qv < -128 ? -128 : qv > 127 ? 127 : qv;
  return (uint32_t)(qv & 0xFF);
}

// four consecutive values -> one word in the packed codes' byte order (+0, +2, +1, +3)
__device__ __forceinline__ uint32_t quant_word(__half2 a, __half2 b, float as, float inv, int az) {
  const float2 fa = __half22float2(a), fb = __half22float2(b);
  return quant_byte(fa.x, as, inv, az) | quant_byte(fb.x, as, inv, az) << 8 | quant_byte(fa.y, as, inv, az) << 16 |
         quant_byte(fb.y, as, inv, az) << 24;
}

__device__ __forceinline__ void range_of(const uint4& v, float& lo, float& hi) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(h[e]);
    lo = fminf(lo, fminf(f.x, f.y));
    hi = fmaxf(hi, fmaxf(f.x, f.y));
  }
}

// columns 8 i .. 8 i + 7 of the row -> their q bytes: block i / 8, 16-column
// step (i % 8) / 2, lanes t = 2 (i % 2) and 2 (i % 2) + 1 of that step
__device__ __forceinline__ void store_q(uint8_t* qrow, int i, const uint4& v, float as, float inv, int az) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  uint8_t* dst = qrow + 64 * (i >> 3) + 32 * (i & 1) + 4 * ((i & 7) >> 1);
  *reinterpret_cast<uint32_t*>(dst) = quant_word(h[0], h[1], as, inv, az);
  *reinterpret_cast<uint32_t*>(dst + 16) = quant_word(h[2], h[3], as, inv, az);
}

// One CTA per token: the row's 16-byte vectors stay in registers between the
// min/max reduction and the quantisation (rows past 32768 columns reload the rest).
__global__ void __launch_bounds__(kQThreads)
q4gsw_dq8ca_quantize_kernel(const __half* __restrict__ x, uint8_t* __restrict__ ws, int M, int K) {
  __shared__ float s_lo[kQThreads / 32], s_hi[kQThreads / 32];
  __shared__ float s_as, s_inv;
  __shared__ int s_az;
  griddep_launch_dependents();
  griddep_wait();   // x may come from the previous kernel of the stream
  const int m = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)m * K);
  const int V = K >> 3;
  uint4 v[kQVec];
#pragma unroll
  for (int u = 0; u < kQVec; ++u) {
    const int i = threadIdx.x + u * kQThreads;
    v[u] = i < V ? row[i] : make_uint4(0u, 0u, 0u, 0u);   // zeros: the range holds 0 anyway
  }
  float lo = 0.f, hi = 0.f;   // the range always holds 0
#pragma unroll
  for (int u = 0; u < kQVec; ++u) range_of(v[u], lo, hi);
  for (int i = threadIdx.x + kQVec * kQThreads; i < V; i += kQThreads) range_of(row[i], lo, hi);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if ((threadIdx.x & 31) == 0) {
    s_lo[threadIdx.x >> 5] = lo;
    s_hi[threadIdx.x >> 5] = hi;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    lo = s_lo[threadIdx.x];
    hi = s_hi[threadIdx.x];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (threadIdx.x == 0) {
      const float as = hi == lo ? 1.f : __fdiv_rn(__fsub_rn(hi, lo), 255.f);
      float z = rintf(__fsub_rn(-128.f, __fdiv_rn(lo, as)));
      z = fminf(127.f, fmaxf(-128.f, z));
      s_as = as;
      s_inv = __fdiv_rn(1.f, as);
      s_az = (int)z;
      reinterpret_cast<float*>(ws + off_as(M, K))[m] = as;
      reinterpret_cast<int*>(ws + off_az(M, K))[m] = (int)z;
    }
  }
  __syncthreads();
  const float as = s_as, inv = s_inv;
  const int az = s_az;
  uint8_t* qrow = ws + (size_t)m * K;
#pragma unroll
  for (int u = 0; u < kQVec; ++u) {
    const int i = threadIdx.x + u * kQThreads;
    if (i < V) store_q(qrow, i, v[u], as, inv, az);
  }
  for (int i = threadIdx.x + kQVec * kQThreads; i < V; i += kQThreads) store_q(qrow, i, row[i], as, inv, az);
}

}  // namespace dq

size_t dq8ca_workspace_bytes(int M, int K) { return dq::ws_bytes(M, K); }
size_t dq8ca_scale_offset(int M, int K) { return dq::off_as(M, K); }
size_t dq8ca_zero_offset(int M, int K) { return dq::off_az(M, K); }

cudaError_t launch_dq8ca_quantize(const uint16_t* x, int M, int K, void* workspace, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M, 1, 1);
  cfg.blockDim = dim3(dq::kQThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dq::q4gsw_dq8ca_quantize_kernel, reinterpret_cast<const __half*>(x),
                            static_cast<uint8_t*>(workspace), M, K);
}

}  // namespace q4gsw
