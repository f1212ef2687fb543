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
// Two kernels.  The quantiser writes q (int8, with the byte order of the packed
// codes inside each 4-column group: columns +0, +2, +1, +3), a_s and a_z into
// the caller's workspace.  The product runs int8 tensor-core MMAs
// (mma.sync m16n8k32, unsigned codes x signed q, exact int32 sums):
//   sum (q - a_z)(c - 8) = sum q c - 8 sum q - a_z sum c + 8 a_z n
// over the n columns a warp accumulates; sum q c is the MMA of the codes (one
// mask per row, no -8), sum c the MMA of the codes with a ones operand, sum q
// the MMA of a ones operand with q.  A finished group is scaled by its fp16
// scale in fp32; a_s multiplies at the end.
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "q4gsw_common.cuh"
#include "q4gsw_internal.h"

namespace q4gsw {
namespace dq {

constexpr int kQThreads = 256;

// Workspace map for M tokens of K features (offsets in bytes).
__host__ __device__ inline size_t off_as(int M, int K) { return round_up((size_t)M * K, 256); }
__host__ __device__ inline size_t off_az(int M, int K) { return off_as(M, K) + round_up((size_t)4 * M, 256); }
__host__ __device__ inline size_t ws_bytes(int M, int K) { return off_az(M, K) + round_up((size_t)4 * M, 256); }

__global__ void __launch_bounds__(kQThreads)
q4gsw_dq8ca_quantize_kernel(const __half* __restrict__ x, uint8_t* __restrict__ ws, int M, int K) {
  __shared__ float s_lo[kQThreads / 32], s_hi[kQThreads / 32];
  __shared__ float s_as;
  __shared__ int s_az;
  griddep_launch_dependents();
  griddep_wait();   // x may come from the previous kernel of the stream
  const int m = blockIdx.x;
  const __half* row = x + (size_t)m * K;
  float lo = 0.f, hi = 0.f;   // the range always holds 0
  for (int k = threadIdx.x; k < K; k += kQThreads) {
    const float v = __half2float(row[k]);
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
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
  if (threadIdx.x == 0) {
    for (int w = 1; w < kQThreads / 32; ++w) {
      lo = fminf(lo, s_lo[w]);
      hi = fmaxf(hi, s_hi[w]);
    }
    lo = fminf(lo, s_lo[0]);
    hi = fmaxf(hi, s_hi[0]);
    const float as = hi == lo ? 1.f : __fdiv_rn(__fsub_rn(hi, lo), 255.f);
    float z = rintf(__fsub_rn(-128.f, __fdiv_rn(lo, as)));
    z = fminf(127.f, fmaxf(-128.f, z));
    s_as = as;
    s_az = (int)z;
    reinterpret_cast<float*>(ws + off_as(M, K))[m] = as;
    reinterpret_cast<int*>(ws + off_az(M, K))[m] = (int)z;
  }
  __syncthreads();
  const float as = s_as;
  const int az = s_az;
  uint32_t* qrow = reinterpret_cast<uint32_t*>(ws + (size_t)m * K);
  for (int c4 = threadIdx.x; c4 < K / 4; c4 += kQThreads) {
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float v = __half2float(row[4 * c4 + e]);
      int qv = (int)rintf(__fdiv_rn(v, as)) + az;
      qv = qv < -128 ? -128 : qv > 127 ? 127 : qv;
      const int slot = e == 1 ? 2 : e == 2 ? 1 : e;   // the packed codes' byte order
      word |= (uint32_t)(qv & 0xFF) << (8 * slot);
    }
    qrow[c4] = word;
  }
}

// D(16x8, s32) += A(16x32, u8, row) * B(32x8, s8, col)
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;

// grid = (ceil(N / 16) row tiles, 1, ceil(M / 8) token tiles); warp u takes the
// 64-column blocks [u KB / 4, (u + 1) KB / 4) of the CTA's 16 rows.
__global__ void __launch_bounds__(kThreads)
q4gsw_dq8ca_gemv_kernel(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ ws, OutSplit out, int M,
                        int N, int K, int gs) {
  __shared__ float red[kWarps][8][16];   // [warp][token][row]
  griddep_launch_dependents();
  griddep_wait();   // the workspace comes from the quantiser just before
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x, tok0 = blockIdx.z * 8;
  const int Mz = min(8, M - tok0);
  const Layout L = layout_of(N, K, gs);
  const __half* scales = reinterpret_cast<const __half*>(packed + L.scales_offset);
  const int p_raw = tile * 8 + g;
  const int p = p_raw < (N >> 1) ? p_raw : 0;            // rows past N read pair 0, never stored
  const uint8_t* crow = packed + (size_t)p * K + 16 * t;
  const int tok = tok0 + min(g, Mz - 1);                  // B column g: this token (repeated past Mz)
  const uint8_t* qrow = ws + (size_t)tok * K + 4 * t;
  const float* as_v = reinterpret_cast<const float*>(ws + off_as(M, K));
  const int* az_v = reinterpret_cast<const int*>(ws + off_az(M, K));
  // D columns 2t, 2t + 1 are tokens tok0 + 2t, tok0 + 2t + 1
  const int ta = tok0 + min(2 * t, Mz - 1), tb = tok0 + min(2 * t + 1, Mz - 1);
  const int az0 = az_v[ta], az1 = az_v[tb];
  const int gsl = __ffs(gs) - 1;
  const int KB = K >> 6;
  const int b_begin = warp * KB / kWarps, b_end = (warp + 1) * KB / kWarps;
  const uint32_t ones[4] = {0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u};
  const uint32_t ones2[2] = {0x01010101u, 0x01010101u};

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int i1[4] = {0, 0, 0, 0}, i2[4] = {0, 0, 0, 0}, i3[4] = {0, 0, 0, 0};
  int ncols = 0;
  auto flush = [&](int grp) {
    const __half2 s2 = *reinterpret_cast<const __half2*>(scales + (size_t)grp * N + 2 * p);
    const float se = __low2float(s2), so = __high2float(s2);
    // D fragment: [0] row g (even), token 2t; [1] row g, token 2t+1; [2] row g+8 (odd), 2t; [3] odd, 2t+1.
    // i2 (code sums) is the same in every column; i3 (q sums) the same in every row.
    const int n8 = 8 * ncols;
    const int t0 = i1[0] - 8 * i3[0] - az0 * i2[0] + n8 * az0;
    const int t1 = i1[1] - 8 * i3[1] - az1 * i2[1] + n8 * az1;
    const int t2 = i1[2] - 8 * i3[2] - az0 * i2[2] + n8 * az0;
    const int t3 = i1[3] - 8 * i3[3] - az1 * i2[3] + n8 * az1;
    acc[0] = fmaf((float)t0, se, acc[0]);
    acc[1] = fmaf((float)t1, se, acc[1]);
    acc[2] = fmaf((float)t2, so, acc[2]);
    acc[3] = fmaf((float)t3, so, acc[3]);
#pragma unroll
    for (int c = 0; c < 4; ++c) i1[c] = i2[c] = i3[c] = 0;
    ncols = 0;
  };
  for (int b = b_begin; b < b_end; ++b) {
    const uint4 w = ldg_stream_v4(crow + 64 * b);
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int h = 0; h < 2; ++h) {   // two 32-column MMA steps: words 2h, 2h + 1
      const uint32_t w0 = words[2 * h], w1 = words[2 * h + 1];
      const uint32_t a[4] = {w0 & 0x0F0F0F0Fu, (w0 >> 4) & 0x0F0F0F0Fu, w1 & 0x0F0F0F0Fu, (w1 >> 4) & 0x0F0F0F0Fu};
      const int k0 = 64 * b + 32 * h;
      const uint32_t bq[2] = {ldg_nc_u32(qrow + k0), ldg_nc_u32(qrow + k0 + 16)};
      mma_u8s8(i1, a, bq);
      mma_u8s8(i2, a, ones2);     // sum of the codes of each row
      mma_u8s8(i3, ones, bq);     // sum of q of each token
      ncols += 32;
      // flush when the next step starts another group, or the warp's range ends
      const int kn = k0 + 32;
      if ((kn >> gsl) != (k0 >> gsl) || (b == b_end - 1 && h == 1)) flush(k0 >> gsl);
    }
  }
  // y = a_s * acc; the warps' column ranges summed in order
  red[warp][2 * t][2 * g] = acc[0];
  red[warp][2 * t + 1][2 * g] = acc[1];
  red[warp][2 * t][2 * g + 1] = acc[2];
  red[warp][2 * t + 1][2 * g + 1] = acc[3];
  __syncthreads();
  for (int e = threadIdx.x; e < Mz * 16; e += kThreads) {
    const int tk = e >> 4, nl = e & 15;
    const int n = tile * 16 + nl;
    if (n >= N) continue;
    const float s = ((red[0][tk][nl] + red[1][tk][nl]) + red[2][tk][nl]) + red[3][tk][nl];
    const size_t m = (size_t)(tok0 + tk);
    const float v = s * as_v[m];
    if (n < out.n1) out.y0[m * out.n1 + n] = v;
    else if (n < out.n2) out.y1[m * (out.n2 - out.n1) + (n - out.n1)] = v;
    else out.y2[m * (out.N - out.n2) + (n - out.n2)] = v;
  }
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

cudaError_t launch_dq8ca_gemv(const void* packed, int N, int K, int gs, int M, const void* workspace, OutSplit out,
                              cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((N + 15) / 16, 1, (M + 7) / 8);
  cfg.blockDim = dim3(dq::kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dq::q4gsw_dq8ca_gemv_kernel, static_cast<const uint8_t*>(packed),
                            static_cast<const uint8_t*>(workspace), out, M, N, K, gs);
}

}  // namespace q4gsw
