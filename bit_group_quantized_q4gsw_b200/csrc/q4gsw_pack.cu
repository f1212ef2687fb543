// q4gsw_pack.cu - the one-time packer and the two debug exports (unpack,
// dequant) of the q4gsw weight.
//
// Packing follows "[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward kernel
// (4-bit input-grad)", PR description, "Key changes" (nibble pairs, even-N low;
// [num_groups, N] scales; one prepack for forward and backward) and
// "[ExecuTorch][WebGPU] Replace broad QKV fusion with BK64 kernel", description
// of #21131 (constant weights and scales packed once).  The byte order inside a
// pair row is this library's layout version 1 (q4gsw_common.cuh).
#include <cuda_runtime.h>

#include "q4gsw_common.cuh"
#include "q4gsw_internal.h"

namespace q4gsw {
namespace pk {

// One thread per 16-byte output chunk of the codes region: pair p, 64-byte
// block b, quarter t of the block.  The chunk holds word slots 4t .. 4t+3, i.e.
// columns 64b + 16 i + 4 t + e for i, e in 0..3.
__global__ void q4gsw_prepack_codes_kernel(const uint8_t* __restrict__ codes, uint8_t* __restrict__ packed,
                                     int N, int K, uint32_t* __restrict__ range_flag) {
  const int blocks_per_row = K / 64;
  const long long chunks = (long long)(N / 2) * blocks_per_row * 4;
  uint32_t bad = 0;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < chunks;
       c += (long long)gridDim.x * blockDim.x) {
    const int t = int(c & 3);
    const long long pb = c >> 2;
    const int b = int(pb % blocks_per_row);
    const int p = int(pb / blocks_per_row);
    const uint8_t* even = codes + (size_t)(2 * p) * K + 64 * b + 4 * t;
    const uint8_t* odd = even + K;
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t e4 = *reinterpret_cast<const uint32_t*>(even + 16 * i);  // columns +0..3
      const uint32_t o4 = *reinterpret_cast<const uint32_t*>(odd + 16 * i);
      bad |= (e4 | o4) & 0xF0F0F0F0u;
      const uint32_t bytes = (e4 & 0x0F0F0F0Fu) | ((o4 & 0x0F0F0F0Fu) << 4);   // byte j = column j
      out[i] = prmt(bytes, 0u, 0x3120u);  // slots (0, 1, 2, 3) <- columns (0, 2, 1, 3)
    }
    *reinterpret_cast<uint4*>(packed + (size_t)p * K + 64 * b + 16 * t) = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (bad) atomicOr(range_flag, 1u);
}

// Scales copy (fp16 or fp32: sbytes per scale), zero padding and trailer
// words 0..4 (word 5, the range flag, is zeroed by the host before this runs
// and only ever OR-ed).
__global__ void q4gsw_prepack_tail_kernel(const void* __restrict__ scales, uint8_t* __restrict__ packed,
                                          int N, int K, int gs, int sbytes) {
  const Layout L = layout_of(N, K, gs, sbytes);
  const size_t tid = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t n16 = L.scales_bytes / 16;  // N % 8 == 0 -> a whole number of 16-byte vectors
  const uint4* src = reinterpret_cast<const uint4*>(scales);
  uint4* dst = reinterpret_cast<uint4*>(packed + L.scales_offset);
  for (size_t i = tid; i < n16; i += stride) dst[i] = src[i];
  for (size_t i = L.codes_bytes + tid; i < L.scales_offset; i += stride) packed[i] = 0;
  for (size_t i = L.scales_offset + L.scales_bytes + tid; i < L.trailer_offset; i += stride) packed[i] = 0;
  if (tid == 0) {
    uint32_t* tr = reinterpret_cast<uint32_t*>(packed + L.trailer_offset);
    tr[0] = kTrailerMagic;
    tr[1] = sbytes == 4 ? kLayoutVersionF32S : kLayoutVersion;
    tr[2] = uint32_t(N);
    tr[3] = uint32_t(K);
    tr[4] = uint32_t(gs);
  }
}

__global__ void q4gsw_unpack_kernel(const uint8_t* __restrict__ packed, uint8_t* __restrict__ codes, int N, int K) {
  const int blocks_per_row = K / 64;
  const long long chunks = (long long)(N / 2) * blocks_per_row * 4;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < chunks;
       c += (long long)gridDim.x * blockDim.x) {
    const int t = int(c & 3);
    const long long pb = c >> 2;
    const int b = int(pb % blocks_per_row);
    const int p = int(pb / blocks_per_row);
    const uint4 v = *reinterpret_cast<const uint4*>(packed + (size_t)p * K + 64 * b + 16 * t);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint8_t* even = codes + (size_t)(2 * p) * K + 64 * b + 4 * t;
    uint8_t* odd = even + K;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t bytes = prmt(w[i], 0u, 0x3120u);  // back to column order (0, 1, 2, 3)
      *reinterpret_cast<uint32_t*>(even + 16 * i) = bytes & 0x0F0F0F0Fu;
      *reinterpret_cast<uint32_t*>(odd + 16 * i) = (bytes >> 4) & 0x0F0F0F0Fu;
    }
  }
}

// The dequantised weight, produced with the same conversions the GEMM
// kernels use.  fp16 scales (F32S false): w16 = fp16((code - 8)) * scale
// rounded once (HMUL2), and the exact fp32 product w32.  fp32 scales (layout
// version 2): w32 = (code - 8) * s32 rounded once in fp32, w16 = fp16_RNE(w32).
template <bool F32S>
__global__ void q4gsw_dequant_kernel(const uint8_t* __restrict__ packed, float* __restrict__ w32,
                                     uint16_t* __restrict__ w16, int N, int K, int gs) {
  const Layout L = layout_of(N, K, gs, F32S ? 4 : 2);
  const int blocks_per_row = K / 64;
  const long long chunks = (long long)(N / 2) * blocks_per_row * 4;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < chunks;
       c += (long long)gridDim.x * blockDim.x) {
    const int t = int(c & 3);
    const long long pb = c >> 2;
    const int b = int(pb % blocks_per_row);
    const int p = int(pb / blocks_per_row);
    const uint4 v = *reinterpret_cast<const uint4*>(packed + (size_t)p * K + 64 * b + 16 * t);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k0 = 64 * b + 16 * i + 4 * t;  // columns k0 .. k0+3
      const int g = k0 >> (__ffs(gs) - 1);
      const RowPairs r = codes_minus8_rows(w[i]);
      const size_t re = (size_t)(2 * p) * K + k0, ro = re + K;
      float4 fe, fo;
      if (F32S) {
        const float2 s2 = *reinterpret_cast<const float2*>(
            reinterpret_cast<const float*>(packed + L.scales_offset) + (size_t)g * N + 2 * p);
        fe = make_float4(__fmul_rn(__low2float(r.ev01), s2.x), __fmul_rn(__high2float(r.ev01), s2.x),
                         __fmul_rn(__low2float(r.ev23), s2.x), __fmul_rn(__high2float(r.ev23), s2.x));
        fo = make_float4(__fmul_rn(__low2float(r.od01), s2.y), __fmul_rn(__high2float(r.od01), s2.y),
                         __fmul_rn(__low2float(r.od23), s2.y), __fmul_rn(__high2float(r.od23), s2.y));
        if (w16) {
          *reinterpret_cast<uint2*>(w16 + re) = make_uint2(h2_as_u32(__floats2half2_rn(fe.x, fe.y)),
                                                           h2_as_u32(__floats2half2_rn(fe.z, fe.w)));
          *reinterpret_cast<uint2*>(w16 + ro) = make_uint2(h2_as_u32(__floats2half2_rn(fo.x, fo.y)),
                                                           h2_as_u32(__floats2half2_rn(fo.z, fo.w)));
        }
      } else {
        const __half2 s2 = *reinterpret_cast<const __half2*>(
            reinterpret_cast<const __half*>(packed + L.scales_offset) + (size_t)g * N + 2 * p);
        const __half2 se = __low2half2(s2), so = __high2half2(s2);
        if (w16) {
          *reinterpret_cast<uint2*>(w16 + re) = make_uint2(h2_as_u32(__hmul2(r.ev01, se)), h2_as_u32(__hmul2(r.ev23, se)));
          *reinterpret_cast<uint2*>(w16 + ro) = make_uint2(h2_as_u32(__hmul2(r.od01, so)), h2_as_u32(__hmul2(r.od23, so)));
        }
        const float ffe = __low2float(s2), ffo = __high2float(s2);
        fe = make_float4(__low2float(r.ev01) * ffe, __high2float(r.ev01) * ffe, __low2float(r.ev23) * ffe,
                         __high2float(r.ev23) * ffe);
        fo = make_float4(__low2float(r.od01) * ffo, __high2float(r.od01) * ffo, __low2float(r.od23) * ffo,
                         __high2float(r.od23) * ffo);
      }
      if (w32) {
        *reinterpret_cast<float4*>(w32 + re) = fe;
        *reinterpret_cast<float4*>(w32 + ro) = fo;
      }
    }
  }
}

}  // namespace pk

static int grid_for(long long work, int threads) {
  long long g = (work + threads - 1) / threads;
  if (g > 148LL * 16) g = 148LL * 16;
  if (g < 1) g = 1;
  return int(g);
}

cudaError_t launch_prepack(const uint8_t* codes, const void* scales, int N, int K, int gs, bool f32s, void* packed,
                           cudaStream_t stream, uint32_t* host_flag) {
  const int sbytes = f32s ? 4 : 2;
  const Layout L = layout_of(N, K, gs, sbytes);
  uint8_t* out = static_cast<uint8_t*>(packed);
  uint32_t* flag = reinterpret_cast<uint32_t*>(out + L.trailer_offset) + 5;
  cudaError_t err = cudaMemsetAsync(out + L.trailer_offset, 0, kTrailerBytes, stream);
  if (err != cudaSuccess) return err;
  const long long chunks = (long long)(N / 2) * (K / 64) * 4;
  pk::q4gsw_prepack_codes_kernel<<<grid_for(chunks, 256), 256, 0, stream>>>(codes, out, N, K, flag);
  pk::q4gsw_prepack_tail_kernel<<<grid_for((long long)(L.scales_bytes / 16) + 256, 256), 256, 0, stream>>>(
      scales, out, N, K, gs, sbytes);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  err = cudaMemcpyAsync(host_flag, flag, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream);
  if (err != cudaSuccess) return err;
  return cudaStreamSynchronize(stream);
}

cudaError_t launch_unpack(const void* packed, int N, int K, uint8_t* codes, cudaStream_t stream) {
  const long long chunks = (long long)(N / 2) * (K / 64) * 4;
  pk::q4gsw_unpack_kernel<<<grid_for(chunks, 256), 256, 0, stream>>>(static_cast<const uint8_t*>(packed), codes, N, K);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const void* packed, int N, int K, int gs, bool f32s, float* w32, uint16_t* w16,
                           cudaStream_t stream) {
  const long long chunks = (long long)(N / 2) * (K / 64) * 4;
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  if (f32s)
    pk::q4gsw_dequant_kernel<true><<<grid_for(chunks, 256), 256, 0, stream>>>(pk, w32, w16, N, K, gs);
  else
    pk::q4gsw_dequant_kernel<false><<<grid_for(chunks, 256), 256, 0, stream>>>(pk, w32, w16, N, K, gs);
  return cudaGetLastError();
}

}  // namespace q4gsw
