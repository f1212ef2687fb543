// q4gsw_embedding.cuh - embedding rows gathered from a packed q4gsw weight
// (sm_100a).  Included once, by q4gsw_gemm_sm100.cu, which owns the device
// error word.
//
//   out[t, k] = (code[idx[t], k] - 8) * s[k / gs, idx[t]]
// The Q4 embedding reads the linear weight's nibble layout ("[ExecuTorch][WebGPU]
// Replace broad QKV fusion with BK64 kernel", description of #21483:
// is_linear_weight); the value of each element is the dequantisation of
// "[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward kernel (4-bit
// input-grad)", PR description, as an exact fp32 product.
//
// A row gather is a pure stream: each thread reads one 16-byte chunk of the
// row's nibble-pair row (16 columns: word i holds columns 16 i + 4 t + e in
// byte slots (0, 2, 1, 3)), keeps its nibble of each byte, scales by the
// group's fp16 scale and writes four float4.  Both rows of a pair share the
// bytes, so a row costs K bytes of codes, K/gs scales and 4 K bytes of output.
#pragma once

namespace q4gsw {

constexpr unsigned int kIndexErrorBit = 0x100u;   // device error word: embedding index out of range
constexpr int kEmbThreads = 128;

namespace emb {

template <bool F32S>
__global__ void __launch_bounds__(kEmbThreads)
q4gsw_embedding_kernel(const uint8_t* __restrict__ packed, const int32_t* __restrict__ indices, float* __restrict__ out,
                       int N, int K, int gs, int T) {
  const Layout L = layout_of(N, K, gs, F32S ? 4 : 2);
  const int gsl = __ffs(gs) - 1;
  const int c = blockIdx.x * kEmbThreads + threadIdx.x;   // 16-byte chunk of the row
  if (c >= K / 16) return;
  const int b = c >> 2, tq = c & 3;                        // 64-column block, chunk in the block
  for (int t = blockIdx.y; t < T; t += gridDim.y) {
    const int r = __ldg(indices + t);
    float* dst = out + (size_t)t * K + 64 * b + 4 * tq;
    if (r < 0 || r >= N) {
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 4; ++i) *reinterpret_cast<float4*>(dst + 16 * i) = z;
      if (c == 0) atomicOr(&g_device_error, kIndexErrorBit);
      continue;
    }
    const uint4 v = ldg_stream_v4(packed + (size_t)(r >> 1) * K + 64 * b + 16 * tq);
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
    const int shift = 4 * (r & 1);   // odd rows live in the high nibbles
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k0 = 64 * b + 16 * i + 4 * tq;   // columns k0 .. k0 + 3 share one group (gs >= 16)
      const size_t si = (size_t)(k0 >> gsl) * N + r;
      const float s = F32S ? __ldg(reinterpret_cast<const float*>(packed + L.scales_offset) + si)
                           : __half2float(__ldg(reinterpret_cast<const __half*>(packed + L.scales_offset) + si));
      const uint32_t w = words[i] >> shift;
      // byte slots (0, 1, 2, 3) hold columns (+0, +2, +1, +3); with fp16 scales
      // the products are exact, with fp32 scales each is rounded once
      const float v0 = __fmul_rn((float)((int)(w & 0xFu) - 8), s);
      const float v2 = __fmul_rn((float)((int)((w >> 8) & 0xFu) - 8), s);
      const float v1 = __fmul_rn((float)((int)((w >> 16) & 0xFu) - 8), s);
      const float v3 = __fmul_rn((float)((int)((w >> 24) & 0xFu) - 8), s);
      *reinterpret_cast<float4*>(dst + 16 * i) = make_float4(v0, v1, v2, v3);
    }
  }
}

}  // namespace emb

cudaError_t launch_embedding(const void* packed, int N, int K, int gs, bool f32s, const int32_t* indices, int T,
                             float* out, cudaStream_t stream) {
  const int chunks = K / 16;
  const dim3 grid((chunks + kEmbThreads - 1) / kEmbThreads, T < 65535 ? T : 65535);
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  if (f32s)
    emb::q4gsw_embedding_kernel<true><<<grid, kEmbThreads, 0, stream>>>(pk, indices, out, N, K, gs, T);
  else
    emb::q4gsw_embedding_kernel<false><<<grid, kEmbThreads, 0, stream>>>(pk, indices, out, N, K, gs, T);
  return cudaGetLastError();
}

}  // namespace q4gsw
