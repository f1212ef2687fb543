// q4gsw_internal.h - launchers shared between the translation units of the
// library.  Not part of the C ABI.
#pragma once

#include <atomic>
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

namespace q4gsw {

// Route pins of the calling host thread (set by q4gsw_debug_pin_routes; 0
// everywhere means the launchers choose).  Thread-local, like the route string.
enum GemvPin { kGemvAuto = 0, kGemvReg = 1, kGemvTma = 2, kGemvTmaXs = 3 };
enum GemmPin { kGemmAuto = 0, kGemmTs = 1, kGemmSs = 2, kGemmSs1 = 3, kGemmSs2 = 4 };
struct RoutePins {
  int gemv = kGemvAuto;
  int gemm = kGemmAuto;
};
RoutePins& route_pins();

// One-time set-up per device (cudaFuncSetAttribute of one kernel variant),
// safe when several host threads make their first call at the same time: the
// first caller runs `fn`, the others wait for it and then see its result.
constexpr int kMaxDevices = 64;
struct PerDeviceOnce {
  std::once_flag flag[kMaxDevices];
  std::atomic<int> err[kMaxDevices];
};
template <typename F>
inline cudaError_t once_per_device(PerDeviceOnce& o, int dev, F&& fn) {
  if (dev < 0 || dev >= kMaxDevices) return fn();   // not cached
  std::call_once(o.flag[dev], [&] { o.err[dev].store(static_cast<int>(fn())); });
  return static_cast<cudaError_t>(o.err[dev].load());
}

// Device the calling thread is bound to (cudaGetDevice), and its SM count.
int current_device();
int sm_count(int dev);

// f32s: the blob holds fp32 scales (packed layout version 2) instead of fp16.
cudaError_t launch_prepack(const uint8_t* codes, const void* scales, int N, int K, int gs, bool f32s, void* packed,
                           cudaStream_t stream, uint32_t* host_flag);
cudaError_t launch_unpack(const void* packed, int N, int K, uint8_t* codes, cudaStream_t stream);
cudaError_t launch_dequant(const void* packed, int N, int K, int gs, bool f32s, float* w32, uint16_t* w16,
                           cudaStream_t stream);

// Output columns [0, N) of a forward split over up to three row-major
// buffers: n < n1 -> y0[m, n], n < n2 -> y1[m, n - n1], else y2[m, n - n2]
// (the fused Q/K/V projection writes three distinct outputs).
struct OutSplit {
  float* y0;
  float* y1;
  float* y2;
  int n1, n2, N;
};

__host__ __device__ inline OutSplit single_output(float* y, int N) { return OutSplit{y, y, y, N, N, N}; }

// The compute launchers take f32s = the packed blob has fp32 scales (layout
// version 2) instead of fp16 (version 1).
// Tensor-core GEMV routes for small token counts.  `M` may exceed 16: token
// chunks of 16 then run as grid z-slices (each re-reads the weight).
cudaError_t launch_gemv_fwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* x, int M,
                            OutSplit out, cudaStream_t stream, char* route, int route_len);
cudaError_t launch_gemv_bwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* d_out, int M,
                            float* d_x, cudaStream_t stream, char* route, int route_len);

// Forward GEMV that streams the packed weight through a TMA ring (M <= 16
// per z-slice).
cudaError_t launch_gemv_tma_fwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* x, int M, OutSplit out,
                                cudaStream_t stream, char* route, int route_len);
cudaError_t launch_gemv_tma_bwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* d_out, int M, float* d_x,
                                cudaStream_t stream, char* route, int route_len);

// tcgen05 GEMM routes (any M >= 1; used above the GEMV range).
cudaError_t launch_gemm_fwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* x, int M, OutSplit out,
                            cudaStream_t stream, char* route, int route_len);
cudaError_t launch_gemm_bwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* d_out, int M, float* d_x,
                            cudaStream_t stream, char* route, int route_len);

// Frozen-base low-rank adapter: the fp16 adapter matrix (forward B [N, r],
// backward A [r, K]), its rank (8 <= r <= 64, r % 8 == 0) and the fp16
// intermediate [M][64] (forward x A^T, backward d_out B; columns r..63 zero).
struct AdapterRef {
  const uint16_t* mat;
  int r;
  const void* inter;
};
// The intermediate: act [M][C] times the projection (by_rows: A [r, C], used
// as A^T; else B [C, r]) into `workspace` as [M][64] fp16.
cudaError_t launch_adapter_proj(const uint16_t* act, const uint16_t* proj, bool by_rows, int M, int C, int r,
                                void* workspace, cudaStream_t stream);
// Device address (on the current device) and size of the library's own fixed
// scratch array for the allocation-free adapter entry point.  The first call
// on a device looks the address up (cudaGetSymbolAddress).
constexpr size_t kNoAllocScratchBytes = (size_t)1 << 20;
cudaError_t noalloc_scratch(void** ptr, size_t* bytes);
// The tensor-memory GEMM (forward when !bwd) with the adapter stage added to
// the accumulator of the last contraction split.
cudaError_t launch_gemm_adapter(bool bwd, const void* packed, int N, int K, int gs, const uint16_t* act, int M,
                                float* out, const AdapterRef& ad, cudaStream_t stream, char* route, int route_len);

// int8 dynamically quantised activations (linear_dq8ca_q4gsw): workspace map
// (q int8 [M][K], a_s fp32 [M], a_z int32 [M]), the quantiser and the product.
size_t dq8ca_workspace_bytes(int M, int K);
size_t dq8ca_scale_offset(int M, int K);
size_t dq8ca_zero_offset(int M, int K);
cudaError_t launch_dq8ca_quantize(const uint16_t* x, int M, int K, void* workspace, cudaStream_t stream);
cudaError_t launch_dq8ca_gemv(const void* packed, int N, int K, int gs, int M, const void* workspace, OutSplit out,
                              cudaStream_t stream, char* route, int route_len);

// Embedding rows out[t] = dequant(W)[indices[t]] (fp32); an index outside
// [0, N) gives a zero row and sets kIndexErrorBit in the device error word.
cudaError_t launch_embedding(const void* packed, int N, int K, int gs, bool f32s, const int32_t* indices, int T, float* out,
                             cudaStream_t stream);

// One thread block that waits on a barrier nothing completes until its
// bounded wait (limit_us microseconds) runs out and records a time-out.
cudaError_t launch_wait_probe(unsigned int limit_us, cudaStream_t stream);

// Swaps the device word in which kernels record waits that ran out (and
// embedding indices out of range) with 0 in one atomic operation, ordered on
// `stream`, and returns the old value; synchronises `stream`.
cudaError_t read_and_clear_device_error(cudaStream_t stream, unsigned int* host_value);

}  // namespace q4gsw
