// q4gsw_api.cu - the extern "C" entry points declared in include/q4gsw.h:
// argument checks, route choice and launches.  Nothing here computes a
// result on the host; every number comes from the CUDA kernels.
//
// Route choice mirrors the geometry predicate of "[ExecuTorch][WebGPU] Replace
// broad QKV fusion with BK64 kernel" (description of #21131): a route is taken
// only for shapes it accepts, and the choice is made on the host per call.
// Argument rules follow "[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward
// kernel (4-bit input-grad)", PR description, "Constraints" (N, K, group_size
// multiples of 4), tightened by the packed layout and TMA stride rules.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstring>

#include "../../include/q4gsw.h"
#include "q4gsw_common.cuh"
#include "q4gsw_internal.h"

namespace q4gsw {

RoutePins& route_pins() {
  thread_local RoutePins pins;
  return pins;
}

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  return dev;
}

int sm_count(int dev) {
  static std::atomic<int> cached[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) dev = 0;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

}  // namespace q4gsw

using namespace q4gsw;

namespace {

thread_local char g_route[160] = "none";

void set_route(const char* s) {
  std::strncpy(g_route, s, sizeof(g_route) - 1);
  g_route[sizeof(g_route) - 1] = 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// Shape rules shared by every entry point.
q4gsw_status check_weight_shape(int N, int K, int gs) {
  if (N <= 0 || K <= 0 || gs <= 0) return Q4GSW_ERR_SHAPE;
  if (N % 4 || K % 4 || gs % 4) return Q4GSW_ERR_SHAPE;        // the page's constraints
  if (N % 8 || K % 64) return Q4GSW_ERR_ALIGN;                  // layout blocks, 16-byte strides
  if (!is_pow2(gs) || gs < 16 || gs > K) return Q4GSW_ERR_UNSUPPORTED;
  return Q4GSW_OK;
}

q4gsw_status from_cuda(cudaError_t e) { return e == cudaSuccess ? Q4GSW_OK : Q4GSW_ERR_CUDA; }

// Token counts up to this run the tensor-core GEMV (weight streaming); above
// it the tcgen05 GEMM.
constexpr int kGemvMaxM = 16;

}  // namespace

namespace {

q4gsw_status prepack_impl(const uint8_t* codes, const void* scales, int N, int K, int group_size, bool f32s,
                          void* packed, size_t packed_bytes, q4gsw_stream_t stream) {
  if (!codes || !scales || !packed) return Q4GSW_ERR_NULL;
  q4gsw_status st = check_weight_shape(N, K, group_size);
  if (st != Q4GSW_OK) return st;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(packed)) return Q4GSW_ERR_ALIGN;
  if (packed_bytes < layout_of(N, K, group_size, f32s ? 4 : 2).total_bytes) return Q4GSW_ERR_SIZE;
  uint32_t flag = 0;
  set_route(f32s ? "prepack_f32s" : "prepack");
  st = from_cuda(launch_prepack(codes, scales, N, K, group_size, f32s, packed, stream, &flag));
  if (st != Q4GSW_OK) return st;
  return flag ? Q4GSW_ERR_CODE_RANGE : Q4GSW_OK;
}

q4gsw_status linear_fwd_impl(const void* packed, int N, int K, int group_size, bool f32s, const uint16_t* x, int M,
                             float* y, q4gsw_stream_t stream) {
  if (M < 0) return Q4GSW_ERR_SHAPE;
  q4gsw_status st = check_weight_shape(N, K, group_size);
  if (st != Q4GSW_OK) return st;
  if (M == 0) { set_route("empty"); return Q4GSW_OK; }
  if (!packed || !x || !y) return Q4GSW_ERR_NULL;
  if (!aligned16(packed) || !aligned16(x) || !aligned16(y)) return Q4GSW_ERR_ALIGN;
  char route[160];
  cudaError_t e = M <= kGemvMaxM
                      ? launch_gemv_fwd(packed, N, K, group_size, f32s, x, M, single_output(y, N), stream, route,
                                        sizeof(route))
                      : launch_gemm_fwd(packed, N, K, group_size, f32s, x, M, single_output(y, N), stream, route,
                                        sizeof(route));
  set_route(route);
  return from_cuda(e);
}

q4gsw_status linear_bwd_impl(const void* packed, int N, int K, int group_size, bool f32s, const uint16_t* d_out, int M,
                             float* d_x, q4gsw_stream_t stream) {
  if (M < 0) return Q4GSW_ERR_SHAPE;
  q4gsw_status st = check_weight_shape(N, K, group_size);
  if (st != Q4GSW_OK) return st;
  if (M == 0) { set_route("empty"); return Q4GSW_OK; }
  if (!packed || !d_out || !d_x) return Q4GSW_ERR_NULL;
  if (!aligned16(packed) || !aligned16(d_out) || !aligned16(d_x)) return Q4GSW_ERR_ALIGN;
  char route[160];
  cudaError_t e = M <= kGemvMaxM
                      ? launch_gemv_bwd(packed, N, K, group_size, f32s, d_out, M, d_x, stream, route, sizeof(route))
                      : launch_gemm_bwd(packed, N, K, group_size, f32s, d_out, M, d_x, stream, route, sizeof(route));
  set_route(route);
  return from_cuda(e);
}

q4gsw_status qkv_fwd_impl(const void* packed_qkv, int Nq, int Nk, int Nv, int K, int group_size, bool f32s,
                          const uint16_t* x, int M, float* y_q, float* y_k, float* y_v, q4gsw_stream_t stream) {
  if (M < 0 || Nq <= 0 || Nk <= 0 || Nv <= 0) return Q4GSW_ERR_SHAPE;
  if ((long long)Nq + Nk + Nv > 0x7fffffffLL) return Q4GSW_ERR_SHAPE;
  const int N = Nq + Nk + Nv;
  q4gsw_status st = check_weight_shape(N, K, group_size);
  if (st != Q4GSW_OK) return st;
  if (Nq % 4 || Nk % 4 || Nv % 4) return Q4GSW_ERR_SHAPE;
  if (Nq % 8 || Nk % 8 || Nv % 8) return Q4GSW_ERR_ALIGN;
  if (M == 0) { set_route("empty"); return Q4GSW_OK; }
  if (!packed_qkv || !x || !y_q || !y_k || !y_v) return Q4GSW_ERR_NULL;
  if (!aligned16(packed_qkv) || !aligned16(x) || !aligned16(y_q) || !aligned16(y_k) || !aligned16(y_v))
    return Q4GSW_ERR_ALIGN;
  OutSplit out{y_q, y_k, y_v, Nq, Nq + Nk, N};
  char route[120];
  cudaError_t e = M <= kGemvMaxM
                      ? launch_gemv_fwd(packed_qkv, N, K, group_size, f32s, x, M, out, stream, route, sizeof(route))
                      : launch_gemm_fwd(packed_qkv, N, K, group_size, f32s, x, M, out, stream, route, sizeof(route));
  char full[160];
  snprintf(full, sizeof(full), "qkv %s", route);
  set_route(full);
  return from_cuda(e);
}

q4gsw_status embedding_impl(const void* packed, int N, int K, int group_size, bool f32s, const int32_t* indices, int T,
                            float* out, q4gsw_stream_t stream) {
  if (T < 0) return Q4GSW_ERR_SHAPE;
  q4gsw_status st = check_weight_shape(N, K, group_size);
  if (st != Q4GSW_OK) return st;
  if (T == 0) {
    set_route("empty");
    return Q4GSW_OK;
  }
  if (!packed || !indices || !out) return Q4GSW_ERR_NULL;
  if (!aligned16(packed) || !aligned16(out) || (reinterpret_cast<uintptr_t>(indices) & 3u)) return Q4GSW_ERR_ALIGN;
  set_route("embedding_gather launches=1");
  return from_cuda(launch_embedding(packed, N, K, group_size, f32s, indices, T, out, stream));
}

q4gsw_status dequant_impl(const void* packed, int N, int K, int group_size, bool f32s, float* w32, uint16_t* w16,
                          q4gsw_stream_t stream) {
  if (!packed || (!w32 && !w16)) return Q4GSW_ERR_NULL;
  q4gsw_status st = check_weight_shape(N, K, group_size);
  if (st != Q4GSW_OK) return st;
  if (!aligned16(packed) || (w32 && !aligned16(w32)) || (w16 && !aligned16(w16))) return Q4GSW_ERR_ALIGN;
  set_route("dequant");
  return from_cuda(launch_dequant(packed, N, K, group_size, f32s, w32, w16, stream));
}

q4gsw_status adapter_impl(bool bwd, const void* packed, int N, int K, int group_size, const uint16_t* a,
                          const uint16_t* b, int r, const uint16_t* act, int M, float* out, void* workspace,
                          size_t workspace_bytes, q4gsw_stream_t stream) {
  if (M < 0) return Q4GSW_ERR_SHAPE;
  q4gsw_status st = check_weight_shape(N, K, group_size);
  if (st != Q4GSW_OK) return st;
  if (r < 8 || r > 64 || r % 8) return Q4GSW_ERR_SHAPE;
  if (M == 0) { set_route("empty"); return Q4GSW_OK; }
  if (!packed || !a || !b || !act || !out || !workspace) return Q4GSW_ERR_NULL;
  if (!aligned16(packed) || !aligned16(a) || !aligned16(b) || !aligned16(act) || !aligned16(out) ||
      !aligned16(workspace))
    return Q4GSW_ERR_ALIGN;
  if (workspace_bytes < (size_t)M * 128) return Q4GSW_ERR_SIZE;
  // the intermediate: forward x A^T (A [r, K] by rows), backward d_out B (B [N, r])
  cudaError_t e = bwd ? launch_adapter_proj(act, b, false, M, N, r, workspace, stream)
                      : launch_adapter_proj(act, a, true, M, K, r, workspace, stream);
  if (e != cudaSuccess) return from_cuda(e);
  char route[160];
  const AdapterRef ad{bwd ? a : b, r, workspace};
  e = launch_gemm_adapter(bwd, packed, N, K, group_size, act, M, out, ad, stream, route, sizeof(route));
  char full[200];
  snprintf(full, sizeof(full), "adapter_%s launches=2 proj + %s", bwd ? "bwd" : "fwd", route);
  set_route(full);
  return from_cuda(e);
}

}  // namespace

extern "C" {

int q4gsw_layout_version(void) { return kLayoutVersion; }

size_t q4gsw_packed_bytes(int N, int K, int group_size) {
  if (check_weight_shape(N, K, group_size) != Q4GSW_OK) return 0;
  return layout_of(N, K, group_size).total_bytes;
}

size_t q4gsw_packed_bytes_f32s(int N, int K, int group_size) {
  if (check_weight_shape(N, K, group_size) != Q4GSW_OK) return 0;
  return layout_of(N, K, group_size, 4).total_bytes;
}

const char* q4gsw_last_route(void) { return g_route; }

const char* q4gsw_status_str(q4gsw_status s) {
  switch (s) {
    case Q4GSW_OK: return "ok";
    case Q4GSW_ERR_NULL: return "null pointer";
    case Q4GSW_ERR_SHAPE: return "invalid shape";
    case Q4GSW_ERR_ALIGN: return "misaligned pointer or shape (16-byte pointers, N % 8, K % 64)";
    case Q4GSW_ERR_UNSUPPORTED: return "unsupported group size (power of two in [16, K]; at least 32 for linear_dq8ca)";
    case Q4GSW_ERR_CODE_RANGE: return "code above 15";
    case Q4GSW_ERR_CUDA: return "CUDA runtime error";
    case Q4GSW_ERR_SIZE: return "buffer too small";
    case Q4GSW_ERR_TIMEOUT: return "a kernel wait ran out (results of the calls since the last check are invalid)";
    case Q4GSW_ERR_INDEX: return "an embedding index was outside [0, N) (its row was written as zeros)";
  }
  return "unknown status";
}

q4gsw_status q4gsw_prepack(const uint8_t* codes, const uint16_t* scales, int N, int K, int group_size,
                           void* packed, size_t packed_bytes, q4gsw_stream_t stream) {
  return prepack_impl(codes, scales, N, K, group_size, false, packed, packed_bytes, stream);
}

q4gsw_status q4gsw_prepack_f32s(const uint8_t* codes, const float* scales, int N, int K, int group_size,
                                void* packed, size_t packed_bytes, q4gsw_stream_t stream) {
  return prepack_impl(codes, scales, N, K, group_size, true, packed, packed_bytes, stream);
}

q4gsw_status q4gsw_linear_fwd(const void* packed, int N, int K, int group_size, const uint16_t* x, int M,
                              float* y, q4gsw_stream_t stream) {
  return linear_fwd_impl(packed, N, K, group_size, false, x, M, y, stream);
}

q4gsw_status q4gsw_linear_fwd_f32s(const void* packed, int N, int K, int group_size, const uint16_t* x, int M,
                                   float* y, q4gsw_stream_t stream) {
  return linear_fwd_impl(packed, N, K, group_size, true, x, M, y, stream);
}

q4gsw_status q4gsw_linear_bwd_input(const void* packed, int N, int K, int group_size, const uint16_t* d_out,
                                    int M, float* d_x, q4gsw_stream_t stream) {
  return linear_bwd_impl(packed, N, K, group_size, false, d_out, M, d_x, stream);
}

q4gsw_status q4gsw_linear_bwd_input_f32s(const void* packed, int N, int K, int group_size, const uint16_t* d_out,
                                         int M, float* d_x, q4gsw_stream_t stream) {
  return linear_bwd_impl(packed, N, K, group_size, true, d_out, M, d_x, stream);
}

q4gsw_status q4gsw_qkv_fwd(const void* packed_qkv, int Nq, int Nk, int Nv, int K, int group_size,
                           const uint16_t* x, int M, float* y_q, float* y_k, float* y_v,
                           q4gsw_stream_t stream) {
  return qkv_fwd_impl(packed_qkv, Nq, Nk, Nv, K, group_size, false, x, M, y_q, y_k, y_v, stream);
}

q4gsw_status q4gsw_qkv_fwd_f32s(const void* packed_qkv, int Nq, int Nk, int Nv, int K, int group_size,
                                const uint16_t* x, int M, float* y_q, float* y_k, float* y_v,
                                q4gsw_stream_t stream) {
  return qkv_fwd_impl(packed_qkv, Nq, Nk, Nv, K, group_size, true, x, M, y_q, y_k, y_v, stream);
}

q4gsw_status q4gsw_device_error_check(q4gsw_stream_t stream) {
  unsigned int v = 0;
  q4gsw_status st = from_cuda(read_and_clear_device_error(stream, &v));
  if (st != Q4GSW_OK) return st;
  if (v & ~0x100u) return Q4GSW_ERR_TIMEOUT;   // bit 8: embedding index range, every other bit: a wait ran out
  return v ? Q4GSW_ERR_INDEX : Q4GSW_OK;
}

q4gsw_status q4gsw_embedding(const void* packed, int N, int K, int group_size, const int32_t* indices, int T,
                             float* out, q4gsw_stream_t stream) {
  return embedding_impl(packed, N, K, group_size, false, indices, T, out, stream);
}

q4gsw_status q4gsw_embedding_f32s(const void* packed, int N, int K, int group_size, const int32_t* indices, int T,
                                  float* out, q4gsw_stream_t stream) {
  return embedding_impl(packed, N, K, group_size, true, indices, T, out, stream);
}

size_t q4gsw_adapter_workspace_bytes(int M, int r) {
  if (M < 0 || r < 8 || r > 64 || r % 8) return 0;
  return (size_t)M * 128;
}

q4gsw_status q4gsw_adapter_fwd(const void* packed, int N, int K, int group_size, const uint16_t* a,
                               const uint16_t* b, int r, const uint16_t* x, int M, float* y, void* workspace,
                               size_t workspace_bytes, q4gsw_stream_t stream) {
  return adapter_impl(false, packed, N, K, group_size, a, b, r, x, M, y, workspace, workspace_bytes, stream);
}

q4gsw_status q4gsw_adapter_bwd_input(const void* packed, int N, int K, int group_size, const uint16_t* a,
                                     const uint16_t* b, int r, const uint16_t* d_out, int M, float* d_x,
                                     void* workspace, size_t workspace_bytes, q4gsw_stream_t stream) {
  return adapter_impl(true, packed, N, K, group_size, a, b, r, d_out, M, d_x, workspace, workspace_bytes, stream);
}

q4gsw_status q4gsw_adapter_fwd_noalloc(const void* packed, int N, int K, int group_size, const uint16_t* a,
                                       const uint16_t* b, int r, const uint16_t* x, int M, float* y,
                                       q4gsw_stream_t stream) {
  if (M < 0) return Q4GSW_ERR_SHAPE;
  if ((size_t)M * 128 > kNoAllocScratchBytes) return Q4GSW_ERR_SIZE;
  void* scratch = nullptr;
  size_t scratch_bytes = 0;
  if (noalloc_scratch(&scratch, &scratch_bytes) != cudaSuccess) return Q4GSW_ERR_CUDA;
  // the projection kernel writes every byte of the rows the GEMM reads, so
  // nothing left in the array by an earlier call needs clearing
  return adapter_impl(false, packed, N, K, group_size, a, b, r, x, M, y, scratch, scratch_bytes, stream);
}

size_t q4gsw_dq8ca_workspace_bytes(int M, int K) {
  if (M < 0 || K <= 0 || K % 64) return 0;
  return dq8ca_workspace_bytes(M, K);
}

q4gsw_status q4gsw_dq8ca_quantize(const uint16_t* x, int M, int K, void* workspace, size_t workspace_bytes,
                                  q4gsw_stream_t stream) {
  if (M < 0 || K <= 0 || K % 4) return Q4GSW_ERR_SHAPE;
  if (K % 64) return Q4GSW_ERR_ALIGN;
  if (M == 0) { set_route("empty"); return Q4GSW_OK; }
  if (!x || !workspace) return Q4GSW_ERR_NULL;
  if (!aligned16(x) || !aligned16(workspace)) return Q4GSW_ERR_ALIGN;
  if (workspace_bytes < dq8ca_workspace_bytes(M, K)) return Q4GSW_ERR_SIZE;
  set_route("dq8ca_quantize launches=1");
  return from_cuda(launch_dq8ca_quantize(x, M, K, workspace, stream));
}

q4gsw_status q4gsw_linear_dq8ca_fwd(const void* packed, int N, int K, int group_size, const uint16_t* x, int M,
                                    float* y, void* workspace, size_t workspace_bytes, q4gsw_stream_t stream) {
  if (M < 0) return Q4GSW_ERR_SHAPE;
  q4gsw_status st = check_weight_shape(N, K, group_size);
  if (st != Q4GSW_OK) return st;
  // a 32-column int8 MMA step lies in one group; a group's int32 sums stay below 2^31
  if (group_size < 32 || group_size > 65536) return Q4GSW_ERR_UNSUPPORTED;
  if (M == 0) { set_route("empty"); return Q4GSW_OK; }
  if (!packed || !x || !y || !workspace) return Q4GSW_ERR_NULL;
  if (!aligned16(packed) || !aligned16(x) || !aligned16(y) || !aligned16(workspace)) return Q4GSW_ERR_ALIGN;
  if (workspace_bytes < dq8ca_workspace_bytes(M, K)) return Q4GSW_ERR_SIZE;
  char inner[96] = "";
  cudaError_t e = launch_dq8ca_quantize(x, M, K, workspace, stream);
  if (e == cudaSuccess)
    e = launch_dq8ca_gemv(packed, N, K, group_size, M, workspace, single_output(y, N), stream, inner, sizeof(inner));
  char route[160];
  snprintf(route, sizeof(route), "dq8ca launches=2 quantize + %s", inner);
  set_route(route);
  return from_cuda(e);
}

q4gsw_status q4gsw_debug_pin_routes(int gemv, int gemm) {
  if (gemv < kGemvAuto || gemv > kGemvTmaXs || gemm < kGemmAuto || gemm > kGemmSs2) return Q4GSW_ERR_SHAPE;
  route_pins().gemv = gemv;
  route_pins().gemm = gemm;
  return Q4GSW_OK;
}

q4gsw_status q4gsw_debug_wait_timeout(unsigned int limit_us, q4gsw_stream_t stream) {
  if (limit_us < 1 || limit_us > 1000000u) return Q4GSW_ERR_SHAPE;
  set_route("wait_probe launches=1");
  return from_cuda(launch_wait_probe(limit_us, stream));
}

q4gsw_status q4gsw_unpack(const void* packed, int N, int K, int group_size, uint8_t* codes,
                          q4gsw_stream_t stream) {
  if (!packed || !codes) return Q4GSW_ERR_NULL;
  q4gsw_status st = check_weight_shape(N, K, group_size);
  if (st != Q4GSW_OK) return st;
  if (!aligned16(packed) || !aligned16(codes)) return Q4GSW_ERR_ALIGN;
  set_route("unpack");
  return from_cuda(launch_unpack(packed, N, K, codes, stream));
}

q4gsw_status q4gsw_dequant(const void* packed, int N, int K, int group_size, float* w32, uint16_t* w16,
                           q4gsw_stream_t stream) {
  return dequant_impl(packed, N, K, group_size, false, w32, w16, stream);
}

q4gsw_status q4gsw_dequant_f32s(const void* packed, int N, int K, int group_size, float* w32, uint16_t* w16,
                                q4gsw_stream_t stream) {
  return dequant_impl(packed, N, K, group_size, true, w32, w16, stream);
}

}  // extern "C"
