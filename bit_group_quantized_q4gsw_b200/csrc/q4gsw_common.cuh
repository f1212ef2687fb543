// q4gsw_common.cuh - layout arithmetic and device helpers shared by the
// q4gsw CUDA kernels (sm_100a).
//
// The weight is w[n,k] = (code[n,k] - 8) * scale[k / gs, n]  ("[ExecuTorch][Vulkan]
// Add et_vk.linear_q4gsw_backward kernel (4-bit input-grad)", PR description).
// The packed blob (layout version 1) is
//   codes   N/2 rows of K bytes; byte (p, k) = code[2p,k] | code[2p+1,k] << 4
//           (same PR, "Key changes": even-N low nibble, odd-N high), placed
//           inside its 64-byte block: column r = 16 i + 4 t + e goes to word
//           slot 4 t + i, byte slot {0, 2, 1, 3}[e];
//   scales  fp16 [G][N] at round_up(N/2*K, 256) (version 2: fp32 [G][N]);
//   trailer 64 bytes at round_up(scales end, 256).
//
// Why this byte order: a 16-byte load at offset 16 t of a block gives word i
// (i = 0..3) = columns 16 i + 4 t + 0..3, so lane t of a quad holds four
// consecutive columns of each 16-column tensor-core step; and inside a word the
// low nibbles of bytes 0 and 2 are columns +0, +1, so one LOP3 with the mask
// 0x000F000F yields a half2 of two consecutive columns of the even row.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_fp16.h>

namespace q4gsw {

constexpr int kRegionAlign = 256;
constexpr int kTrailerBytes = 64;
constexpr uint32_t kTrailerMagic = 0x53473451u;  // "Q4GS"
constexpr int kLayoutVersion = 1;      // fp16 scales
constexpr int kLayoutVersionF32S = 2;  // fp32 scales

struct Layout {
  size_t codes_bytes;
  size_t scales_offset;
  size_t scales_bytes;
  size_t trailer_offset;
  size_t total_bytes;
};

__host__ __device__ inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// sbytes: bytes per scale, 2 (fp16, layout version 1) or 4 (fp32, version 2;
// the codes region is the same in both versions)
__host__ __device__ inline Layout layout_of(int N, int K, int gs, int sbytes = 2) {
  Layout L;
  L.codes_bytes = size_t(N / 2) * size_t(K);
  L.scales_offset = round_up(L.codes_bytes, kRegionAlign);
  L.scales_bytes = size_t(sbytes) * size_t(K / gs) * size_t(N);
  L.trailer_offset = round_up(L.scales_offset + L.scales_bytes, kRegionAlign);
  L.total_bytes = L.trailer_offset + kTrailerBytes;
  return L;
}

// Byte offset of column k inside its pair row.
__host__ __device__ inline int column_offset(int k) {
  const int r = k & 63;
  const int i = r >> 4, t = (r >> 2) & 3, e = r & 3;
  const int slot = (e == 1) ? 2 : (e == 2) ? 1 : e;
  return (k & ~63) + 4 * (4 * t + i) + slot;
}

// ---------------------------------------------------------------------------
// Nibble -> fp16 conversions.  0x6400 is the fp16 bit pattern of 1024, whose
// ulp is 1: OR-ing a nibble c into bits 0..3 gives exactly 1024 + c, and into
// bits 4..7 gives exactly 1024 + 16 c.  Subtracting 1032, or scaling by 1/16
// and subtracting 72, leaves the exact integer c - 8 in fp16.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t magic) {
  uint32_t d;
  // (a & mask) | magic
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));
  return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ __half2 u32_as_h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }
__device__ __forceinline__ uint32_t h2_as_u32(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

// Word W of one pair row holds columns c0..c3 of a 4-column run in byte slots
// (c0, c2, c1, c3).  Returns the four half2 values (exact integers code - 8):
//   ev01 = (even row c0, c1)  ev23 = (even row c2, c3)
//   od01 = (odd  row c0, c1)  od23 = (odd  row c2, c3)
struct RowPairs { __half2 ev01, ev23, od01, od23; };

__device__ __forceinline__ RowPairs codes_minus8_rows(uint32_t W) {
  const uint32_t kMagic = 0x64006400u;
  const __half2 kSub = u32_as_h2(0x64086408u);        // 1032, 1032
  const __half2 kInv16 = u32_as_h2(0x2C002C00u);      // 1/16, 1/16
  const __half2 kSub72 = u32_as_h2(0xD480D480u);      // -72, -72
  const uint32_t W8 = W >> 8;
  RowPairs r;
  r.ev01 = __hsub2(u32_as_h2(lop3_and_or(W, 0x000F000Fu, kMagic)), kSub);
  r.ev23 = __hsub2(u32_as_h2(lop3_and_or(W8, 0x000F000Fu, kMagic)), kSub);
  r.od01 = __hfma2(u32_as_h2(lop3_and_or(W, 0x00F000F0u, kMagic)), kInv16, kSub72);
  r.od23 = __hfma2(u32_as_h2(lop3_and_or(W8, 0x00F000F0u, kMagic)), kInv16, kSub72);
  return r;
}

// Same word, split per column instead of per row: returns for each column
// c0..c3 the half2 (even row, odd row) = (lo nibble - 8, hi nibble - 8).
struct ColPairs { __half2 c0, c1, c2, c3; };

__device__ __forceinline__ ColPairs codes_minus8_cols(uint32_t W) {
  const uint32_t kMagic = 0x64006400u;
  const __half2 kMul = u32_as_h2(0x2C003C00u);        // (1, 1/16)
  const __half2 kAdd = u32_as_h2(0xD480E408u);        // (-1032, -72)
  const uint32_t A = prmt(W, 0u, 0x1010u);             // bytes (c0, c2, c0, c2)
  const uint32_t B = prmt(W, 0u, 0x3232u);             // bytes (c1, c3, c1, c3)
  ColPairs r;
  r.c0 = __hfma2(u32_as_h2(lop3_and_or(A, 0x00F0000Fu, kMagic)), kMul, kAdd);
  r.c2 = __hfma2(u32_as_h2(lop3_and_or(A >> 8, 0x00F0000Fu, kMagic)), kMul, kAdd);
  r.c1 = __hfma2(u32_as_h2(lop3_and_or(B, 0x00F0000Fu, kMagic)), kMul, kAdd);
  r.c3 = __hfma2(u32_as_h2(lop3_and_or(B >> 8, 0x00F0000Fu, kMagic)), kMul, kAdd);
  return r;
}

// ---------------------------------------------------------------------------
// Memory helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// Per-thread asynchronous 16-byte global -> shared copy (L2 only), with the
// commit / wait-group pair that orders a thread's own copies.
__device__ __forceinline__ void cp_async_16(uint32_t smem_addr, const void* gptr) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint4 lds128_u32addr(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel of the stream drains.
// `griddep_wait` blocks until that kernel has completed and its memory is
// visible; everything a kernel reads that an earlier kernel may have written
// (activations) or writes that an earlier kernel may read (outputs) comes
// after it.  The packed weight is constant and may be read before it.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// D(16x8, f32) += A(16x16, f16, row) * B(16x8, f16, col)
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Scale words of one nibble pair (rows 2p, 2p+1) in the packed blob: a half2
// for fp16 scales (layout version 1, in .x) or a float2 for fp32 scales
// (version 2).  Returns them as two floats.
template <bool F32S>
__device__ __forceinline__ float2 scale_pair(uint2 w) {
  if (F32S) return make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
  const __half2 h = u32_as_h2(w.x);
  return make_float2(__low2float(h), __high2float(h));
}

// Tensor-core operand of two weights with fp32 scales (layout version 2):
// fp16_RNE(fp32_RNE((code - 8) * s)) for the exact integers c = code - 8.
__device__ __forceinline__ uint32_t weight_pair_f32s(__half2 c, float s_lo, float s_hi) {
  return h2_as_u32(__floats2half2_rn(__fmul_rn(__low2float(c), s_lo), __fmul_rn(__high2float(c), s_hi)));
}

// D(16x8, f32) = A(16x16, f16, row) * B(16x8, f16, col): the accumulator
// starts from zero (no register moves to clear it)
__device__ __forceinline__ void mma_16816_zero(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(0.f));
}

}  // namespace q4gsw
