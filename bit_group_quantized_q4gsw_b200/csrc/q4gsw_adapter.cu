// q4gsw_adapter.cu - the low-rank intermediate of the frozen-base adapter step.
//
// The q4gsw input gradient exists for on-device adapter training on a frozen
// 4-bit base ("[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward kernel
// (4-bit input-grad)", PR description).  With a rank-r adapter beside the base,
//   forward    y   = x dequant(W)^T + (x A^T) B^T      A fp16 [r, K], B fp16 [N, r]
//   backward   d_x = d_out dequant(W) + (d_out B) A
// this file computes the intermediate u = x A^T (forward) or v = d_out B
// (backward), [M][r] with fp32 accumulation, rounded to fp16 and stored as
// rows of 64 halves (columns r..63 zero) in the caller's workspace.  The GEMM
// then adds u B^T (or v A) as one more 64-deep contraction stage of its
// accumulator.
//
// A cluster of KS CTAs per 16 tokens splits the contraction (KS <= 8, chosen
// to give the launch about two CTAs per SM); the eight warps of a CTA split its
// slice again, each running mma.sync m16n8k16 (A = 16 tokens x 16 contraction
// indices of the activation, B = 16 contraction indices x 8 rank columns of the
// projection).  The eight warp tiles are summed in shared memory, and each CTA
// stores its sums of token rows [16 rk / KS, 16 (rk + 1) / KS) into rank rk's
// receive slot for it (distributed shared memory); after one cluster barrier
// rank rk adds its KS slots, both sums in a fixed order.
//
// The kernel moves a few megabytes, so its time is latencies: a warp issues
// every load of up to two of its 64-column chunks (activations, then the
// projection's fragments) before the first MMA, and the cluster barrier that must precede the first remote store (every
// CTA of the cluster running) is arrived at on entry and waited for only there.
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "q4gsw_common.cuh"
#include "q4gsw_internal.h"

namespace q4gsw {
namespace ad {
namespace cg = cooperative_groups;

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kRankMax = 64;

// Cluster-wide barrier: arrive with release, wait with acquire.
__device__ __forceinline__ void cluster_barrier_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// act [M][C] fp16 row-major; the projection P(c, j) is proj[j * C + c] when
// BY_ROWS (forward: A [r, C]) or proj[c * r + j] (backward: B [C, r]).
__device__ __forceinline__ uint4 ldg_nc_v4h(const __half* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// NJ: 8-column rank tiles held per lane (2, 4 or 8: ranks up to 16, 32, 64)
template <bool BY_ROWS, int NJ>
__global__ void __launch_bounds__(kThreads)
q4gsw_adapter_proj_kernel(const __half* __restrict__ act, const __half* __restrict__ proj, __half* __restrict__ out,
                          int M, int C, int r) {
  __shared__ float red[kWarps][16][kRankMax];
  __shared__ float recv[8][8][kRankMax];   // [sender rank][owned row][rank column], KS >= 2: <= 8 rows owned
  const int KS = gridDim.y, ks = blockIdx.y;
  if (KS > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  griddep_launch_dependents();
  griddep_wait();   // the activations may come from the previous kernel of the stream
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int m0 = blockIdx.x * 16;
  const int chunks = (C + 63) / 64;   // 64-column chunks; C % 8 == 0, so an 8-column group is wholly in or out
  const int c_begin = ks * chunks / KS, c_end = (ks + 1) * chunks / KS;
  const int s_begin = c_begin + warp * (c_end - c_begin) / kWarps;
  const int s_end = c_begin + (warp + 1) * (c_end - c_begin) / kWarps;
  const int nj = (r + 7) / 8;  // 8-column rank tiles
  // rows past M read row M - 1 (never stored)
  const __half* a0 = act + (size_t)min(m0 + g, M - 1) * C;
  const __half* a1 = act + (size_t)min(m0 + g + 8, M - 1) * C;
  float acc[NJ][4];
#pragma unroll
  for (int jt = 0; jt < NJ; ++jt)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[jt][c] = 0.f;
  auto pval = [&](int c, int j) -> uint32_t {   // P(c, j) as fp16 bits, zero past the rank
    if (j >= r) return 0u;
    const __half v = BY_ROWS ? proj[(size_t)j * C + c] : proj[(size_t)c * r + j];
    return __half_as_ushort(v);
  };
  // Chunk of 64 columns: lane t loads columns c0 + 16 t .. + 15 of its two
  // token rows as two 16-byte vectors each, and MMA step s (0..3) takes the
  // column pairs (16 t + 2 s, + 1) as contraction indices (2t, 2t + 1) and
  // (16 t + 8 + 2 s, + 1) as (2t + 8, 2t + 9).  The permutation depends on t
  // only, so the projection's fragments follow it (16-byte loads of A's rows
  // in the forward).  Every load of a chunk is issued before its MMAs.
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
  constexpr int NB = NJ <= 2 ? 2 : 1;   // chunks whose activations are loaded together (register budget)
  for (int ch0 = s_begin; ch0 < s_end; ch0 += NB) {
    // the activation vectors of chunks ch0 .. ch0 + NB - 1 (those in this
    // warp's range): rows g and g + 8, columns c0 .. c0 + 7 and c0 + 8 .. c0 + 15
    uint4 xv[NB][4];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int c0 = 64 * (ch0 + b) + 16 * t;
      const bool live = ch0 + b < s_end;
      const bool in0 = live && c0 + 8 <= C, in1 = live && c0 + 16 <= C;
      xv[b][0] = in0 ? ldg_nc_v4h(a0 + c0) : z4;
      xv[b][1] = in1 ? ldg_nc_v4h(a0 + c0 + 8) : z4;
      xv[b][2] = in0 ? ldg_nc_v4h(a1 + c0) : z4;
      xv[b][3] = in1 ? ldg_nc_v4h(a1 + c0 + 8) : z4;
    }
    uint4 p[NB][NJ][2];   // projection column j = 8 jt + g at the same columns
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int c0 = 64 * (ch0 + b) + 16 * t;
      const bool live = ch0 + b < s_end;
      const bool in0 = live && c0 + 8 <= C, in1 = live && c0 + 16 <= C;
#pragma unroll
      for (int jt = 0; jt < NJ; ++jt) {
        const int j = 8 * jt + g;
        if (live && jt < nj && j < r) {
          if (BY_ROWS) {
            p[b][jt][0] = in0 ? ldg_nc_v4h(proj + (size_t)j * C + c0) : z4;
            p[b][jt][1] = in1 ? ldg_nc_v4h(proj + (size_t)j * C + c0 + 8) : z4;
          } else {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int c = c0 + 2 * (e & 3) + 8 * (e >> 2);
              w[e] = c + 2 <= C ? pval(c, j) | (pval(c + 1, j) << 16) : 0u;
            }
            p[b][jt][0] = make_uint4(w[0], w[1], w[2], w[3]);
            p[b][jt][1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        } else {
          p[b][jt][0] = p[b][jt][1] = z4;
        }
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (ch0 + b >= s_end) break;
      const uint32_t* r0 = reinterpret_cast<const uint32_t*>(&xv[b][0]);   // row g: columns c0 .. c0 + 15
      const uint32_t* r1 = reinterpret_cast<const uint32_t*>(&xv[b][2]);   // row g + 8
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        const uint32_t af[4] = {r0[st], r1[st], r0[4 + st], r1[4 + st]};
#pragma unroll
        for (int jt = 0; jt < NJ; ++jt) {
          if (jt >= nj) break;
          const uint32_t* pj = reinterpret_cast<const uint32_t*>(p[b][jt]);
          const uint32_t bf[2] = {pj[st], pj[4 + st]};
          mma_16816(acc[jt], af, bf);
        }
      }
    }
  }
  // D fragment: rows g, g + 8 (tokens), columns 2t, 2t + 1 of rank tile jt.
  // Only the JW = 8 NJ columns that can hold a rank are summed; the rest of
  // each 64-half workspace row is written as zeros.
  constexpr int JW = 8 * NJ;
#pragma unroll
  for (int jt = 0; jt < NJ; ++jt) {
    red[warp][g][8 * jt + 2 * t] = acc[jt][0];
    red[warp][g][8 * jt + 2 * t + 1] = acc[jt][1];
    red[warp][g + 8][8 * jt + 2 * t] = acc[jt][2];
    red[warp][g + 8][8 * jt + 2 * t + 1] = acc[jt][3];
  }
  __syncthreads();
  auto store_row_tail = [&](int m) {   // columns JW .. 63 of output row m: zeros
    for (int j = JW + (threadIdx.x & 31); j < kRankMax; j += 32) out[(size_t)m * kRankMax + j] = __float2half_rn(0.f);
  };
  if (KS == 1) {
    for (int e = threadIdx.x; e < 16 * JW; e += kThreads) {
      const int row = e / JW, j = e % JW;
      if (m0 + row >= M) continue;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += red[w][row][j];
      out[(size_t)(m0 + row) * kRankMax + j] = j < r ? __float2half_rn(s) : __float2half_rn(0.f);
    }
    if (JW < kRankMax)
      for (int row = threadIdx.x >> 5; row < 16; row += kWarps)
        if (m0 + row < M) store_row_tail(m0 + row);
    return;
  }
  // every CTA of the cluster has started (arrived on entry): remote stores are safe
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  cg::cluster_group cluster = cg::this_cluster();
  for (int e = threadIdx.x; e < 16 * JW; e += kThreads) {
    const int row = e / JW, j = e % JW;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[w][row][j];
    const int owner = ((row + 1) * KS - 1) / 16;   // largest rank with rank * 16 / KS <= row
    const int ob = owner * 16 / KS;
    *cluster.map_shared_rank(&recv[ks][row - ob][j], owner) = s;
  }
  cluster_barrier_sync();   // every CTA's rows delivered
  const int rb = ks * 16 / KS, re = (ks + 1) * 16 / KS;
  for (int e = threadIdx.x; e < (re - rb) * JW; e += kThreads) {
    const int row = e / JW, j = e % JW;
    if (m0 + rb + row >= M) continue;
    float s = 0.f;
    for (int q = 0; q < KS; ++q) s += recv[q][row][j];
    out[(size_t)(m0 + rb + row) * kRankMax + j] = j < r ? __float2half_rn(s) : __float2half_rn(0.f);
  }
  if (JW < kRankMax)
    for (int row = rb + (threadIdx.x >> 5); row < re; row += kWarps)
      if (m0 + row < M) store_row_tail(m0 + row);
}

}  // namespace ad

// Scratch of the allocation-free adapter entry point (q4gsw_adapter_fwd_noalloc):
// the intermediate [M][64] fp16 of one call, M <= kNoAllocScratchBytes / 128.
// It is a fixed array in the library's device image, so every GPU that loads
// the library holds it until the process exits, and every call shares it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

cudaError_t noalloc_scratch(void** ptr, size_t* bytes) {
  // In host code the array's name is only a stand-in for the symbol, never a
  // device address: its address on the current device is looked up once per
  // device (with that device current) and reused.
  static std::once_flag once[kMaxDevices];
  static void* addr[kMaxDevices];
  static cudaError_t err[kMaxDevices];
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] { err[dev] = cudaGetSymbolAddress(&addr[dev], g_noalloc_scratch); });
  if (err[dev] != cudaSuccess) return err[dev];
  *ptr = addr[dev];
  *bytes = kNoAllocScratchBytes;
  return cudaSuccess;
}

cudaError_t launch_adapter_proj(const uint16_t* act, const uint16_t* proj, bool by_rows, int M, int C, int r,
                                void* workspace, cudaStream_t stream) {
  // contraction splits: about two CTAs per SM, at least one 64-column chunk
  // per warp, clusters of at most 8
  const int tiles = (M + 15) / 16;
  const int chunks = (C + 63) / 64;
  int KS = (2 * sm_count(current_device()) + tiles - 1) / tiles;
  KS = KS > 8 ? 8 : KS;
  while (KS > 1 && chunks / KS < ad::kWarps) --KS;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles, KS, 1);
  cfg.blockDim = dim3(ad::kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = KS;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const __half* a = reinterpret_cast<const __half*>(act);
  const __half* p = reinterpret_cast<const __half*>(proj);
  __half* o = static_cast<__half*>(workspace);
  const int nj = (r + 7) / 8;
#define Q4_PROJ(BR, NJ_) cudaLaunchKernelEx(&cfg, ad::q4gsw_adapter_proj_kernel<BR, NJ_>, a, p, o, M, C, r)
  if (by_rows) return nj <= 2 ? Q4_PROJ(true, 2) : nj <= 4 ? Q4_PROJ(true, 4) : Q4_PROJ(true, 8);
  return nj <= 2 ? Q4_PROJ(false, 2) : nj <= 4 ? Q4_PROJ(false, 4) : Q4_PROJ(false, 8);
#undef Q4_PROJ
}

}  // namespace q4gsw
