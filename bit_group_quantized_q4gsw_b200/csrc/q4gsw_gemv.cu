// q4gsw_gemv.cu - tensor-core GEMV routes of the q4gsw linear layer for small
// token counts (M <= 16 per z-slice).
//
//   forward   y[m,n]   = sum_k x[m,k]     * (code[n,k] - 8) * s[k/gs, n]
//   backward  d_x[m,k] = sum_n d_out[m,n] * (code[n,k] - 8) * s[k/gs, n]
// ("[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward kernel (4-bit
// input-grad)", PR description: the input gradient contracts over N and reads
// the same packed weight as the forward).
//
// Both stream the packed weight once with 16-byte non-caching loads and feed
// mma.sync m16n8k16 (fp16 in, fp32 accumulate) straight from registers:
//  * forward: A = weight tile (16 output rows = 8 nibble pairs, 16 columns),
//    B = x^T (16 columns, 8 tokens).  Codes enter the MMA as exact integers
//    code - 8; the fp16 scale multiplies the fp32 partial sum of each group
//    (a group never straddles a 16-column step since gs >= 16), so the forward
//    GEMV carries no per-weight scale multiply.
//  * backward: A = d_out (16 tokens, 16 contraction rows n), B = weight^T
//    (16 n, 8 output columns k).  The scale varies along the contraction, so
//    each weight pair is scaled in fp16 (one rounding, as in the GEMM).
// The split of the contraction over CTAs is reduced through distributed shared
// memory inside a thread-block cluster: no atomics, no memset, deterministic.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cstdio>

#include "q4gsw_common.cuh"
#include "q4gsw_internal.h"

namespace cg = cooperative_groups;

namespace q4gsw {

constexpr int kGemvWarps = 4;
constexpr int kGemvThreads = 32 * kGemvWarps;

// ---------------------------------------------------------------------------
// Forward
// ---------------------------------------------------------------------------
// grid = (N/16 row tiles, S contraction splits, ceil(M/16) token slices),
// cluster = (1, S, 1).  Warp u = split*4 + warp owns the 64-column blocks
// [u*KB/U, (u+1)*KB/U) of its row tile (KB = K/64, U = 4 S).
// NT = number of 8-token MMA tiles (1: M <= 8 per slice, 2: M <= 16).
// SPG = 16-column steps per scale group (1: gs 16, 2: gs 32, 4: gs >= 64).
template <int NT, int SPG>
__global__ void __launch_bounds__(kGemvThreads) gemv_fwd_kernel(const uint8_t* __restrict__ packed,
                                                                const __half* __restrict__ x, OutSplit out,
                                                                int M, int N, int K, int gs) {
  __shared__ float red[kGemvWarps][16][16];  // [warp][token][row]
  __shared__ float cta_part[16][16];         // [token][row]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x;
  const int split = blockIdx.y, S = gridDim.y;
  const int tok0 = blockIdx.z * 16;
  const int Mz = min(16, M - tok0);

  const Layout L = layout_of(N, K, gs);
  const __half* scales = reinterpret_cast<const __half*>(packed + L.scales_offset);
  const int p_raw = tile * 8 + g;  // nibble pair of this lane: rows 2p (even) and 2p+1 (odd)
  const bool pvalid = p_raw < (N >> 1);  // the last tile holds 4 pairs when N % 16 == 8
  const int p = pvalid ? p_raw : 0;
  const uint8_t* row = packed + (size_t)p * K + 16 * t;

  const int KB = K >> 6;
  const int U = S * kGemvWarps, u = split * kGemvWarps + warp;
  const int b_begin = (int)((long long)u * KB / U), b_end = (int)((long long)(u + 1) * KB / U);

  // token rows this lane feeds into B (column g of each 8-token tile)
  const __half* xrow[NT];
  bool xvalid[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int tok = 8 * j + g;
    xvalid[j] = tok < Mz;
    xrow[j] = x + (size_t)(tok0 + (xvalid[j] ? tok : 0)) * K + 4 * t;
  }

  float acc[NT][4], part[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[j][c] = part[j][c] = 0.f;

  auto flush = [&](int col) {  // scale the group that holds column `col` into acc
    const __half2 s2 = *reinterpret_cast<const __half2*>(scales + (size_t)(col / gs) * N + 2 * p);
    const float se = __low2float(s2), so = __high2float(s2);
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      acc[j][0] = fmaf(part[j][0], se, acc[j][0]);
      acc[j][1] = fmaf(part[j][1], se, acc[j][1]);
      acc[j][2] = fmaf(part[j][2], so, acc[j][2]);
      acc[j][3] = fmaf(part[j][3], so, acc[j][3]);
      part[j][0] = part[j][1] = part[j][2] = part[j][3] = 0.f;
    }
  };

  constexpr int PF = 4;  // 64-column blocks in flight per lane
  for (int b0 = b_begin; b0 < b_end; b0 += PF) {
    uint4 wv[PF];
#pragma unroll
    for (int q = 0; q < PF; ++q)
      wv[q] = (b0 + q < b_end && pvalid) ? ldg_stream_v4(row + 64 * (b0 + q)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int q = 0; q < PF; ++q) {
      const int b = b0 + q;
      if (b >= b_end) break;
      const uint32_t words[4] = {wv[q].x, wv[q].y, wv[q].z, wv[q].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = 64 * b + 16 * i;  // first column of this 16-column step
        const RowPairs r = codes_minus8_rows(words[i]);
        const uint32_t a[4] = {h2_as_u32(r.ev01), h2_as_u32(r.od01), h2_as_u32(r.ev23), h2_as_u32(r.od23)};
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          uint2 xv = make_uint2(0u, 0u);
          if (xvalid[j]) xv = ldg_nc_v2(xrow[j] + col);
          const uint32_t bf[2] = {xv.x, xv.y};
          mma_16816(part[j], a, bf);
        }
        if (SPG == 1 || (SPG == 2 && (i & 1))) flush(col);
      }
      if (SPG == 4 && (((b + 1) * 64) % gs == 0 || b + 1 == b_end)) flush(64 * b);
    }
  }

  // D fragment: rows g (even n) and g+8 (odd n), tokens 2t, 2t+1 of tile j.
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    red[warp][8 * j + 2 * t][2 * g] = acc[j][0];
    red[warp][8 * j + 2 * t + 1][2 * g] = acc[j][1];
    red[warp][8 * j + 2 * t][2 * g + 1] = acc[j][2];
    red[warp][8 * j + 2 * t + 1][2 * g + 1] = acc[j][3];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 16 * 8 * NT; e += kGemvThreads) {
    const int tok = e >> 4, n = e & 15;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) s += red[w][tok][n];
    cta_part[tok][n] = s;
  }
  cg::cluster_group cluster = cg::this_cluster();
  if (S > 1) cluster.sync(); else __syncthreads();
  if (cluster.block_rank() == 0) {
    for (int e = threadIdx.x; e < 16 * Mz; e += kGemvThreads) {
      const int tok = e >> 4, nl = e & 15;
      float s = cta_part[tok][nl];
      for (int r = 1; r < S; ++r) s += cluster.map_shared_rank(&cta_part[0][0], r)[tok * 16 + nl];
      const int n = tile * 16 + nl;
      if (n >= N) continue;
      const size_t m = (size_t)(tok0 + tok);
      if (n < out.n1) out.y0[m * out.n1 + n] = s;
      else if (n < out.n2) out.y1[m * (out.n2 - out.n1) + (n - out.n1)] = s;
      else out.y2[m * (out.N - out.n2) + (n - out.n2)] = s;
    }
  }
  if (S > 1) cluster.sync();
}

// ---------------------------------------------------------------------------
// Backward (input gradient)
// ---------------------------------------------------------------------------
// grid = (ceil(K/128) column tiles, S contraction splits, ceil(M/16) token
// slices), cluster = (1, S, 1), kBwdWarps warps per CTA.  A column tile is two
// 64-column blocks J = 2*tile + (g >> 2); lane (g, t) reads 16 bytes at offset
// 16 (g & 3) of block J in pair rows pb+t and pb+t+4.  MMA (i, e) has output
// column c <-> k = 64 J(c) + 16 i + 4 (c & 3) + e.  Warp u = split*W + warp
// owns the 16-row contraction steps [u*NS/U, (u+1)*NS/U) (NS = N/16).
constexpr int kBwdWarps = 8;
constexpr int kBwdThreads = 32 * kBwdWarps;

template <int SPB>  // scale groups per 64-column block: 1 (gs >= 64), 2 (gs 32), 4 (gs 16)
__global__ void __launch_bounds__(kBwdThreads) gemv_bwd_kernel(const uint8_t* __restrict__ packed,
                                                               const __half* __restrict__ dout,
                                                               float* __restrict__ dx,
                                                               int M, int N, int K, int gs) {
  __shared__ float cta_part[16 * 128];  // [token][local column]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int split = blockIdx.y, S = gridDim.y;
  const int tok0 = blockIdx.z * 16;
  const int Mz = min(16, M - tok0);
  const int KB = K >> 6;
  const int J = 2 * blockIdx.x + (g >> 2);  // this lane's 64-column block
  const bool jvalid = J < KB;

  const Layout L = layout_of(N, K, gs);
  const __half* scales = reinterpret_cast<const __half*>(packed + L.scales_offset);
  const int NS = (N + 15) >> 4;   // the last step holds 4 pairs when N % 16 == 8
  const int NP = N >> 1;
  const int U = S * kBwdWarps, u = split * kBwdWarps + warp;
  const int s_begin = (int)((long long)u * NS / U), s_end = (int)((long long)(u + 1) * NS / U);

  // scale group of each 16-column step i of this lane's columns
  // (lanes past the last block use block 0: their columns are never stored)
  const int Jc = jvalid ? J : 0;
  int grp[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) grp[i] = (64 * Jc + 16 * i + 4 * (g & 3)) / gs;

  const bool tv0 = g < Mz, tv1 = g + 8 < Mz;
  const __half* drow0 = dout + (size_t)(tok0 + (tv0 ? g : 0)) * N;
  const __half* drow1 = dout + (size_t)(tok0 + (tv1 ? g + 8 : 0)) * N;
  const uint8_t* wcol = packed + 64 * Jc + 16 * (g & 3);

  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][e][c] = 0.f;

  for (int st = s_begin; st < s_end; ++st) {
    const int pA = st * 8 + t;
    const bool bvalid = pA + 4 < NP;
    const int pB = bvalid ? pA + 4 : pA;
    uint4 va = make_uint4(0, 0, 0, 0), vb = make_uint4(0, 0, 0, 0);
    if (jvalid) {
      va = ldg_stream_v4(wcol + (size_t)pA * K);
      if (bvalid) vb = ldg_stream_v4(wcol + (size_t)pB * K);
    }
    uint32_t a[4] = {0u, 0u, 0u, 0u};
    if (tv0) {
      a[0] = ldg_nc_u32(drow0 + 2 * pA);
      if (bvalid) a[2] = ldg_nc_u32(drow0 + 2 * pB);
    }
    if (tv1) {
      a[1] = ldg_nc_u32(drow1 + 2 * pA);
      if (bvalid) a[3] = ldg_nc_u32(drow1 + 2 * pB);
    }
    __half2 sa[SPB], sb[SPB];
#pragma unroll
    for (int q = 0; q < SPB; ++q) {
      const int gq = grp[q * (4 / SPB)];
      sa[q] = u32_as_h2(ldg_nc_u32(scales + (size_t)gq * N + 2 * pA));
      sb[q] = bvalid ? u32_as_h2(ldg_nc_u32(scales + (size_t)gq * N + 2 * pB)) : u32_as_h2(0u);
    }
    const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
    const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = i / (4 / SPB);
      const ColPairs ca = codes_minus8_cols(wa[i]);
      const ColPairs cb = codes_minus8_cols(wb[i]);
      const __half2 la[4] = {ca.c0, ca.c1, ca.c2, ca.c3};
      const __half2 lb[4] = {cb.c0, cb.c1, cb.c2, cb.c3};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t bf[2] = {h2_as_u32(__hmul2(la[e], sa[q])), h2_as_u32(__hmul2(lb[e], sb[q]))};
        mma_16816(acc[i][e], a, bf);
      }
    }
  }

  // D fragment of MMA (i, e): rows g / g+8 = tokens, columns 2t, 2t+1;
  // column c -> local output column 64 (c >> 2) + 16 i + 4 (c & 3) + e.
  // Warps add their partials into cta_part one after another (fixed order).
  for (int w = 0; w < kBwdWarps; ++w) {
    if (warp == w) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = 2 * t + h;
            const int kl = 64 * (c >> 2) + 16 * i + 4 * (c & 3) + e;
            if (w == 0) {
              cta_part[g * 128 + kl] = acc[i][e][h];
              cta_part[(g + 8) * 128 + kl] = acc[i][e][2 + h];
            } else {
              cta_part[g * 128 + kl] += acc[i][e][h];
              cta_part[(g + 8) * 128 + kl] += acc[i][e][2 + h];
            }
          }
    }
    __syncthreads();
  }
  cg::cluster_group cluster = cg::this_cluster();
  if (S > 1) cluster.sync();
  if (cluster.block_rank() == 0) {
    const int kbase = 128 * blockIdx.x;
    const int kw = min(128, K - kbase);
    for (int idx = threadIdx.x; idx < Mz * 128; idx += kBwdThreads) {
      const int tok = idx >> 7, kl = idx & 127;
      if (kl >= kw) continue;
      float s = cta_part[idx];
      for (int r = 1; r < S; ++r) s += cluster.map_shared_rank(cta_part, r)[idx];
      dx[(size_t)(tok0 + tok) * K + kbase + kl] = s;
    }
  }
  if (S > 1) cluster.sync();
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
static int sm_count() {
  static int cached = 0;
  if (!cached) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached = n > 0 ? n : 148;
  }
  return cached;
}

// Contraction splits: grow S (cluster size) until the grid holds about
// `warps_target` warps, keeping at least `min_units` contraction units per warp.
static int pick_splits(long long tiles, int warps_per_cta, int units_per_tile, int min_units, int max_s,
                       long long warps_target) {
  int S = 1;
  while (S * 2 <= max_s && tiles * S * warps_per_cta < warps_target &&
         units_per_tile / (warps_per_cta * S * 2) >= min_units)
    S *= 2;
  return S;
}

template <typename Kern, typename... Args>
static cudaError_t launch_cluster(Kern kernel, dim3 grid, int threads, int cluster_y, size_t smem,
                                  cudaStream_t stream, Args... args) {
  if (cluster_y > 8) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = cluster_y;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_gemv_fwd(const void* packed, int N, int K, int gs, const uint16_t* x, int M,
                            OutSplit out, cudaStream_t stream, char* route, int route_len) {
  const int tiles = (N + 15) / 16;
  const int S = pick_splits(tiles, kGemvWarps, K / 64, 1, 8, 24LL * sm_count());
  const int NT = (M <= 8) ? 1 : 2;
  const int spg = gs == 16 ? 1 : gs == 32 ? 2 : 4;
  dim3 grid(tiles, S, (M + 15) / 16);
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  const __half* xh = reinterpret_cast<const __half*>(x);
  cudaError_t err;
#define Q4_FWD(NT_, SPG_) \
  err = launch_cluster(gemv_fwd_kernel<NT_, SPG_>, grid, kGemvThreads, S, 0, stream, pk, xh, out, M, N, K, gs)
  if (NT == 1) {
    if (spg == 1) Q4_FWD(1, 1); else if (spg == 2) Q4_FWD(1, 2); else Q4_FWD(1, 4);
  } else {
    if (spg == 1) Q4_FWD(2, 1); else if (spg == 2) Q4_FWD(2, 2); else Q4_FWD(2, 4);
  }
#undef Q4_FWD
  if (route) snprintf(route, route_len, "gemv_fwd launches=1 nt=%d splits=%d zslices=%d", NT, S, (M + 15) / 16);
  return err;
}

cudaError_t launch_gemv_bwd(const void* packed, int N, int K, int gs, const uint16_t* d_out, int M,
                            float* d_x, cudaStream_t stream, char* route, int route_len) {
  const int tiles = (K + 127) / 128;
  const int S = pick_splits(tiles, kBwdWarps, (N + 15) / 16, 2, 16, 24LL * sm_count());
  const int spb = gs >= 64 ? 1 : gs == 32 ? 2 : 4;
  dim3 grid(tiles, S, (M + 15) / 16);
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  const __half* dh = reinterpret_cast<const __half*>(d_out);
  cudaError_t err;
#define Q4_BWD(SPB_) \
  err = launch_cluster(gemv_bwd_kernel<SPB_>, grid, kBwdThreads, S, 0, stream, pk, dh, d_x, M, N, K, gs)
  if (spb == 1) Q4_BWD(1); else if (spb == 2) Q4_BWD(2); else Q4_BWD(4);
#undef Q4_BWD
  if (route) snprintf(route, route_len, "gemv_bwd launches=1 splits=%d zslices=%d", S, (M + 15) / 16);
  return err;
}

}  // namespace q4gsw
