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

#include <cmath>
#include <cstdio>

#include "q4gsw_common.cuh"
#include "q4gsw_internal.h"

namespace cg = cooperative_groups;

namespace q4gsw {
namespace rg {

constexpr int kGemvWarps = 4;
constexpr int kGemvThreads = 32 * kGemvWarps;

// ---------------------------------------------------------------------------
// Forward
// ---------------------------------------------------------------------------
// grid = (ceil(N/16) row tiles, S contraction splits, ceil(M/16) token
// slices), cluster = (1, S, 1).  Warp u = split*4 + warp owns the 64-column
// blocks [u*KB/U, (u+1)*KB/U) of its row tile (KB = K/64, U = 4 S).
// NT = number of 8-token MMA tiles (1: M <= 8 per slice, 2: M <= 16).
// SPG = 16-column steps per scale group (1: gs 16, 2: gs 32, 4: gs >= 64).
template <int NT, int SPG, bool F32S>
__global__ void __launch_bounds__(kGemvThreads, NT == 1 ? 7 : 4)
q4gsw_gemv_fwd_reg_kernel(const uint8_t* __restrict__ packed, const __half* __restrict__ x, OutSplit out, int M, int N,
                int K, int gs) {
  __shared__ float red[kGemvWarps][16][16];  // [warp][token][row]
  __shared__ float cta_part[16][16];         // [token][row]
  griddep_launch_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x;
  const int split = blockIdx.y, S = gridDim.y;
  const int tok0 = blockIdx.z * 16;
  const int Mz = min(16, M - tok0);

  const Layout L = layout_of(N, K, gs, F32S ? 4 : 2);
  const int gsl = __ffs(gs) - 1;  // gs is a power of two
  const int p_raw = tile * 8 + g;  // nibble pair of this lane: rows 2p (even) and 2p+1 (odd)
  const bool pvalid = p_raw < (N >> 1);  // the last tile holds 4 pairs when N % 16 == 8
  const int p = pvalid ? p_raw : 0;
  const uint8_t* row = packed + (size_t)p * K + 16 * t;

  const int KB = K >> 6;
  const int U = S * kGemvWarps, u = split * kGemvWarps + warp;
  const int b_begin = (int)((long long)u * KB / U), b_end = (int)((long long)(u + 1) * KB / U);

  // Two partial-sum sets (even / odd 16-column steps) keep two independent
  // MMA chains in flight; a finished group is scaled into acc in fp32.
  float acc[NT][4], part[2][NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[j][c] = part[0][j][c] = part[1][j][c] = 0.f;

  auto flush = [&](uint2 s_word) {  // scale one finished group into acc
    const float2 sp = scale_pair<F32S>(s_word);
    const float se = sp.x, so = sp.y;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      acc[j][0] = fmaf(part[0][j][0] + part[1][j][0], se, acc[j][0]);
      acc[j][1] = fmaf(part[0][j][1] + part[1][j][1], se, acc[j][1]);
      acc[j][2] = fmaf(part[0][j][2] + part[1][j][2], so, acc[j][2]);
      acc[j][3] = fmaf(part[0][j][3] + part[1][j][3], so, acc[j][3]);
#pragma unroll
      for (int c = 0; c < 4; ++c) part[0][j][c] = part[1][j][c] = 0.f;
    }
  };

  // Lanes whose rows or tokens do not exist read valid memory (row 0, token
  // 0) and their results are never stored, so no load is predicated.  x rows
  // of this lane: token 8j + g feeds column g of 8-token tile j.
  const __half* xrow[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int tok = 8 * j + g;
    xrow[j] = x + (size_t)(tok0 + (tok < Mz ? tok : 0)) * K + 4 * t;
  }
  constexpr int NGB = (SPG == 4) ? 1 : 4 / SPG;            // scale groups per block
  const int bpg_mask = (SPG == 4) ? (gs >> 6) - 1 : 0;      // blocks per group - 1 (gs >= 64)
  // scale words of pair p: half2 (fp16 scales) or float2 (fp32 scales), one row per group
  const uint8_t* srow = packed + L.scales_offset + (size_t)(F32S ? 8 : 4) * p;
  const size_t srow_stride = (size_t)(F32S ? 4 : 2) * N;

  // One 64-column block of this lane: packed word quad, scale words, x fragments.
  struct Blk {
    uint4 w;
    uint2 s[NGB];
    uint2 xv[NT][4];
  };
  const int b_last = b_end - 1;
  auto load_w = [&](int b, Blk& d) {
    b = min(b, b_last);
    d.w = ldg_stream_v4(row + 64 * b);
#pragma unroll
    for (int r = 0; r < NGB; ++r) {
      const uint8_t* sp = srow + (size_t)((64 * b + r * (64 / NGB)) >> gsl) * srow_stride;
      d.s[r] = F32S ? ldg_nc_v2(sp) : make_uint2(ldg_nc_u32(sp), 0u);
    }
  };
  auto load_x = [&](int b, Blk& d) {
    b = min(b, b_last);
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) d.xv[j][i] = ldg_nc_v2(xrow[j] + 64 * b + 16 * i);
  };
  auto compute = [&](int b, const Blk& d) {
    const uint32_t words[4] = {d.w.x, d.w.y, d.w.z, d.w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const RowPairs r = codes_minus8_rows(words[i]);
      const uint32_t a[4] = {h2_as_u32(r.ev01), h2_as_u32(r.od01), h2_as_u32(r.ev23), h2_as_u32(r.od23)};
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const uint32_t bf[2] = {d.xv[j][i].x, d.xv[j][i].y};
        mma_16816(part[i & 1][j], a, bf);
      }
      if (SPG == 1) flush(d.s[i]);
      if (SPG == 2 && (i & 1)) flush(d.s[i >> 1]);
    }
    if (SPG == 4 && (((b + 1) & bpg_mask) == 0 || b == b_last)) flush(d.s[0]);
  };

  // Three blocks rotate through three register sets (no copies): while one
  // block is dequantised and multiplied, the next two are in flight.  The
  // packed weight is constant, so its first loads precede the wait for the
  // previous kernel of the stream (which may produce x).
  if (b_begin < b_end) {
    Blk A, B, C;
    load_w(b_begin, A);
    load_w(b_begin + 1, B);
    load_w(b_begin + 2, C);
    griddep_wait();
    load_x(b_begin, A);
    load_x(b_begin + 1, B);
    load_x(b_begin + 2, C);
    for (int b = b_begin; b < b_end; b += 3) {
      compute(b, A);
      if (b + 1 >= b_end) break;
      load_w(b + 3, A);
      load_x(b + 3, A);
      compute(b + 1, B);
      if (b + 2 >= b_end) break;
      load_w(b + 4, B);
      load_x(b + 4, B);
      compute(b + 2, C);
      load_w(b + 5, C);
      load_x(b + 5, C);
    }
  } else {
    griddep_wait();
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
// MMA roles: A = weight^T tile (16 output columns k x 16 contraction rows n =
// 8 nibble pairs; a register holds the (even n, odd n) half2 of ONE byte),
// B = d_out^T (16 n x 8 tokens), D = 16 k x 8 tokens.
// grid = (ceil(K/128) column tiles, S contraction splits, ceil(M/16) token
// slices), cluster = (1, S, 1), kBwdWarps warps per CTA.  A column tile is two
// 64-column blocks J = 2*tile + (g >> 2); lane (g, t) reads 16 bytes at offset
// 16 (g & 3) of block J in pair rows pb+t and pb+t+4, i.e. columns
// k = 64 J + 16 i + 4 (g & 3) + e.  MMA q = 2 i + h maps A row g to
// e = 2h and row g+8 to e = 2h+1.  Warp u = split*W + warp owns the 16-row
// contraction steps [u*NS/U, (u+1)*NS/U) (NS = N/16); the next step's loads are
// issued before the current step is computed.
constexpr int kBwdWarps = 8;
constexpr int kBwdThreads = 32 * kBwdWarps;

template <int NT, int SPB, bool F32S>  // NT 8-token tiles; SPB scale groups per block: 1 (gs >= 64), 2 (gs 32), 4 (gs 16)
__global__ void __launch_bounds__(kBwdThreads) q4gsw_gemv_bwd_reg_kernel(const uint8_t* __restrict__ packed,
                                                               const __half* __restrict__ dout,
                                                               float* __restrict__ dx,
                                                               int M, int N, int K, int gs) {
  extern __shared__ float red[];   // [warp][8 NT tokens][128 local columns]
  float* cta_part = red;           // reused after the warp partials are summed (rank 0 reads peers' copies)
  griddep_launch_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int split = blockIdx.y, S = gridDim.y;
  const int tok0 = blockIdx.z * 16;
  const int Mz = min(16, M - tok0);
  const int KB = K >> 6;
  const int J = 2 * blockIdx.x + (g >> 2);  // this lane's 64-column block
  const bool jvalid = J < KB;
  const int Jc = jvalid ? J : 0;            // lanes past the last block read block 0, never stored

  const Layout L = layout_of(N, K, gs, F32S ? 4 : 2);
  const uint8_t* scales = packed + L.scales_offset;
  const size_t sstride = (size_t)(F32S ? 4 : 2) * N;   // bytes per scale row
  const int NS = (N + 15) >> 4;   // the last step holds 4 pairs when N % 16 == 8
  const int NP = N >> 1;
  const int U = S * kBwdWarps, u = split * kBwdWarps + warp;
  const int s_begin = (int)((long long)u * NS / U), s_end = (int)((long long)(u + 1) * NS / U);

  int grp[SPB];   // scale group of the columns of step i (i = q * 4 / SPB .. )
#pragma unroll
  for (int q = 0; q < SPB; ++q) grp[q] = (64 * Jc + 16 * (q * (4 / SPB)) + 4 * (g & 3)) >> (__ffs(gs) - 1);

  // Rows, blocks and tokens that do not exist are read from valid places
  // (token 0, block 0, pair pA) and their results are never stored; only the
  // second pair of a ragged last step (N % 16 == 8) is zeroed explicitly.
  const __half* drow[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) drow[j] = dout + (size_t)(tok0 + (8 * j + g < Mz ? 8 * j + g : 0)) * N;
  const uint8_t* wcol = packed + 64 * Jc + 16 * (g & 3);

  float acc[NT][8][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[j][q][c] = 0.f;

  struct StepData {
    uint4 va, vb;              // packed bytes of pairs pA and pB
    uint32_t b[NT][2];         // d_out fragments
    uint2 sa[SPB], sb[SPB];    // scale words of pairs pA, pB per group
  };
  const int s_last = s_end - 1;
  auto load_step = [&](int st, StepData& d) {
    const int pA = st * 8 + t;
    const bool bvalid = pA + 4 < NP;
    const int pB = bvalid ? pA + 4 : pA;
    d.va = ldg_stream_v4(wcol + (size_t)pA * K);
    d.vb = ldg_stream_v4(wcol + (size_t)pB * K);
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      d.b[j][0] = ldg_nc_u32(drow[j] + 2 * pA);
      const uint32_t v = ldg_nc_u32(drow[j] + 2 * pB);
      d.b[j][1] = bvalid ? v : 0u;
    }
#pragma unroll
    for (int q = 0; q < SPB; ++q) {
      const uint8_t* ra = scales + (size_t)grp[q] * sstride + (size_t)(F32S ? 8 : 4) * pA;
      const uint8_t* rb = scales + (size_t)grp[q] * sstride + (size_t)(F32S ? 8 : 4) * pB;
      d.sa[q] = F32S ? ldg_nc_v2(ra) : make_uint2(ldg_nc_u32(ra), 0u);
      const uint2 v = F32S ? ldg_nc_v2(rb) : make_uint2(ldg_nc_u32(rb), 0u);
      d.sb[q] = bvalid ? v : make_uint2(0u, 0u);
    }
  };
  auto compute_step = [&](const StepData& d) {
    const uint32_t wa[4] = {d.va.x, d.va.y, d.va.z, d.va.w};
    const uint32_t wb[4] = {d.vb.x, d.vb.y, d.vb.z, d.vb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = i / (4 / SPB);
      const ColPairs ca = codes_minus8_cols(wa[i]);
      const ColPairs cb = codes_minus8_cols(wb[i]);
      const __half2 la[4] = {ca.c0, ca.c1, ca.c2, ca.c3};
      const __half2 lb[4] = {cb.c0, cb.c1, cb.c2, cb.c3};
      auto op = [&](__half2 c, uint2 sw) -> uint32_t {   // one byte's (even n, odd n) weights, scaled
        if (F32S) return weight_pair_f32s(c, __uint_as_float(sw.x), __uint_as_float(sw.y));
        return h2_as_u32(__hmul2(c, u32_as_h2(sw.x)));
      };
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t af[4] = {op(la[2 * h], d.sa[q]), op(la[2 * h + 1], d.sa[q]), op(lb[2 * h], d.sb[q]),
                                op(lb[2 * h + 1], d.sb[q])};
#pragma unroll
        for (int j = 0; j < NT; ++j) mma_16816(acc[j][2 * i + h], af, d.b[j]);
      }
    }
  };

  // d_out may come from the previous kernel of the stream: wait before the
  // first load (the step loads mix weights and d_out).
  griddep_wait();
  if (s_begin < s_end) {
    StepData dA, dB;
    load_step(s_begin, dA);
    for (int st = s_begin; st < s_end; st += 2) {
      load_step(min(st + 1, s_last), dB);
      compute_step(dA);
      if (st + 1 >= s_end) break;
      load_step(min(st + 2, s_last), dA);
      compute_step(dB);
    }
  }

  // Warp partials -> shared memory: D of MMA q = 2i + h, rows g / g+8 = columns
  // 64 (g >> 2) + 16 i + 4 (g & 3) + 2h (+1), columns 2t, 2t+1 = tokens.
  float* mine = red + warp * (8 * NT * 128);
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = q >> 1, h = q & 1;
      const int kl = 64 * (g >> 2) + 16 * i + 4 * (g & 3) + 2 * h;
      const int tk = 8 * j + 2 * t;
      mine[tk * 128 + kl] = acc[j][q][0];
      mine[(tk + 1) * 128 + kl] = acc[j][q][1];
      mine[tk * 128 + kl + 1] = acc[j][q][2];
      mine[(tk + 1) * 128 + kl + 1] = acc[j][q][3];
    }
  __syncthreads();
  float sums[8 * NT * 128 / kBwdThreads];
#pragma unroll
  for (int r = 0; r < 8 * NT * 128 / kBwdThreads; ++r) {
    const int idx = threadIdx.x + r * kBwdThreads;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kBwdWarps; ++w) s += red[w * (8 * NT * 128) + idx];
    sums[r] = s;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 8 * NT * 128 / kBwdThreads; ++r) cta_part[threadIdx.x + r * kBwdThreads] = sums[r];
  cg::cluster_group cluster = cg::this_cluster();
  if (S > 1) cluster.sync(); else __syncthreads();
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

}  // namespace rg

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
using rg::kGemvWarps;
using rg::kGemvThreads;
using rg::kBwdWarps;
using rg::kBwdThreads;
// Contraction splits S (the cluster size), from measurements on B200 over the
// decode, MLP and 8B-layer shapes: the forward wants about six CTAs per SM and
// no split that leaves a large weight's warps with fewer than 8 blocks; the
// input gradient, whose output tile is narrow, wants about 320 CTAs.
static int fwd_splits(long long tiles, int blocks_per_tile, size_t weight_bytes) {
  int S = (int)lround(6.0 * sm_count(current_device()) / (double)tiles);
  S = S < 1 ? 1 : S > 8 ? 8 : S;
  // a large weight keeps at least 8 blocks (a few pipeline turns) per warp
  const int min_blocks = weight_bytes >= ((size_t)16 << 20) ? 8 : 1;
  while (S > 1 && blocks_per_tile / (kGemvWarps * S) < min_blocks) --S;
  return S;
}

static int bwd_splits(long long tiles, int steps_per_tile, int warps_per_cta) {
  int S = (int)lround(320.0 / (double)tiles);
  S = S < 1 ? 1 : S > 16 ? 16 : S;
  while (S > 1 && steps_per_tile / (warps_per_cta * S) < 2) --S;
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
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = cluster_y;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Route between the two forward GEMVs: the TMA-ring kernel by default; the
// register-fed kernel only when q4gsw_debug_pin_routes pins it.
static bool use_reg_gemv() { return route_pins().gemv == kGemvReg; }

cudaError_t launch_gemv_fwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* x, int M,
                            OutSplit out, cudaStream_t stream, char* route, int route_len) {
  if (!use_reg_gemv()) return launch_gemv_tma_fwd(packed, N, K, gs, f32s, x, M, out, stream, route, route_len);
  const int tiles = (N + 15) / 16;
  const int zs = (M + 15) / 16;
  const int NT = (M <= 8) ? 1 : 2;
  const int spg = gs == 16 ? 1 : gs == 32 ? 2 : 4;
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  const __half* xh = reinterpret_cast<const __half*>(x);
  cudaError_t err;
  int S = 1;
#define Q4_FWD(NT_, SPG_)                                                                                        \
  do {                                                                                                           \
    S = fwd_splits((long long)tiles * zs, K / 64, (size_t)N * K / 2);                                            \
    err = f32s ? launch_cluster(rg::q4gsw_gemv_fwd_reg_kernel<NT_, SPG_, true>, dim3(tiles, S, zs), kGemvThreads, \
                                S, 0, stream, pk, xh, out, M, N, K, gs)                                          \
               : launch_cluster(rg::q4gsw_gemv_fwd_reg_kernel<NT_, SPG_, false>, dim3(tiles, S, zs), kGemvThreads,\
                                S, 0, stream, pk, xh, out, M, N, K, gs);                                         \
  } while (0)
  if (NT == 1) {
    if (spg == 1) Q4_FWD(1, 1); else if (spg == 2) Q4_FWD(1, 2); else Q4_FWD(1, 4);
  } else {
    if (spg == 1) Q4_FWD(2, 1); else if (spg == 2) Q4_FWD(2, 2); else Q4_FWD(2, 4);
  }
#undef Q4_FWD
  if (route) snprintf(route, route_len, "gemv_fwd launches=1 nt=%d splits=%d zslices=%d", NT, S, zs);
  return err;
}

cudaError_t launch_gemv_bwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* d_out, int M,
                            float* d_x, cudaStream_t stream, char* route, int route_len) {
  // the TMA-ring input gradient is the default; the register-fed one runs only when pinned
  if (route_pins().gemv != kGemvReg)
    return launch_gemv_tma_bwd(packed, N, K, gs, f32s, d_out, M, d_x, stream, route, route_len);
  const int tiles = (K + 127) / 128;
  const int zs = (M + 15) / 16;
  const int NT = (M <= 8) ? 1 : 2;
  const int spb = gs >= 64 ? 1 : gs == 32 ? 2 : 4;
  int S = 1;
  const size_t smem = sizeof(float) * kBwdWarps * 8 * NT * 128;
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  const __half* dh = reinterpret_cast<const __half*>(d_out);
  cudaError_t err;
#define Q4_BWD_F(NT_, SPB_, F_)                                                                                   \
  do {                                                                                                            \
    err = cudaFuncSetAttribute(rg::q4gsw_gemv_bwd_reg_kernel<NT_, SPB_, F_>,                                      \
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                           \
    if (err == cudaSuccess) {                                                                                     \
      S = bwd_splits((long long)tiles * zs, (N + 15) / 16, kBwdWarps);                                           \
      err = launch_cluster(rg::q4gsw_gemv_bwd_reg_kernel<NT_, SPB_, F_>, dim3(tiles, S, zs), kBwdThreads, S, smem, \
                           stream, pk, dh, d_x, M, N, K, gs);                                                     \
    }                                                                                                             \
  } while (0)
#define Q4_BWD(NT_, SPB_)                     \
  do {                                        \
    if (f32s) Q4_BWD_F(NT_, SPB_, true);      \
    else Q4_BWD_F(NT_, SPB_, false);          \
  } while (0)
  if (NT == 1) {
    if (spb == 1) Q4_BWD(1, 1); else if (spb == 2) Q4_BWD(1, 2); else Q4_BWD(1, 4);
  } else {
    if (spb == 1) Q4_BWD(2, 1); else if (spb == 2) Q4_BWD(2, 2); else Q4_BWD(2, 4);
  }
#undef Q4_BWD
#undef Q4_BWD_F
  if (route) snprintf(route, route_len, "gemv_bwd launches=1 nt=%d splits=%d zslices=%d", NT, S, zs);
  return err;
}

}  // namespace q4gsw
