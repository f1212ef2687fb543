// q4gsw_dq8ca_tma.cuh - the product of linear_dq8ca_q4gsw (int8 dynamically
// quantised activations times the q4gsw weight; shader list of "Upstream the
// Gemma 4 Vulkan support we carry on our ExecuTorch fork", issue #1361) for up
// to 16 tokens per z-slice, streaming the packed weight through the same TMA
// ring as the fp16 forward GEMV.
// Included once, by q4gsw_gemm_sm100.cu, after q4gsw_gemv_tma.cuh (ring
// constants, control block, row permutation, shared-memory loads).
//
//   y[m, n] = a_s[m] sum_g s[g, n] sum_{k in g} (q[m, k] - a_z[m]) (code[n, k] - 8)
//
// The weights enter mma.sync m16n8k32 (signed bytes) as 16 (code - 8): the
// code nibble moved to the high half of a byte with its top bit flipped, one
// LOP3 per register (plus a shift for the low nibbles).  The activations enter
// as q.  Per group and row tile the warp accumulates, exactly in int32,
//   P = sum 16 (c - 8) q    (one MMA per 8-token tile)
//   C = sum 16 (c - 8)      (one MMA against a ones operand, shared by the tiles)
// and folds (P - a_z C) / 16 = sum (c - 8)(q - a_z) into the fp32 sum with the
// fp16 scale.  a_s multiplies the final sum.
#pragma once

namespace q4gsw {
namespace dqt {

using gv::CODE_BYTES;
using gv::CTL_BYTES;
using gv::Ctl;
using gv::RP;
using gv::SK;
using gv::lds128;
using gv::lds32;
using gv::pair_of;

// NT 8-token MMA tiles: 4 consumer warps (all four row tiles each) for up to 8
// tokens, 8 (two row tiles each) for 9..16, as the fp16 ring.  Stage: codes
// 8 KB | q of the stage's 256 columns for 8 NT token rows, two [8 NT][128 B]
// boxes (128-byte swizzle; rows past the batch are zero-filled) | fp16 scale
// rows (256 / gs of them, at most 8 as gs >= 32), 1 KB aligned.  Unlike the
// fp16 ring, the activations travel in the stage: the int8 consumer spends so
// few instructions per stage that a global load issued one stage ahead would
// not arrive in time.
template <int NT>
struct Cfg {
  static constexpr int CW = NT == 2 ? 8 : 4;
  static constexpr int RTW = 4 / (CW / 4);
  static constexpr int THREADS = 32 * (CW + 1);
  static constexpr int MINB = NT == 1 ? 4 : 2;
  static constexpr int OFF_Q = CODE_BYTES;
  static constexpr int QBOX = 8 * NT * 128;
  static constexpr int OFF_SC = OFF_Q + 2 * QBOX;
  static constexpr int STAGE = (OFF_SC + 8 * 64 * 2 + 1023) / 1024 * 1024;
  // ring bytes: four CTAs per SM at NT = 1 (228 KB less 1 KB each), two at NT = 2
  static constexpr int ST = (NT == 1 ? 54 : 100) * 1024 / STAGE;
  static constexpr int OFF_CTL = ST * STAGE;
  static constexpr int BYTES = OFF_CTL + CTL_BYTES + 1024;
  static_assert(4 * 16 * 64 * 4 <= OFF_CTL, "warp partials fit in the ring");
  static_assert(ST >= 3 && ST <= 12, "ring depth");
  static_assert(MINB * (BYTES + 1024) <= 228 * 1024, "resident CTAs");
};

// D(16x8, s32) += A(16x32, s8, row) * B(32x8, s8, col)
__device__ __forceinline__ void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A * B (the first MMA of a group: no accumulator to clear)
__device__ __forceinline__ void mma_s8_zero(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

// 16 (c - 8) as signed bytes from the nibble pairs of one code word: the low
// nibbles (even row) and the high nibbles (odd row); c << 4 ^ 0x80 = 16 (c - 8).
__device__ __forceinline__ uint32_t even16(uint32_t w) { return ((w << 4) & 0xF0F0F0F0u) ^ 0x80808080u; }
__device__ __forceinline__ uint32_t odd16(uint32_t w) { return (w & 0xF0F0F0F0u) ^ 0x80808080u; }

// ONES (at most 7 tokens, NT = 1): B column 7 is a spare token column (its q
// row is zero-filled), so lanes g = 7 put ones there and column 7 of the
// product MMA gives C = sum 16 (c - 8) of each row: no separate ones-MMA.
// grid = (ceil(N / 64) row blocks, S contraction splits (one cluster), ceil(M / 16)).
// q: int8 [M][K] in the codes' order (inside each 64-column block, the 16 bytes
// at 16 t hold columns 4 t + 16 i + (0, 2, 1, 3), i = 0..3); a_s fp32 [M]; a_z int32 [M].
// GM: where groups start, fixed at compile time where gs allows it:
//   0 (gs 32): every 32-column step is a group;  1 (gs 64, 128): every block of
//   the warp (its two steps) lies in one group;  2 (gs >= 256): a group spans
//   blocks of several stages (tracked at run time).
template <int NT, bool ONES, int GM>
__global__ void __launch_bounds__(Cfg<NT>::THREADS, Cfg<NT>::MINB)
q4gsw_dq8ca_gemv_tma_kernel(const __grid_constant__ CUtensorMap map_pk, const __grid_constant__ CUtensorMap map_sc,
                            const __grid_constant__ CUtensorMap map_q, const float* __restrict__ a_s,
                            const int* __restrict__ a_z, OutSplit out, int M, int N, int K, int gs,
                            int stages_total) {
  using namespace sm100;
  using C = Cfg<NT>;
  constexpr int RTW = C::RTW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + C::OFF_CTL);
  volatile int* abort_flag = &ctl->abort;
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, split = blockIdx.y, S = gridDim.y;
  const int tok0 = blockIdx.z * 16;
  const int Mz = min(16, M - tok0);
  const int n0 = tile * 64;
  const int st_begin = (int)((long long)split * stages_total / S);
  const int st_end = (int)((long long)(split + 1) * stages_total / S);
  const int nit = st_end - st_begin;
  const int gsl = __ffs(gs) - 1;

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::ST; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->empty[i], C::CW);
    }
    ctl->abort = 0;
    fence_mbar_init();
    prefetch_tmap(&map_pk);
    prefetch_tmap(&map_sc);
    prefetch_tmap(&map_q);
  }
  __syncthreads();

  const int sc_rows = gs < SK ? SK / gs : 1;
  const uint32_t tx = CODE_BYTES + 2 * C::QBOX + sc_rows * 64 * 2;
  const int g = lane >> 2, t = lane & 3;
  float acc[RTW][NT][4];
#pragma unroll
  for (int rt = 0; rt < RTW; ++rt)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[rt][j][c] = 0.f;

  if (warp == C::CW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      auto load_weights = [&](int it) {
        const int s = it % C::ST;
        const int kc = (st_begin + it) * SK;
        uint8_t* st = smem + s * C::STAGE;
        tma_load_2d(st, &map_pk, &ctl->full[s], kc, n0 / 2);
        tma_load_2d(st + CODE_BYTES / 2, &map_pk, &ctl->full[s], kc + 128, n0 / 2);
        tma_load_2d(st + C::OFF_SC, &map_sc, &ctl->full[s], n0, kc >> gsl);
      };
      auto load_q = [&](int it) {
        const int s = it % C::ST;
        const int kc = (st_begin + it) * SK;
        uint8_t* st = smem + s * C::STAGE + C::OFF_Q;
        tma_load_2d(st, &map_q, &ctl->full[s], kc, tok0);
        tma_load_2d(st + C::QBOX, &map_q, &ctl->full[s], kc + 128, tok0);
      };
      // the packed weight is constant: the ring's weights load while the
      // quantiser still runs, its q once the quantiser is done
      const int pre = nit < C::ST ? nit : C::ST;
      for (int it = 0; it < pre; ++it) {
        mbar_arrive_expect_tx(&ctl->full[it], tx);
        load_weights(it);
      }
      griddep_wait();
      for (int it = 0; it < pre; ++it) load_q(it);
      int issued = pre;
      for (int it = pre; it < nit; ++it) {
        const int s = it % C::ST;
        if (!mbar_wait(&ctl->empty[s], ((it / C::ST) - 1) & 1, abort_flag, &g_device_error, 0x400u)) break;
        mbar_arrive_expect_tx(&ctl->full[s], tx);
        load_weights(it);
        load_q(it);
        issued = it + 1;
      }
      for (int it = (issued > C::ST ? issued - C::ST : 0); it < issued; ++it)
        mbar_wait_teardown(&ctl->full[it % C::ST], (it / C::ST) & 1);
    }
  } else {
    // ------------------------------------------------------------ consumers
    griddep_wait();   // a_s and a_z come from the quantiser just before
    const int w = warp & 3;             // 64-column block of every stage
    const int rt0 = (warp >> 2) * RTW;  // first row tile of this warp
    uint32_t code_off[RTW];
#pragma unroll
    for (int rt = 0; rt < RTW; ++rt) {
      const int r = pair_of(rt0 + rt, g);
      code_off[rt] = (w >> 1) * (CODE_BYTES / 2) + r * 128 + 16 * ((4 * (w & 1) + t) ^ (r & 7));
    }
    // B column g of token tile j: q row 8 j + g of the stage (zero past the
    // batch, never stored), the 16 bytes of lane t in the warp's block
    uint32_t q_off[NT];
    int az0[NT], az1[NT];   // zero points of the D columns 2t, 2t + 1
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int r = 8 * j + g;
      q_off[j] = C::OFF_Q + (w >> 1) * C::QBOX + r * 128 + 16 * ((4 * (w & 1) + t) ^ (r & 7));
      az0[j] = a_z[tok0 + min(8 * j + 2 * t, Mz - 1)];
      az1[j] = a_z[tok0 + min(8 * j + 2 * t + 1, Mz - 1)];
    }
    // scale half2 of row tile rt: stage row (64 w + 32 h) >> gsl, pair perm(g)
    uint32_t sc_off[2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
      sc_off[h] = C::OFF_SC + (uint32_t)(gs < SK ? ((64 * w + 32 * h) >> gsl) : 0) * 64 * 2 + 4 * pair_of(rt0, g);

    static_assert(!ONES || NT == 1, "the spare column exists for up to 7 tokens");
    int pq[RTW][NT][4], pc[RTW][4];
    bool gstart = true;   // no MMA since the last flush: the next one starts a group
    auto flush = [&](const uint32_t (&sw)[RTW]) {
#pragma unroll
      for (int rt = 0; rt < RTW; ++rt) {
        if (ONES) {   // C of row g (even) and g + 8 (odd) from lane (g, 3), D column 7
          pc[rt][0] = pc[rt][1] = __shfl_sync(0xffffffffu, pq[rt][0][1], (g << 2) | 3);
          pc[rt][2] = pc[rt][3] = __shfl_sync(0xffffffffu, pq[rt][0][3], (g << 2) | 3);
        }
        const float2 sp = __half22float2(*reinterpret_cast<const __half2*>(&sw[rt]));
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          // D: [0] row g (even), column 2t; [1] even, 2t + 1; [2] row g + 8 (odd), 2t; [3] odd, 2t + 1
          acc[rt][j][0] = fmaf((float)((pq[rt][j][0] - az0[j] * pc[rt][0]) >> 4), sp.x, acc[rt][j][0]);
          acc[rt][j][1] = fmaf((float)((pq[rt][j][1] - az1[j] * pc[rt][1]) >> 4), sp.x, acc[rt][j][1]);
          acc[rt][j][2] = fmaf((float)((pq[rt][j][2] - az0[j] * pc[rt][2]) >> 4), sp.y, acc[rt][j][2]);
          acc[rt][j][3] = fmaf((float)((pq[rt][j][3] - az1[j] * pc[rt][3]) >> 4), sp.y, acc[rt][j][3]);
        }
      }
      gstart = true;
    };
    constexpr uint32_t kOnes = 0x01010101u;
    auto stage = [&](int it) -> bool {
      const int s = it % C::ST;
      if (!mbar_wait(&ctl->full[s], (it / C::ST) & 1, abort_flag, &g_device_error, 0x800u)) return false;
      const uint32_t st = sbase + s * C::STAGE;
      uint4 qv[NT];
#pragma unroll
      for (int j = 0; j < NT; ++j) qv[j] = lds128(st + q_off[j]);
      if (ONES && g == 7) qv[0] = make_uint4(kOnes, kOnes, kOnes, kOnes);
      uint4 wv[RTW];
      uint32_t sw[2][RTW];
#pragma unroll
      for (int rt = 0; rt < RTW; ++rt) {
        wv[rt] = lds128(st + code_off[rt]);
#pragma unroll
        for (int h = 0; h < 2; ++h) sw[h][rt] = lds32(st + sc_off[h] + 32 * rt);
      }
      {
        uint32_t dep = 0u;
#pragma unroll
        for (int j = 0; j < NT; ++j) dep ^= qv[j].x ^ qv[j].y ^ qv[j].z ^ qv[j].w;
#pragma unroll
        for (int rt = 0; rt < RTW; ++rt) dep ^= wv[rt].x ^ wv[rt].y ^ wv[rt].z ^ wv[rt].w ^ sw[0][rt] ^ sw[1][rt];
        stage_reads_done(dep);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->empty[s]);   // the stage is in registers
      const int k0 = (st_begin + it) * SK + 64 * w;
      // a block past K (zero-filled codes, which would count as 16 (0 - 8))
      // takes no MMA; K % 64 == 0, so a block is wholly inside or outside
      const bool in = k0 < K;
#pragma unroll
      for (int h = 0; h < 2; ++h) {   // 32-column steps: code words 2h, 2h + 1; q words likewise
        if (in) {
#pragma unroll
          for (int rt = 0; rt < RTW; ++rt) {
            const uint32_t w0 = h == 0 ? wv[rt].x : wv[rt].z, w1 = h == 0 ? wv[rt].y : wv[rt].w;
            const uint32_t a[4] = {even16(w0), odd16(w0), even16(w1), odd16(w1)};
            // the first MMA of a group takes a zero accumulator
            const bool zero = GM == 0 ? true : GM == 1 ? h == 0 : gstart;
            if (!ONES) {
              if (zero) mma_s8_zero(pc[rt], a, kOnes, kOnes);
              else mma_s8(pc[rt], a, kOnes, kOnes);
            }
#pragma unroll
            for (int j = 0; j < NT; ++j) {
              const uint32_t b0 = h == 0 ? qv[j].x : qv[j].z, b1 = h == 0 ? qv[j].y : qv[j].w;
              if (zero) mma_s8_zero(pq[rt][j], a, b0, b1);
              else mma_s8(pq[rt][j], a, b0, b1);
            }
          }
          gstart = false;
        }
        // a group ends with this step: at every step (GM 0), at the block end
        // (GM 1), else when the warp's next block (256 columns on) starts
        // another group or the split ends; blocks past K took no MMA and add
        // nothing (they come last, after the warp's final flush, for GM 0 and 1)
        if (GM == 0) {
          if (in) flush(sw[h]);
        } else if (GM == 1) {
          if (in && h == 1) flush(sw[0]);
        } else if (h == 1 && !gstart && (((k0 + SK) >> gsl) != (k0 >> gsl) || it == nit - 1)) {
          flush(sw[0]);
        }
      }
      return true;
    };
    for (int it = 0; it < nit; ++it)
      if (!stage(it)) break;
  }

  // warp partials -> [block][token][row]; the four block slices summed in order
  __syncthreads();
  griddep_wait();   // every thread reads a_s below (returns at once where it has waited)
  float* red = reinterpret_cast<float*>(smem);
  if (warp < C::CW) {
    float* rs = red + (warp & 3) * 16 * 64;
    const int rt0 = (warp >> 2) * RTW;
#pragma unroll
    for (int rt = 0; rt < RTW; ++rt) {
      const int r = pair_of(rt0 + rt, g);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        rs[(8 * j + 2 * t) * 64 + 2 * r] = acc[rt][j][0];
        rs[(8 * j + 2 * t + 1) * 64 + 2 * r] = acc[rt][j][1];
        rs[(8 * j + 2 * t) * 64 + 2 * r + 1] = acc[rt][j][2];
        rs[(8 * j + 2 * t + 1) * 64 + 2 * r + 1] = acc[rt][j][3];
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < Mz * 64; e += C::THREADS)
    red[e] = ((red[e] + red[16 * 64 + e]) + red[2 * 16 * 64 + e]) + red[3 * 16 * 64 + e];

  // rank rk of the cluster sums tokens [rk Mz / S, (rk + 1) Mz / S) of the S
  // partial tiles in rank order, scales them by a_s and stores them
  cg::cluster_group cluster = cg::this_cluster();
  if (S > 1) cluster.sync();
  else __syncthreads();
  if (!(S > 1 ? cluster_any_abort(cluster, &ctl->abort, S) : *abort_flag)) {
    const int rk = S > 1 ? (int)cluster.block_rank() : 0;
    const int tb = rk * Mz / S, te = (rk + 1) * Mz / S;
    for (int e = threadIdx.x; e < (te - tb) * 64; e += C::THREADS) {
      const int tok = tb + (e >> 6), nl = e & 63;
      const int n = n0 + nl;
      if (n >= N) continue;
      float v = 0.f;
      for (int q = 0; q < S; ++q) v += (q == rk ? red : cluster.map_shared_rank(red, q))[tok * 64 + nl];
      const size_t m = (size_t)(tok0 + tok);
      v *= a_s[m];
      if (n < out.n1) out.y0[m * out.n1 + n] = v;
      else if (n < out.n2) out.y1[m * (out.n2 - out.n1) + (n - out.n1)] = v;
      else out.y2[m * (out.N - out.n2) + (n - out.n2)] = v;
    }
  }
  if (S > 1) cluster.sync();
}

}  // namespace dqt

template <int NT, bool ONES, int GM>
static cudaError_t launch_dq8ca_variant(const CUtensorMap& map_pk, const CUtensorMap& map_sc, const CUtensorMap& map_q,
                                        const float* a_s, const int* a_z, OutSplit out, int M, int N, int K, int gs,
                                        int stages_total, dim3 grid, cudaStream_t stream) {
  using C = dqt::Cfg<NT>;
  auto kern = dqt::q4gsw_dq8ca_gemv_tma_kernel<NT, ONES, GM>;
  static PerDeviceOnce attr_once;
  {
    cudaError_t e = once_per_device(attr_once, current_device(), [&] {
      return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES);
    });
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = grid.y;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, map_pk, map_sc, map_q, a_s, a_z, out, M, N, K, gs, stages_total);
}

cudaError_t launch_dq8ca_gemv(const void* packed, int N, int K, int gs, int M, const void* workspace, OutSplit out,
                              cudaStream_t stream, char* route, int route_len) {
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  const Layout L = layout_of(N, K, gs);
  const int G = K / gs;
  const int NT = (M <= 8) ? 1 : 2;
  const int zs = (M + 15) / 16;
  const int tiles = (N + 63) / 64;
  const int stages_total = (K + gv::SK - 1) / gv::SK;
  // contraction splits as the fp16 ring: fill the resident CTA slots, at least
  // two stages per split, clusters of at most 8
  const int per_sm = NT == 1 ? 4 : 2;
  int S = sm_count(current_device()) * per_sm / (tiles * zs);
  S = S < 1 ? 1 : (S > 8 ? 8 : S);
  while (S > 1 && stages_total / S < 2) --S;
  const int sc_rows = gs < gv::SK ? gv::SK / gs : 1;
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  CUtensorMap map_pk, map_sc, map_q;
  const bool ok =
      make_map_2d(&map_pk, CU_TENSOR_MAP_DATA_TYPE_UINT8, pk, K, N / 2, K, 128, gv::RP, CU_TENSOR_MAP_SWIZZLE_128B) &&
      make_map_2d(&map_sc, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, pk + L.scales_offset, N, G, (uint64_t)N * 2, 64, sc_rows,
                  CU_TENSOR_MAP_SWIZZLE_NONE) &&
      make_map_2d(&map_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws, K, M, K, 128, 8 * NT, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  const float* a_s = reinterpret_cast<const float*>(ws + dq8ca_scale_offset(M, K));
  const int* a_z = reinterpret_cast<const int*>(ws + dq8ca_zero_offset(M, K));
  const dim3 grid(tiles, S, zs);
  const int gm = gs == 32 ? 0 : gs < gv::SK ? 1 : 2;
#define Q4_DQ(NT_, ONES_)                                                                                          \
  (gm == 0   ? launch_dq8ca_variant<NT_, ONES_, 0>(map_pk, map_sc, map_q, a_s, a_z, out, M, N, K, gs, stages_total, \
                                                   grid, stream)                                                   \
   : gm == 1 ? launch_dq8ca_variant<NT_, ONES_, 1>(map_pk, map_sc, map_q, a_s, a_z, out, M, N, K, gs, stages_total, \
                                                   grid, stream)                                                   \
             : launch_dq8ca_variant<NT_, ONES_, 2>(map_pk, map_sc, map_q, a_s, a_z, out, M, N, K, gs, stages_total, \
                                                   grid, stream))
  const cudaError_t e = NT == 2 ? Q4_DQ(2, false) : M <= 7 ? Q4_DQ(1, true) : Q4_DQ(1, false);
#undef Q4_DQ
  if (route)
    snprintf(route, route_len, "int8_gemv_tma nt=%d tiles=%d splits=%d zslices=%d stages=%d%s", NT, tiles, S, zs,
             NT == 1 ? dqt::Cfg<1>::ST : dqt::Cfg<2>::ST, NT == 1 && M <= 7 ? " ones_column=7" : "");
  return e;
}

}  // namespace q4gsw
