// q4gsw_gemv_tma.cuh - GEMV routes for small token counts (M <= 16 per
// z-slice) that stream the packed weight through a TMA ring (sm_100a):
// forward and input gradient.
// Included once, by q4gsw_gemm_sm100.cu, which owns the device error word and
// the tensor-map helpers.
//
//   y[m, n] = sum_k x[m, k] (code[n, k] - 8) s[k / gs, n]
// ("[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward kernel (4-bit
// input-grad)", PR description; this is the forward it mirrors.)
//
// At M <= 16 the layer is a weight stream: every code byte is read once and
// used for at most 16 tokens, so the kernel lives or dies by the bytes it keeps
// in flight and by the instructions it spends per weight.  Forward: one
// producer thread per CTA keeps ST stages of 256 contraction columns in flight
// with TMA (codes of 32 nibble pairs = 64 output rows, their scale rows, the
// activation columns); each of four consumer warps takes one 64-column block
// of every stage for all four 16-row MMA tiles, so one activation fragment
// feeds four mma.sync m16n8k16 (A = 16 weight rows, B = 8 tokens).  The codes
// enter the MMA as exact integers code - 8; the fp16 scale multiplies the fp32
// partial sum of each group, whose first MMA starts from a zero accumulator.
// The four block slices are summed in shared memory, split-K CTAs of a cluster
// through distributed shared memory, both in a fixed order.
#pragma once

namespace q4gsw {
namespace gv {

constexpr int RP = 32;                                  // nibble pairs per CTA (64 rows = 4 MMA row tiles)
constexpr int SK = 256;                                 // contraction columns per stage
constexpr int CODE_BYTES = RP * SK;                     // two [32 pairs][128 B] boxes, 8 KB
constexpr int CTL_BYTES = 256;

// Forward configuration for NT 8-token MMA tiles, SPG 16-column steps per
// scale group, fp32 or fp16 scales.
//   consumer warps: 4 (one 64-column block of every stage each, all four row
//   tiles, so one activation fragment feeds four MMAs) for up to 8 tokens;
//   8 (two per block, two row tiles each) for 9..16, whose twice as many MMAs
//   per weight need the extra warps (measured on B200, 14336x4096: M=1
//   12.3 us with 4 warps vs 16.1 us with 8; M=16 17.0 us with 8 vs 20.5 us
//   with 4).
//   stage: [codes 8 KB | scale rows], 1 KB aligned.  The scale rows of a stage
//   are 256 / gs rows (at least one) of 64 scales.  The activations are not
//   staged: every CTA of the launch reads the same few kilobytes, which stay in
//   L1 and L2, and each of them would cost the TMA unit a tiny box per stage.
//   ST: the ring depth that keeps a CTA near 56 KB, so that two CTAs of this
//   launch and two of the next fit on one SM.
//   XS: the activations travel in the stage too, four [8 NT tokens][64 fp16]
//   boxes (128-byte swizzle, rows past the batch zero-filled) after the codes,
//   so they arrive ST stages ahead like the weights; the ring then holds four
//   stages (NT = 1, four CTAs per SM) or five (NT = 2, two CTAs per SM).
template <int NT, int SPG, bool F32S, bool XS = false>
struct FwdCfg {
  static constexpr int CW = NT == 2 ? 8 : 4;                 // consumer warps
  static constexpr int RTW = 4 / (CW / 4);                   // row tiles per consumer warp
  static constexpr int THREADS = 32 * (CW + 1);              // the last warp produces
  // resident CTAs per SM the registers are sized for
  static constexpr int MINB = NT == 1 ? 4 : 2;
  static constexpr int SB = F32S ? 4 : 2;                    // bytes per scale
  static constexpr int SCB = (SPG == 1 ? 16 : SPG == 2 ? 8 : 4) * 64 * SB;
  static constexpr int XBOX = 8 * NT * 128;                  // one activation box
  static constexpr int OFF_X = CODE_BYTES;
  static constexpr int OFF_SC = XS ? OFF_X + 4 * XBOX : CODE_BYTES;
  static constexpr int STAGE = (OFF_SC + SCB + 1023) / 1024 * 1024;
  static constexpr int ST0 = (XS ? (NT == 1 ? 54 : 100) : 56) * 1024 / STAGE;
  static constexpr int ST = ST0 < 3 ? 3 : ST0 > 8 ? 8 : ST0;
  static constexpr int OFF_CTL = ST * STAGE;
  static constexpr int BYTES = OFF_CTL + CTL_BYTES + 1024;
  static constexpr int RED_FLOATS = 4 * 16 * 64;             // [block][token][row], reuses the ring
  static_assert(RED_FLOATS * 4 <= OFF_CTL, "warp partials fit in the ring");
  static_assert(ST <= 12, "barrier arrays");
  static_assert(!XS || MINB * (BYTES + 1024) <= 228 * 1024, "resident CTAs");
};

struct Ctl {
  uint64_t full[12];
  uint64_t empty[12];
  int abort;
};
static_assert(sizeof(Ctl) <= CTL_BYTES, "control block");

// MMA row g of row tile rt reads pair row 8 rt + perm(g): the two pairs a
// quarter of the warp reads together then differ in bit 2, so under the
// 128-byte swizzle their 16-byte code chunks fall on distinct banks.
__device__ __forceinline__ int pair_of(int rt, int g) { return 8 * rt + ((g & 1) << 2) + (g >> 1); }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// grid = (ceil(N / 64) row tiles, S contraction splits, ceil(M / 16) token
// slices), cluster = (1, S, 1).  SPG = 16-column steps per scale group
// (1: gs 16, 2: gs 32, 4: gs 64 or 128, where a warp's 64-column block is one
// group; 8: gs >= 256, where a group spans the warp's blocks of several stages).
template <int NT, int SPG, bool F32S, bool XS>
__global__ void __launch_bounds__(FwdCfg<NT, SPG, F32S, XS>::THREADS, FwdCfg<NT, SPG, F32S, XS>::MINB)
q4gsw_gemv_fwd_tma_kernel(const __grid_constant__ CUtensorMap map_pk, const __grid_constant__ CUtensorMap map_sc,
                          const __grid_constant__ CUtensorMap map_x, const __half* __restrict__ x, OutSplit out,
                          int M, int N, int K, int gs, int stages_total) {
  using namespace sm100;
  using C = FwdCfg<NT, SPG, F32S, XS>;
  constexpr int RTW = C::RTW;
  constexpr int NGB = SPG >= 4 ? 1 : 4 / SPG;   // scale groups per 64-column block
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
    if (XS) prefetch_tmap(&map_x);
  }
  __syncthreads();

  // scale rows per stage: 256 / gs for gs <= 256, else 1
  const int sc_rows = gs < SK ? SK / gs : 1;
  const uint32_t tx = CODE_BYTES + sc_rows * 64 * C::SB + (XS ? 4 * C::XBOX : 0);

  float acc[RTW][NT][4];
#pragma unroll
  for (int rt = 0; rt < RTW; ++rt)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[rt][j][c] = 0.f;
  const int g = lane >> 2, t = lane & 3;

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
      auto load_x = [&](int it) {   // XS: the stage's activation boxes
        const int s = it % C::ST;
        const int kc = (st_begin + it) * SK;
        uint8_t* st = smem + s * C::STAGE + C::OFF_X;
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(st + b * C::XBOX, &map_x, &ctl->full[s], kc + 64 * b, tok0);
      };
      // the packed weight is constant: the ring is filled before (and while)
      // the consumers wait for the kernel that produces x
      const int pre = nit < C::ST ? nit : C::ST;
      for (int it = 0; it < pre; ++it) {
        mbar_arrive_expect_tx(&ctl->full[it], tx);
        load_weights(it);
      }
      if (XS) {
        griddep_wait();
        for (int it = 0; it < pre; ++it) load_x(it);
      }
      int issued = pre;
      for (int it = pre; it < nit; ++it) {
        const int s = it % C::ST;
        if (!mbar_wait(&ctl->empty[s], ((it / C::ST) - 1) & 1, abort_flag, &g_device_error, 64u)) break;
        mbar_arrive_expect_tx(&ctl->full[s], tx);
        load_weights(it);
        if (XS) load_x(it);
        issued = it + 1;
      }
      for (int it = (issued > C::ST ? issued - C::ST : 0); it < issued; ++it)
        mbar_wait_teardown(&ctl->full[it % C::ST], (it / C::ST) & 1);
    }
  } else {
    // ------------------------------------------------------------ consumers
    griddep_wait();   // outputs of this kernel may still be read by the previous one
    const int w = warp & 3;             // 64-column block of every stage
    const int rt0 = (warp >> 2) * RTW;  // first row tile of this warp
    // per-thread shared-memory offsets inside a stage: 16-byte code chunk t of
    // block w (128-byte swizzle inside the [32 pairs][128 B] box w / 2) for the
    // pair row of each row tile
    uint32_t code_off[RTW];
#pragma unroll
    for (int rt = 0; rt < RTW; ++rt) {
      const int r = pair_of(rt0 + rt, g);
      code_off[rt] = (w >> 1) * (CODE_BYTES / 2) + r * 128 + 16 * ((4 * (w & 1) + t) ^ (r & 7));
    }
    // activation fragment of token tile j: token row min(8 j + g, Mz - 1),
    // columns 16 i + 4 t .. + 3 of the warp's block (lanes past the last token
    // repeat it, so for one token every lane of a quad position reads the same
    // 8 bytes); read from global memory one stage ahead of its use
    const __half* xrow[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) xrow[j] = x + (size_t)(tok0 + min(8 * j + g, Mz - 1)) * K + 64 * w + 4 * t;
    // XS: the same fragment from the stage's box w, row 8 j + g, 16-byte
    // chunk 2 i + t / 2 under the 128-byte swizzle, half t % 2 of it
    uint32_t x_row[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) x_row[j] = C::OFF_X + w * C::XBOX + (8 * j + g) * 128 + 8 * (t & 1);
    auto load_xf = [&](int it, uint2 (&d)[NT][4]) {
      if (XS) return;
      const int kb = (st_begin + it) * SK;   // the warp's block starts at kb + 64 w
      const bool in = kb + 64 * w < K;       // K % 64 == 0: a block is wholly inside or outside
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) d[j][i] = in ? ldg_nc_v2(xrow[j] + kb + 16 * i) : make_uint2(0u, 0u);
    };
    // scale words of block w: row (64 w + 16 SPG q) >> gsl of the stage's box
    // (stages start on multiples of 256 columns), the (even, odd) pair of pair
    // perm(g) of the warp's first row tile (+ 16 scales per row tile)
    uint32_t sc_off[NGB];
#pragma unroll
    for (int q = 0; q < NGB; ++q) {
      const int col = 64 * w + (SPG >= 4 ? 0 : 16 * SPG * q);
      sc_off[q] = C::OFF_SC + (uint32_t)(gs < SK ? (col >> gsl) : 0) * 64 * C::SB + 2 * C::SB * pair_of(rt0, g);
    }

    float part[RTW][NT][4];
    bool fresh = true;   // the next MMA starts a new group (zero accumulator)
    // Release of a stage: with 16 tokens (NT = 2) after its MMAs, whose
    // operands are then known to be in registers (M=16, 14336x4096 forward:
    // 14.5 -> 13.9 us); with 8 tokens as soon as its words are loaded, which
    // measured as fast or faster there (the refill starts earlier).
    constexpr bool kLateRelease = NT == 2;
    // one stage: wait for its codes and scales, then dequantise and multiply;
    // false when a wait ran out
    auto stage = [&](int it, const uint2 (&xg)[NT][4]) -> bool {
      const int s = it % C::ST;
      if (!mbar_wait(&ctl->full[s], (it / C::ST) & 1, abort_flag, &g_device_error, 128u)) return false;
      const uint32_t st = sbase + s * C::STAGE;
      uint2 xv[NT][4];
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          xv[j][i] = XS ? lds64(st + x_row[j] + 16 * ((2 * i + (t >> 1)) ^ g)) : xg[j][i];
      uint4 wv[RTW];
#pragma unroll
      for (int rt = 0; rt < RTW; ++rt) wv[rt] = lds128(st + code_off[rt]);
      uint2 sw[RTW][NGB];
#pragma unroll
      for (int rt = 0; rt < RTW; ++rt)
#pragma unroll
        for (int q = 0; q < NGB; ++q) {
          const uint32_t a = st + sc_off[q] + 16 * C::SB * rt;
          sw[rt][q] = F32S ? lds64(a) : make_uint2(lds32(a), 0u);
        }
      {
        uint32_t dep = 0u;
#pragma unroll
        for (int rt = 0; rt < RTW; ++rt) {
          dep ^= wv[rt].x ^ wv[rt].y ^ wv[rt].z ^ wv[rt].w;
#pragma unroll
          for (int q = 0; q < NGB; ++q) dep ^= sw[rt][q].x ^ sw[rt][q].y;
        }
        if (XS)
#pragma unroll
          for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) dep ^= xv[j][i].x ^ xv[j][i].y;
        if (!kLateRelease) stage_reads_done(dep);
      }
      if (!kLateRelease) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->empty[s]);   // the stage is in registers
      }

      auto flush = [&](int q) {   // scale the finished group of every row tile into acc
#pragma unroll
        for (int rt = 0; rt < RTW; ++rt) {
          const float2 sp = scale_pair<F32S>(sw[rt][q]);
          const float se = sp.x, so = sp.y;
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            acc[rt][j][0] = fmaf(part[rt][j][0], se, acc[rt][j][0]);
            acc[rt][j][1] = fmaf(part[rt][j][1], se, acc[rt][j][1]);
            acc[rt][j][2] = fmaf(part[rt][j][2], so, acc[rt][j][2]);
            acc[rt][j][3] = fmaf(part[rt][j][3], so, acc[rt][j][3]);
          }
        }
      };
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // the first MMA of a group starts from a zero accumulator; where the
        // groups start is fixed at compile time except for groups over stages
        const bool first = SPG == 8 ? (i == 0 && fresh) : SPG == 4 ? i == 0 : (i % SPG == 0);
#pragma unroll
        for (int rt = 0; rt < RTW; ++rt) {
          const uint32_t word = i == 0 ? wv[rt].x : i == 1 ? wv[rt].y : i == 2 ? wv[rt].z : wv[rt].w;
          const RowPairs rp = codes_minus8_rows(word);
          const uint32_t a[4] = {h2_as_u32(rp.ev01), h2_as_u32(rp.od01), h2_as_u32(rp.ev23), h2_as_u32(rp.od23)};
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            const uint32_t bf[2] = {xv[j][i].x, xv[j][i].y};
            if (first) mma_16816_zero(part[rt][j], a, bf);
            else mma_16816(part[rt][j], a, bf);
          }
        }
        if (SPG < 4 && (i % SPG) == SPG - 1) flush(i / SPG);
      }
      if (SPG == 4) flush(0);   // the block is one group (gs 64 or 128)
      if (SPG == 8) {
        // this warp's block of the next stage starts another group, or the split ends here
        const int k0 = (st_begin + it) * SK + 64 * w;
        fresh = ((k0 + SK) >> gsl) != (k0 >> gsl) || it == nit - 1;
        if (fresh) flush(0);
      }
      if (kLateRelease) {
        // the MMAs consumed the codes and activations; the scale words of a
        // group that continues into the next stage (gs >= 256) may be unused
        uint32_t dep = 0u;
#pragma unroll
        for (int rt = 0; rt < RTW; ++rt)
#pragma unroll
          for (int q = 0; q < NGB; ++q) dep ^= sw[rt][q].x ^ sw[rt][q].y;
        stage_reads_done(dep);
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->empty[s]);
      }
      return true;
    };
    // two register sets of activation fragments alternate: the next stage's
    // are in flight while the current stage is multiplied
    uint2 xa[NT][4], xb[NT][4];
    if (nit > 0) load_xf(0, xa);
    for (int it = 0; it < nit; it += 2) {
      if (it + 1 < nit) load_xf(it + 1, xb);
      if (!stage(it, xa) || it + 1 >= nit) break;
      if (it + 2 < nit) load_xf(it + 2, xa);
      if (!stage(it + 1, xb)) break;
    }
  }

  // warp partials -> [warp][token][row]; the four block slices summed in order
  __syncthreads();
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

  // Rank rk of the cluster sums tokens [rk Mz / S, (rk + 1) Mz / S) of the S
  // partial tiles in rank order and stores them (64 features per token).
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
      if (n < out.n1) out.y0[m * out.n1 + n] = v;
      else if (n < out.n2) out.y1[m * (out.n2 - out.n1) + (n - out.n1)] = v;
      else out.y2[m * (out.N - out.n2) + (n - out.n2)] = v;
    }
  }
  if (S > 1) cluster.sync();
}


// ---------------------------------------------------------------------------
// Input gradient: d_x[m, k] = sum_n d_out[m, n] (code[n, k] - 8) s[k / gs, n]
// ---------------------------------------------------------------------------
// MMA roles as in the register-fed kernel: A = weight^T tile (16 output
// columns k x 16 contraction rows n = 8 nibble pairs; a register holds the
// (even n, odd n) half2 of one byte, scaled per element), B = d_out^T (16 n x
// 8 tokens).  A CTA owns 128 output columns (two 64-byte blocks) and streams
// stages of 64 nibble pairs (128 contraction rows): codes [64 pairs][128 B]
// (128-byte swizzle), d_out [MB tokens][2 x 64 n] and the scale rows of the
// CTA's column groups for those 128 n.  Consumer warp c takes the 8 pairs
// 8c .. 8c + 7 of every stage; lane (g, t) reads 16 bytes at chunk g & 3 of
// block g >> 2 in pair rows 8c + t and 8c + t + 4, i.e. columns
// 64 (g >> 2) + 16 i + 4 (g & 3) + e; MMA q = 2 i + h maps A row g to e = 2h
// and row g + 8 to e = 2h + 1.
constexpr int kBwdConsumers = 8;
constexpr int kBwdThreads = 32 * (1 + kBwdConsumers);
constexpr int BWD_CODE_BYTES = 64 * 128;   // 64 pairs x 128 columns

template <int NT, bool F32S>
struct BwdCfg {
  static constexpr int SB = F32S ? 4 : 2;                          // bytes per scale
  static constexpr int SCB = 8 * 128 * SB;                         // up to 8 scale rows of 128 n
  static constexpr int MB = 8 * NT;
  static constexpr int DBOX = MB * 128 < 1024 ? 1024 : MB * 128;   // one [MB][64 n] box
  static constexpr int STAGE = BWD_CODE_BYTES + SCB + 2 * DBOX;
  static constexpr int ST = NT == 1 ? (F32S ? 7 : 8) : (F32S ? 6 : 7);
  static constexpr int OFF_CTL = ST * STAGE;
  static constexpr int BYTES = OFF_CTL + CTL_BYTES + 1024;
  static constexpr int RED_FLOATS = kBwdConsumers * MB * 128;   // warp partials, reuse the ring
  static_assert(STAGE % 1024 == 0, "stages stay 1024-byte aligned");
  static_assert(RED_FLOATS * 4 + MB * 128 * 4 <= OFF_CTL, "reduction fits in the ring");
  static_assert(BYTES <= 113 * 1024, "two CTAs per SM");
};

template <int NT, int SPB, bool F32S>  // SPB scale groups per 64-column block: 1 (gs >= 64), 2 (gs 32), 4 (gs 16)
__global__ void __launch_bounds__(kBwdThreads, 2)
q4gsw_gemv_bwd_tma_kernel(const __grid_constant__ CUtensorMap map_pk, const __grid_constant__ CUtensorMap map_sc,
                    const __grid_constant__ CUtensorMap map_d, float* __restrict__ dx, int M, int N, int K,
                    int gs, int stages_total) {
  using namespace sm100;
  using C = BwdCfg<NT, F32S>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + C::OFF_CTL);
  volatile int* abort_flag = &ctl->abort;
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.y, S = gridDim.y;
  const int tok0 = blockIdx.z * 16;
  const int Mz = min(16, M - tok0);
  const int kbase = 128 * blockIdx.x;
  const int st_begin = (int)((long long)split * stages_total / S);
  const int st_end = (int)((long long)(split + 1) * stages_total / S);
  const int nit = st_end - st_begin;
  const int gsl = __ffs(gs) - 1;
  const int sc_rows = gs < 128 ? 128 / gs : 1;

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::ST; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->empty[i], kBwdConsumers);
    }
    ctl->abort = 0;
    fence_mbar_init();
    prefetch_tmap(&map_pk);
    prefetch_tmap(&map_sc);
    prefetch_tmap(&map_d);
  }
  __syncthreads();
  const uint32_t tx = BWD_CODE_BYTES + sc_rows * 128 * C::SB + 2 * C::MB * 128;

  float acc[NT][8][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[j][q][c] = 0.f;
  const int g = lane >> 2, t = lane & 3;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      auto load_weights = [&](int it) {
        const int s = it % C::ST;
        const int n0 = (st_begin + it) * 128;
        uint8_t* st = smem + s * C::STAGE;
        tma_load_2d(st, &map_pk, &ctl->full[s], kbase, n0 / 2);
        tma_load_2d(st + BWD_CODE_BYTES, &map_sc, &ctl->full[s], n0, kbase >> gsl);
      };
      auto load_d = [&](int it) {
        const int s = it % C::ST;
        const int n0 = (st_begin + it) * 128;
        uint8_t* ds = smem + s * C::STAGE + BWD_CODE_BYTES + C::SCB;
        tma_load_2d(ds, &map_d, &ctl->full[s], n0, tok0);
        tma_load_2d(ds + C::DBOX, &map_d, &ctl->full[s], n0 + 64, tok0);
      };
      const int pre = nit < C::ST ? nit : C::ST;
      for (int it = 0; it < pre; ++it) {
        mbar_arrive_expect_tx(&ctl->full[it], tx);
        load_weights(it);
      }
      griddep_wait();   // d_out may come from the previous kernel of the stream
      for (int it = 0; it < pre; ++it) load_d(it);
      int issued = pre;
      for (int it = pre; it < nit; ++it) {
        const int s = it % C::ST;
        if (!mbar_wait(&ctl->empty[s], ((it / C::ST) - 1) & 1, abort_flag, &g_device_error, 64u)) break;
        mbar_arrive_expect_tx(&ctl->full[s], tx);
        load_weights(it);
        load_d(it);
        issued = it + 1;
      }
      for (int it = (issued > C::ST ? issued - C::ST : 0); it < issued; ++it)
        mbar_wait_teardown(&ctl->full[it % C::ST], (it / C::ST) & 1);
    }
  } else {
    // ------------------------------------------------------------ consumers
    griddep_wait();   // outputs may still be read by the previous kernel
    const int c = warp - 1;
    const int rowA = 8 * c + t, rowB = rowA + 4;   // pair rows of the stage
    const int J = g >> 2;                          // 64-column block of this lane
    const uint32_t offA = rowA * 128 + 16 * ((4 * J + (g & 3)) ^ (rowA & 7));
    const uint32_t offB = rowB * 128 + 16 * ((4 * J + (g & 3)) ^ (rowB & 7));
    // d_out words (n = 2 rowA, 2 rowA + 1) and (2 rowB, 2 rowB + 1) of token 8 j + g
    uint32_t dA[NT], dB[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int row = 8 * j + g;
      const int nA = 2 * rowA, nB = 2 * rowB;      // 0..127 within the stage
      dA[j] = BWD_CODE_BYTES + C::SCB + (nA >> 6) * C::DBOX + row * 128 +
              16 * ((((nA & 63) * 2) >> 4) ^ (row & 7)) + (((nA & 63) * 2) & 15);
      dB[j] = BWD_CODE_BYTES + C::SCB + (nB >> 6) * C::DBOX + row * 128 +
              16 * ((((nB & 63) * 2) >> 4) ^ (row & 7)) + (((nB & 63) * 2) & 15);
    }
    // scale half2 of pairs rowA / rowB in the row of each column group
    uint32_t scA[SPB], scB[SPB];
#pragma unroll
    for (int q = 0; q < SPB; ++q) {
      const int col = 64 * J + 16 * (q * (4 / SPB)) + 4 * (g & 3);
      const int r = ((kbase + col) >> gsl) - (kbase >> gsl);
      scA[q] = BWD_CODE_BYTES + r * 128 * C::SB + 2 * C::SB * rowA;
      scB[q] = BWD_CODE_BYTES + r * 128 * C::SB + 2 * C::SB * rowB;
    }
    for (int it = 0; it < nit; ++it) {
      const int s = it % C::ST;
      if (!mbar_wait(&ctl->full[s], (it / C::ST) & 1, abort_flag, &g_device_error, 128u)) break;
      const uint32_t st = sbase + s * C::STAGE;
      const uint4 va = lds128(st + offA), vb = lds128(st + offB);
      uint32_t bfr[NT][2];
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        bfr[j][0] = lds32(st + dA[j]);
        bfr[j][1] = lds32(st + dB[j]);
      }
      uint2 sa[SPB], sb[SPB];
#pragma unroll
      for (int q = 0; q < SPB; ++q) {
        sa[q] = F32S ? lds64(st + scA[q]) : make_uint2(lds32(st + scA[q]), 0u);
        sb[q] = F32S ? lds64(st + scB[q]) : make_uint2(lds32(st + scB[q]), 0u);
      }
      {
        uint32_t dep = va.x ^ va.y ^ va.z ^ va.w ^ vb.x ^ vb.y ^ vb.z ^ vb.w;
#pragma unroll
        for (int j = 0; j < NT; ++j) dep ^= bfr[j][0] ^ bfr[j][1];
#pragma unroll
        for (int q = 0; q < SPB; ++q) dep ^= sa[q].x ^ sa[q].y ^ sb[q].x ^ sb[q].y;
        stage_reads_done(dep);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->empty[s]);   // the stage is in registers
      const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
      const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = i / (4 / SPB);
        auto op = [&](__half2 c, uint2 sw) -> uint32_t {   // one byte's (even n, odd n) weights, scaled
          if (F32S) return weight_pair_f32s(c, __uint_as_float(sw.x), __uint_as_float(sw.y));
          return h2_as_u32(__hmul2(c, u32_as_h2(sw.x)));
        };
        const ColPairs ca = codes_minus8_cols(wa[i]);
        const ColPairs cb = codes_minus8_cols(wb[i]);
        const __half2 la[4] = {ca.c0, ca.c1, ca.c2, ca.c3};
        const __half2 lb[4] = {cb.c0, cb.c1, cb.c2, cb.c3};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t af[4] = {op(la[2 * h], sa[q]), op(la[2 * h + 1], sa[q]), op(lb[2 * h], sb[q]),
                                  op(lb[2 * h + 1], sb[q])};
#pragma unroll
          for (int j = 0; j < NT; ++j) mma_16816(acc[j][2 * i + h], af, bfr[j]);
        }
      }
    }
  }

  // Warp partials (into the idle ring), summed over the warps in order, then
  // over the cluster in rank order.
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);                 // [consumer][MB tokens][128 columns]
  float* cta_part = red + C::RED_FLOATS;                       // [MB tokens][128 columns]
  if (warp > 0) {
    float* mine = red + (warp - 1) * (C::MB * 128);
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
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < Mz * 128; idx += kBwdThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kBwdConsumers; ++w) v += red[w * (C::MB * 128) + idx];
    cta_part[idx] = v;
  }
  cg::cluster_group cluster = cg::this_cluster();
  if (S > 1) cluster.sync();
  else __syncthreads();
  if (!(S > 1 ? cluster_any_abort(cluster, &ctl->abort, S) : *abort_flag)) {
    const int rk = S > 1 ? (int)cluster.block_rank() : 0;
    const int tb = rk * Mz / S, te = (rk + 1) * Mz / S;
    const int kw = min(128, K - kbase);
    for (int e = tb * 128 + threadIdx.x; e < te * 128; e += kBwdThreads) {
      const int tok = e >> 7, kl = e & 127;
      if (kl >= kw) continue;
      float v = 0.f;
      for (int q = 0; q < S; ++q) v += (q == rk ? cta_part : cluster.map_shared_rank(cta_part, q))[e];
      dx[(size_t)(tok0 + tok) * K + kbase + kl] = v;
    }
  }
  if (S > 1) cluster.sync();
}

}  // namespace gv

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int NT, int SPG, bool F32S, bool XS>
static cudaError_t launch_gemv_tma_variant(const CUtensorMap& map_pk, const CUtensorMap& map_sc,
                                           const CUtensorMap& map_x, const __half* x, OutSplit out, int M, int N,
                                           int K, int gs, int stages_total, dim3 grid, cudaStream_t stream) {
  using C = gv::FwdCfg<NT, SPG, F32S, XS>;
  auto kern = gv::q4gsw_gemv_fwd_tma_kernel<NT, SPG, F32S, XS>;
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
  return cudaLaunchKernelEx(&cfg, kern, map_pk, map_sc, map_x, x, out, M, N, K, gs, stages_total);
}

cudaError_t launch_gemv_tma_fwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* x, int M,
                                OutSplit out, cudaStream_t stream, char* route, int route_len) {
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  const int sb = f32s ? 4 : 2;
  const Layout L = layout_of(N, K, gs, sb);
  const int G = K / gs;
  const int NT = (M <= 8) ? 1 : 2;
  const int zs = (M + 15) / 16;
  const int tiles = (N + 63) / 64;
  const int stages_total = (K + gv::SK - 1) / gv::SK;
  const int spg = gs == 16 ? 1 : gs == 32 ? 2 : gs < gv::SK ? 4 : 8;
  // Contraction splits: as many CTAs as the SMs hold at once (each CTA's
  // stages are consumed at a bounded rate, so the stream needs many of them),
  // at least two stages per split, clusters of at most 8.
  const int per_sm = NT == 1 ? 4 : 2;
  int S = sm_count(current_device()) * per_sm / (tiles * zs);
  S = S < 1 ? 1 : (S > 8 ? 8 : S);
  while (S > 1 && stages_total / S < 2) --S;
  const int sc_rows = gs < gv::SK ? gv::SK / gs : 1;
  // Activations staged in the ring (see FwdCfg) for 9..16 tokens or at least
  // six stages per split; from global memory otherwise, where the smaller ring
  // of the staged form has little to prefetch.  Measured on B200 (us per
  // launch, from global -> staged): 16 x 14336 x 4096 17.1 -> 15.3,
  // 16 x 4096 x 14336 18.0 -> 15.0, 1 x 4096 x 14336 12.2 -> 11.3,
  // 1 x 8192 x 2048 5.8 -> 6.0.  Pins: 2 from global memory, 3 staged.
  const int pin = route_pins().gemv;
  const bool xs = pin == kGemvTmaXs || (pin != kGemvTma && (NT == 2 || stages_total / S >= 6));
  CUtensorMap map_pk, map_sc, map_x;
  const bool ok =
      make_map_2d(&map_pk, CU_TENSOR_MAP_DATA_TYPE_UINT8, pk, K, N / 2, K, 128, gv::RP, CU_TENSOR_MAP_SWIZZLE_128B) &&
      make_map_2d(&map_sc, f32s ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                  pk + L.scales_offset, N, G, (uint64_t)N * sb, 64, sc_rows, CU_TENSOR_MAP_SWIZZLE_NONE) &&
      (!xs || make_map_2d(&map_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, K, M, (uint64_t)K * 2, 64, 8 * NT,
                          CU_TENSOR_MAP_SWIZZLE_128B));
  if (!ok) return cudaErrorInvalidValue;
  if (!xs) map_x = map_pk;   // not read
  const dim3 grid(tiles, S, zs);
  cudaError_t e;
  const __half* xh = reinterpret_cast<const __half*>(x);
#define Q4_TMA_FWD_X(NT_, SPG_, XS_)                                                                           \
  (f32s ? launch_gemv_tma_variant<NT_, SPG_, true, XS_>(map_pk, map_sc, map_x, xh, out, M, N, K, gs, stages_total, \
                                                        grid, stream)                                          \
        : launch_gemv_tma_variant<NT_, SPG_, false, XS_>(map_pk, map_sc, map_x, xh, out, M, N, K, gs,          \
                                                         stages_total, grid, stream))
#define Q4_TMA_FWD(NT_, SPG_) (xs ? Q4_TMA_FWD_X(NT_, SPG_, true) : Q4_TMA_FWD_X(NT_, SPG_, false))
  if (NT == 1)
    e = spg == 1 ? Q4_TMA_FWD(1, 1) : spg == 2 ? Q4_TMA_FWD(1, 2) : spg == 4 ? Q4_TMA_FWD(1, 4) : Q4_TMA_FWD(1, 8);
  else
    e = spg == 1 ? Q4_TMA_FWD(2, 1) : spg == 2 ? Q4_TMA_FWD(2, 2) : spg == 4 ? Q4_TMA_FWD(2, 4) : Q4_TMA_FWD(2, 8);
#undef Q4_TMA_FWD
#undef Q4_TMA_FWD_X
  if (route)
    snprintf(route, route_len, "gemv_tma_fwd launches=1 nt=%d tiles=%d splits=%d zslices=%d stages=%d%s", NT, tiles,
             S, zs, stages_total, xs ? " x=staged" : "");
  return e;
}

cudaError_t launch_gemv_tma_bwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* d_out, int M,
                                float* d_x, cudaStream_t stream, char* route, int route_len) {
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  const int sb = f32s ? 4 : 2;
  const Layout L = layout_of(N, K, gs, sb);
  const int G = K / gs;
  const int NT = (M <= 8) ? 1 : 2;
  const int zs = (M + 15) / 16;
  const int tiles = (K + 127) / 128;
  const int stages_total = (N + 127) / 128;
  const int sms = sm_count(current_device());
  // fill the two resident CTA slots per SM, at least two stages per split
  int S = 2 * sms / (tiles * zs);
  S = S < 1 ? 1 : (S > 8 ? 8 : S);
  while (S > 1 && stages_total / S < 2) --S;
  const int sc_rows = gs < 128 ? 128 / gs : 1;
  CUtensorMap map_pk, map_sc, map_d;
  const bool ok =
      make_map_2d(&map_pk, CU_TENSOR_MAP_DATA_TYPE_UINT8, pk, K, N / 2, K, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
      make_map_2d(&map_sc, f32s ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                  pk + L.scales_offset, N, G, (uint64_t)N * sb, 128,
                  sc_rows, CU_TENSOR_MAP_SWIZZLE_NONE) &&
      make_map_2d(&map_d, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, d_out, N, M, (uint64_t)N * 2, 64, 8 * NT,
                  CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  const int spb = gs >= 64 ? 1 : gs == 32 ? 2 : 4;
  const dim3 grid(tiles, S, zs);
  auto launch = [&](auto kern, int smem) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(gv::kBwdThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = S;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, map_pk, map_sc, map_d, d_x, M, N, K, gs, stages_total);
  };
  cudaError_t e;
#define Q4_TMA_BWD(NT_, SPB_)                                                                        \
  (f32s ? launch(gv::q4gsw_gemv_bwd_tma_kernel<NT_, SPB_, true>, gv::BwdCfg<NT_, true>::BYTES)       \
        : launch(gv::q4gsw_gemv_bwd_tma_kernel<NT_, SPB_, false>, gv::BwdCfg<NT_, false>::BYTES))
  if (NT == 1)
    e = spb == 1 ? Q4_TMA_BWD(1, 1) : spb == 2 ? Q4_TMA_BWD(1, 2) : Q4_TMA_BWD(1, 4);
  else
    e = spb == 1 ? Q4_TMA_BWD(2, 1) : spb == 2 ? Q4_TMA_BWD(2, 2) : Q4_TMA_BWD(2, 4);
#undef Q4_TMA_BWD
  if (route)
    snprintf(route, route_len, "gemv_tma_bwd launches=1 nt=%d tiles=%d splits=%d zslices=%d stages=%d", NT, tiles, S,
             zs, stages_total);
  return e;
}

}  // namespace q4gsw
