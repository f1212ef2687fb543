// q4gsw_gemm_sm100.cu - tcgen05 / tensor-memory GEMM route of the q4gsw linear
// layer for larger token counts (sm_100a).
//
//   forward   y[m,n]   = sum_k x[m,k]     * w[n,k]     (w[n,k] = (code - 8) * s[k/gs, n])
//   backward  d_x[m,k] = sum_n d_out[m,n] * w[n,k]
// ("[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward kernel (4-bit
// input-grad)", PR description; the fused Q/K/V forward of "[ExecuTorch][WebGPU]
// Replace broad QKV fusion with BK64 kernel" is the forward with its output
// columns scattered over three buffers.)
//
// One CTA computes a (128 or 256)-token x 256-feature tile of the output,
// optionally for one slice of the contraction (split-K, reduced in a cluster
// through distributed shared memory).  Warp roles:
//   warp 0       TMA producer: activation tile (fp16, 128-byte swizzle) and the
//                packed-code tile of each 64-deep contraction stage;
//   warp 1       allocates tensor memory and issues tcgen05.mma from one thread
//                (one 128-token accumulator per 128 tokens of the tile);
//   warps 2..17  dequantise every stage's codes into fp16 (code - 8) * scale,
//                written straight into the 128-byte-swizzled layout the MMA
//                descriptors read, then run the epilogue (tcgen05.ld -> global).
// Every consumer waits on every phase of the barriers it uses: a waiter that
// skipped a phase could mistake an older completion of the same parity for
// the one it wants.
// The forward reads the weight tile [256 n][64 k] as a K-major B operand; the
// backward writes the same kind of tile ([64 n][256 k], k contiguous) and reads
// it as an MN-major B operand, so both directions use one packed blob and one
// dequantisation routine.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>

#include "q4gsw_common.cuh"
#include "q4gsw_internal.h"
#include "q4gsw_sm100.cuh"

namespace cg = cooperative_groups;

namespace q4gsw {

// OR of the codes of waits that timed out and of out-of-range embedding
// indices: one word per device, shared by every stream and host thread (read
// and cleared by q4gsw_device_error_check).
__device__ unsigned int g_device_error = 0;
// Values swapped out of g_device_error, one slot per concurrent check.
constexpr int kErrorSlots = 64;
__device__ unsigned int g_error_snapshot[kErrorSlots];

namespace gemm {

constexpr int BM = 128;                 // tokens per MMA (M) and per accumulator
constexpr int BN = 256;                 // output features per tile (MMA N)
constexpr int TK = 64;                  // contraction depth per stage
constexpr int WST = 3;                  // dequantised-weight ring
constexpr int kDequantWarps = 16;       // all of them dequantise every stage
constexpr int kThreads = 32 * (2 + kDequantWarps);
constexpr int A_BYTES = BM * TK * 2;    // activation tile, 16 KB
constexpr int P_BYTES = BN / 2 * TK;    // packed codes, 8 KB
constexpr int W_BYTES = BN * TK * 2;    // dequantised fp16 weights, 32 KB
constexpr int CTL_BYTES = 256;

// Shared-memory map for a TMA ring of ST stages (MSUB 128-row activation
// tiles, packed codes, a scale slot of SCB bytes: 1 KB for gs >= 32, 2 KB for
// gs 16) and a ring of WST dequantised-weight tiles.  One CTA computes MSUB
// 128-token sub-tiles against each dequantised weight tile, so the
// dequantisation work per multiply-add falls by MSUB.
template <int ST, int SCB, int MSUB>
struct Smem {
  static constexpr int A_STAGE = MSUB * A_BYTES;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_P = OFF_A + ST * A_STAGE;
  static constexpr int OFF_W = OFF_P + ST * P_BYTES;
  static constexpr int OFF_SC = OFF_W + WST * W_BYTES;
  static constexpr int OFF_CTL = OFF_SC + ST * SCB;
  static constexpr int BYTES = OFF_CTL + CTL_BYTES + 1024;
  static constexpr int TMEM_COLS = 256 * MSUB;
  static_assert(OFF_P % 1024 == 0 && OFF_W % 1024 == 0 && OFF_SC % 1024 == 0, "1024-byte aligned regions");
  static_assert(BM * BN * 4 <= OFF_SC, "split-K staging of one sub-tile must fit below the scale buffers");
  static_assert(BYTES <= 232448, "shared memory per CTA");
};

struct Args {
  OutSplit out;
  int M, N, K, gs;
  int out_cols;       // forward: N, backward: K
  int stages_total;   // contraction / TK
  int sc_bytes;       // bytes of the scale box loaded per stage
};

constexpr int kMaxST = 5;
struct SmemCtl {
  uint64_t full[kMaxST];       // stage s loaded (TMA transaction bytes)
  uint64_t consumed[kMaxST];   // the MMAs of the stage in slot s completed (one commit per stage)
  uint64_t wready[WST];        // dequantised tile w written (all dequantisation warps)
  uint64_t accfull;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(SmemCtl) <= CTL_BYTES, "control block");

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
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

template <bool BWD, int ST, int SCB, int MSUB, bool F32S>
__global__ void __launch_bounds__(kThreads, 1)
q4gsw_gemm_kernel(const __grid_constant__ CUtensorMap map_act, const __grid_constant__ CUtensorMap map_pk,
                  const __grid_constant__ CUtensorMap map_sc, const Args args) {
  using namespace sm100;
  using SM = Smem<ST, SCB, MSUB>;
  constexpr int SB = F32S ? 4 : 2;   // bytes per scale
  constexpr int OFF_A = SM::OFF_A, OFF_P = SM::OFF_P, OFF_W = SM::OFF_W, OFF_SC = SM::OFF_SC,
                OFF_CTL = SM::OFF_CTL, SC_BYTES = SCB, A_STAGE = SM::A_STAGE,
                TMEM_COLS = SM::TMEM_COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + OFF_CTL);
  volatile int* abort_flag = &ctl->abort;
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;    // first output feature of the tile
  const int m0 = blockIdx.y * BM * MSUB;    // first token of the tile
  const int S = gridDim.z, split = blockIdx.z;
  const int st_begin = (int)((long long)split * args.stages_total / S);
  const int st_end = (int)((long long)(split + 1) * args.stages_total / S);
  const int nit = st_end - st_begin;

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->consumed[i], 1);
    }
    for (int i = 0; i < WST; ++i) {
      mbar_init(&ctl->wready[i], kDequantWarps);
    }
    mbar_init(&ctl->accfull, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
    prefetch_tmap(&map_act);
    prefetch_tmap(&map_pk);
    prefetch_tmap(&map_sc);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      auto load_weights = [&](int it) {
        const int s = it % ST;
        const int kc = (st_begin + it) * TK;
        uint8_t* pk = smem + OFF_P + s * P_BYTES;
        uint8_t* sc = smem + OFF_SC + s * SC_BYTES;
        if (!BWD) {
          tma_load_2d(pk, &map_pk, &ctl->full[s], kc, n0 / 2);
          tma_load_2d(sc, &map_sc, &ctl->full[s], n0, kc >> (__ffs(args.gs) - 1));
        } else {
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) tma_load_2d(pk + jb * (P_BYTES / 4), &map_pk, &ctl->full[s], n0 + 64 * jb, kc / 2);
          tma_load_2d(sc, &map_sc, &ctl->full[s], kc, n0 >> (__ffs(args.gs) - 1));
        }
      };
      auto load_act = [&](int it) {
        const int s = it % ST;
        tma_load_2d(smem + OFF_A + s * A_STAGE, &map_act, &ctl->full[s], (st_begin + it) * TK, m0);
      };
      // The packed weight is constant: the first stages' codes and scales are
      // requested before waiting for the previous kernel of the stream, which
      // may still be producing the activations.
      const int pre = nit < ST ? nit : ST;
      for (int it = 0; it < pre; ++it) {
        mbar_arrive_expect_tx(&ctl->full[it], A_STAGE + P_BYTES + args.sc_bytes);
        load_weights(it);
      }
      griddep_wait();
      for (int it = 0; it < pre; ++it) load_act(it);
      int issued = pre;
      for (int it = pre; it < nit; ++it) {
        const int s = it % ST;
        if (!mbar_wait(&ctl->consumed[s], ((it / ST) - 1) & 1, abort_flag, &g_device_error, 1u)) break;
        mbar_arrive_expect_tx(&ctl->full[s], A_STAGE + P_BYTES + args.sc_bytes);
        load_weights(it);
        load_act(it);
        issued = it + 1;
      }
      // never leave with copies in flight: wait for the last fill of each stage
      for (int it = (issued > ST ? issued - ST : 0); it < issued; ++it)
        mbar_wait_teardown(&ctl->full[it % ST], (it / ST) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Between stages this thread only waits on wready (each dequantisation
    // warp saw the stage's full barrier before arriving), tests the next
    // stage's wready while the last MMAs of this stage are queued, and
    // commits once: the tensor core holds little more than the MMA it runs.
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(BM, BN, BWD);
      bool next_ready = false;
      for (int it = 0; it < nit; ++it) {
        const int s = it % ST, w = it % WST;
        if (!next_ready && !mbar_wait(&ctl->wready[w], (it / WST) & 1, abort_flag, &g_device_error, 4u)) break;
        tc_fence_after();
        const uint32_t a0 = sbase + OFF_A + s * A_STAGE, w0 = sbase + OFF_W + w * W_BYTES;
#pragma unroll
        for (int ks = 0; ks < TK / 16; ++ks) {
          const uint64_t bd = BWD ? smem_desc_sw128(w0 + ks * 2048, 8192, 1024)
                                  : smem_desc_sw128(w0 + 32 * ks, 16, 1024);
          if (ks == TK / 16 - 1)
            next_ready = it + 1 < nit && mbar_test_wait(&ctl->wready[(it + 1) % WST], ((it + 1) / WST) & 1);
#pragma unroll
          for (int ms = 0; ms < MSUB; ++ms) {
            const uint64_t ad = smem_desc_sw128(a0 + ms * A_BYTES + 32 * ks, 16, 1024);
            mma_f16_ss(tmem + ms * 256, ad, bd, idesc, (it > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit(&ctl->consumed[s]);
      }
      mma_commit(&ctl->accfull);
      mma_commit(&ctl->drain);
      mbar_wait_teardown(&ctl->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ dequantisation
    // Thread td owns pair row p (rows 2p, 2p+1 of the tile), half u of each
    // 16-column step and the steps i = 2h, 2h+1 of each 64-column block; in the
    // backward also the 64-column block j of the 256-column tile.  Lanes vary
    // (u, h) fastest so that the 8-byte code loads of a half-warp and the
    // 16-byte stores of a quarter-warp hit distinct banks.
    const int td = threadIdx.x - 64;
    const int u = td & 1, h = (td >> 1) & 1;
    const int p = BWD ? ((td >> 2) & 31) : (td >> 2);
    const int j = BWD ? (td >> 7) : 0;
    // Per-thread offsets, fixed for the whole contraction: packed-code words
    // (64-byte swizzle), scale words (the scale row of each 8-column chunk is
    // the same in every stage because stages start on 64-column boundaries),
    // dequantised-tile chunks (128-byte swizzle).
    const int gsl = __ffs(args.gs) - 1;
    const int sz = (p >> 1) & 3;
    const uint32_t pk_base = (BWD ? j * (P_BYTES / 4) : 0) + p * 64 + 8 * h;
    const uint32_t pk_off0 = pk_base + 16 * ((2 * u) ^ sz);       // columns +0..3 of each step
    const uint32_t pk_off1 = pk_base + 16 * ((2 * u + 1) ^ sz);   // columns +4..7
    uint32_t sc_off[2], st_off_e[2], st_off_o[2];
    const int re = 2 * p, ro = 2 * p + 1;
#pragma unroll
    for (int ii = 0; ii < 2; ++ii) {
      const int i = 2 * h + ii;
      if (!BWD) {
        // stage base column kc: with gs >= 64 the 64 columns sit in one group,
        // with gs < 64 the stage starts a group; either way the row is
        // ((kc mod gs) + 16 i + 8 u) >> gsl = (16 i + 8 u) >> gsl for gs < 64, else 0
        sc_off[ii] = (args.gs < 64 ? ((16 * i + 8 * u) >> gsl) : 0) * 256 * SB + 2 * SB * p;
      } else {
        sc_off[ii] = (((n0 & (args.gs - 1)) + 64 * j + 16 * i + 8 * u) >> gsl) * 64 * SB + 2 * SB * p;
      }
      const int chunk = 2 * i + u;
      st_off_e[ii] = (BWD ? j * 8192 : 0) + re * 128 + 16 * (chunk ^ (re & 7));
      st_off_o[ii] = (BWD ? j * 8192 : 0) + ro * 128 + 16 * (chunk ^ (ro & 7));
    }
    for (int it = 0; it < nit; ++it) {
      const int s = it % ST, w = it % WST;
      if (!mbar_wait(&ctl->full[s], (it / ST) & 1, abort_flag, &g_device_error, 8u)) break;
      // tile w is free once the MMAs of stage it - WST completed
      if (it >= WST &&
          !mbar_wait(&ctl->consumed[(it - WST) % ST], ((it - WST) / ST) & 1, abort_flag, &g_device_error, 32u))
        break;
      const uint32_t pk = sbase + OFF_P + s * P_BYTES;
      const uint32_t sc = sbase + OFF_SC + s * SC_BYTES;
      const uint2 c0 = lds64(pk + pk_off0);
      const uint2 c1 = lds64(pk + pk_off1);
      const uint2 sw[2] = {F32S ? lds64(sc + sc_off[0]) : make_uint2(lds32(sc + sc_off[0]), 0u),
                           F32S ? lds64(sc + sc_off[1]) : make_uint2(lds32(sc + sc_off[1]), 0u)};
      const uint32_t wlo[2] = {c0.x, c0.y};
      const uint32_t whi[2] = {c1.x, c1.y};
      const uint32_t wt = sbase + OFF_W + w * W_BYTES;
#pragma unroll
      for (int ii = 0; ii < 2; ++ii) {
        const RowPairs a = codes_minus8_rows(wlo[ii]);   // columns +0..3 of this 8-column chunk
        const RowPairs b = codes_minus8_rows(whi[ii]);   // columns +4..7
        uint4 ve, vo;
        if (F32S) {
          const float se = __uint_as_float(sw[ii].x), so = __uint_as_float(sw[ii].y);
          ve = make_uint4(weight_pair_f32s(a.ev01, se, se), weight_pair_f32s(a.ev23, se, se),
                          weight_pair_f32s(b.ev01, se, se), weight_pair_f32s(b.ev23, se, se));
          vo = make_uint4(weight_pair_f32s(a.od01, so, so), weight_pair_f32s(a.od23, so, so),
                          weight_pair_f32s(b.od01, so, so), weight_pair_f32s(b.od23, so, so));
        } else {
          const __half2 s2 = u32_as_h2(sw[ii].x);
          const __half2 se = __low2half2(s2), so = __high2half2(s2);
          ve = make_uint4(h2_as_u32(__hmul2(a.ev01, se)), h2_as_u32(__hmul2(a.ev23, se)),
                          h2_as_u32(__hmul2(b.ev01, se)), h2_as_u32(__hmul2(b.ev23, se)));
          vo = make_uint4(h2_as_u32(__hmul2(a.od01, so)), h2_as_u32(__hmul2(a.od23, so)),
                          h2_as_u32(__hmul2(b.od01, so)), h2_as_u32(__hmul2(b.od23, so)));
        }
        sts128(wt + st_off_e[ii], ve);
        sts128(wt + st_off_o[ii], vo);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->wready[w]);
    }
  }

  // ---------------------------------------------------------------- epilogue
  // Warps 2..17: warp w reads TMEM lanes 32 (w % 4) .. +31 (tokens) and the 64
  // accumulator columns [64 h, 64 h + 64) with h = (w - 2) / 4, for each of
  // the MSUB accumulators (sub-tile ms holds tokens m0 + 128 ms ..), and parks
  // them in shared memory (the operand rings are idle by now).  All threads
  // then copy whole rows out, so each warp store covers 512 contiguous bytes
  // of one output row; with split-K the copy-out also sums the S partial
  // tiles of the cluster.
  const bool epi = warp >= 2;
  float* stage_f32 = reinterpret_cast<float*>(smem);   // staging [128][256] fp32, 16-byte chunks swizzled
  griddep_wait();   // outputs may still be read by the previous kernel of the stream
  bool have_acc = false;
  if (epi) have_acc = mbar_wait(&ctl->accfull, 0, abort_flag, &g_device_error, 16u);
  if (epi && have_acc) tc_fence_after();
  auto store4 = [&](int m, int n, float4 val) {
    const OutSplit& o = args.out;
    float* dst;
    if (n < o.n1) dst = o.y0 + (size_t)m * o.n1 + n;
    else if (n < o.n2) dst = o.y1 + (size_t)m * (o.n2 - o.n1) + (n - o.n1);
    else dst = o.y2 + (size_t)m * (o.N - o.n2) + (n - o.n2);
    *reinterpret_cast<float4*>(dst) = val;
  };
#pragma unroll 1
  for (int ms = 0; ms < MSUB; ++ms) {
    const int mb = m0 + ms * BM;
    if (epi && have_acc) {
      const int q = warp & 3, h = (warp - 2) >> 2;
      const int row = 32 * q + lane;
#pragma unroll 1
      for (int c32 = 0; c32 < 2; ++c32) {
        const int col = 64 * h + 32 * c32;
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(ms * 256 + col), r);
        tmem_wait_ld();
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const int chunk = (col >> 2) + v;   // 16-byte chunk of the 1 KB row
          const float4 val = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                         __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
          *reinterpret_cast<float4*>(stage_f32 + row * 256 + 4 * (chunk ^ (row & 7))) = val;
        }
      }
    }
    if (S == 1) {
      __syncthreads();
      const int rows = args.M - mb < BM ? args.M - mb : BM;
      if (!*abort_flag) {
        for (int idx = threadIdx.x; idx < rows * 64; idx += kThreads) {
          const int row = idx >> 6, chunk = idx & 63;
          const int n = n0 + 4 * chunk;
          if (n >= args.out_cols) continue;
          store4(mb + row, n, *reinterpret_cast<const float4*>(stage_f32 + row * 256 + 4 * (chunk ^ (row & 7))));
        }
      }
      __syncthreads();
    } else {
      // every thread of every CTA of the cluster passes both barriers, aborted or not
      cg::cluster_group cluster = cg::this_cluster();
      cluster.sync();
      const int r = (int)cluster.block_rank();
      const int row_b = r * BM / S, row_e = (r + 1) * BM / S;
      if (!cluster_any_abort(cluster, &ctl->abort, S)) {
        for (int idx = threadIdx.x; idx < (row_e - row_b) * 64; idx += kThreads) {
          const int row = row_b + (idx >> 6), chunk = idx & 63;
          const int m = mb + row, n = n0 + 4 * chunk;
          if (m >= args.M || n >= args.out_cols) continue;
          const int off = row * 256 + 4 * (chunk ^ (row & 7));
          // all S loads in flight at once, then the sum in rank order
          float4 part[8];
#pragma unroll
          for (int qq = 0; qq < 8; ++qq)
            if (qq < S) part[qq] = *reinterpret_cast<const float4*>(cluster.map_shared_rank(stage_f32, qq) + off);
          float4 acc = part[0];
#pragma unroll
          for (int qq = 1; qq < 8; ++qq)
            if (qq < S) {
              acc.x += part[qq].x;
              acc.y += part[qq].y;
              acc.z += part[qq].z;
              acc.w += part[qq].w;
            }
          store4(m, n, acc);
        }
      }
      cluster.sync();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace gemm

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 lookup_encode_fn() {
  cudaDriverEntryPointQueryResult q;
  void* p = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  return nullptr;
}

// The driver's tensor-map encoder, looked up once (thread-safe static init).
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = lookup_encode_fn();
  return fn;
}

static bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t dim0, uint64_t dim1,
                        uint64_t stride1_bytes, uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {dim0, dim1};
  cuuint64_t strides[1] = {stride1_bytes};
  cuuint32_t box[2] = {box0, box1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Relative main-loop time of one 64-column stage: one 128-token accumulator
// (1.0), or two sharing the dequantised tile (less than twice: the weight
// tile's dequantisation, its shared-memory stores and the packed-code copy are
// paid once).
static double stage_time(int msub) { return msub == 2 ? 1.6 : 1.0; }

// Chooses the split-K factor S of one kernel variant (and its cost), and
// launches it when `launch` is set.  Each candidate S costs waves(S) *
// (stages / S * stage time + fixed overhead: 2 stage times per accumulator, or
// 8 with the cluster reduction), where waves(S) uses how many S-CTA clusters
// the device can hold at once (a GPC must host a whole cluster).
template <bool BWD, int ST, int SCB, int MSUB, bool F32S>
static cudaError_t gemm_variant(const CUtensorMap& map_act, const CUtensorMap& map_pk, const CUtensorMap& map_sc,
                                const gemm::Args& a, int tiles_n, cudaStream_t stream, bool launch, int* S_out,
                                double* cost_out) {
  using namespace gemm;
  auto kern = q4gsw_gemm_kernel<BWD, ST, SCB, MSUB, F32S>;
  constexpr int smem = Smem<ST, SCB, MSUB>::BYTES;
  static PerDeviceOnce attr_once;
  static std::atomic<int> max_clusters[kMaxDevices][9];
  const int dev = current_device();
  const int d = (dev >= 0 && dev < kMaxDevices) ? dev : 0;
  {
    cudaError_t e = once_per_device(attr_once, dev, [&] {
      return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (e != cudaSuccess) return e;
  }
  const int tiles_m = (a.M + BM * MSUB - 1) / (BM * MSUB);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;

  const int tiles = tiles_n * tiles_m;
  const double t = stage_time(MSUB);
  int best_S = 1;
  double best_cost = 1e30;
  for (int S = 1; S <= 8; ++S) {
    if (S > 1 && a.stages_total / S < 4) break;
    int n = max_clusters[d][S].load(std::memory_order_relaxed);
    if (n == 0) {   // not measured yet on this device (concurrent callers store the same value)
      attr[0].val.clusterDim.z = S;
      cfg.gridDim = dim3(tiles_n, tiles_m, S);
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) n = -1;
      max_clusters[d][S].store(n, std::memory_order_relaxed);
    }
    if (n < 1) continue;
    const double waves = ceil((double)tiles / n);
    const double cost = waves * ((double)a.stages_total / S * t + (S > 1 ? 8.0 : 2.0) * MSUB);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best_S = S;
    }
  }
  *S_out = best_S;
  *cost_out = best_cost;
  if (!launch) return cudaSuccess;
  attr[0].val.clusterDim.z = best_S;
  cfg.gridDim = dim3(tiles_n, tiles_m, best_S);
  return cudaLaunchKernelEx(&cfg, kern, map_act, map_pk, map_sc, a);
}

// Number of 128-token accumulators per CTA pinned by q4gsw_debug_pin_routes
// (1 or 2), or 0: the cost model chooses.
static int forced_msub() {
  const int g = route_pins().gemm;
  return g == kGemmSs1 ? 1 : g == kGemmSs2 ? 2 : 0;
}

template <bool BWD, bool F32S>
static cudaError_t launch_gemm_impl(const void* packed, int N, int K, int gs, const uint16_t* act, int M,
                                    OutSplit out, cudaStream_t stream, char* route, int route_len) {
  using namespace gemm;
  constexpr int SB = F32S ? 4 : 2;
  const CUtensorMapDataType sdt = F32S ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  CUtensorMap map_pk, map_sc;
  const Layout L = layout_of(N, K, gs, SB);
  const void* scales = pk + L.scales_offset;
  const int G = K / gs;
  bool ok;
  int sc_bytes;
  if (!BWD) {
    const int rows = TK / gs > 1 ? TK / gs : 1;   // scale groups of one 64-column stage
    sc_bytes = rows * BN * SB;
    ok = make_map_2d(&map_pk, CU_TENSOR_MAP_DATA_TYPE_UINT8, pk, K, N / 2, K, TK, BN / 2, CU_TENSOR_MAP_SWIZZLE_64B) &&
         make_map_2d(&map_sc, sdt, scales, N, G, (uint64_t)N * SB, BN, rows, CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    const int rows = BN / gs > 1 ? BN / gs : 1;   // scale groups of one 256-column tile
    sc_bytes = rows * TK * SB;
    ok = make_map_2d(&map_pk, CU_TENSOR_MAP_DATA_TYPE_UINT8, pk, K, N / 2, K, TK, TK / 2,
                     CU_TENSOR_MAP_SWIZZLE_64B) &&
         make_map_2d(&map_sc, sdt, scales, N, G, (uint64_t)N * SB, TK, rows, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (!ok || sc_bytes > (F32S ? 4096 : 2048)) return cudaErrorInvalidValue;

  Args a;
  a.sc_bytes = sc_bytes;
  a.out = out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.gs = gs;
  a.out_cols = BWD ? K : N;
  const int contraction = BWD ? N : K;
  a.stages_total = (contraction + TK - 1) / TK;
  const int tiles_n = (a.out_cols + BN - 1) / BN;
  // Scale slots of 4 KB (fp32 scales with 16-column groups) leave room for one
  // 128-token accumulator per CTA only.
  const bool one_acc_only = sc_bytes > 2048;
  // The activation box is re-encoded per variant (128 or 256 tokens high).
  auto run = [&](int msub, bool launch, int* S, double* cost) -> cudaError_t {
    CUtensorMap map_a;
    const uint64_t act_cols = BWD ? (uint64_t)N : (uint64_t)K;
    if (!make_map_2d(&map_a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, act, act_cols, M, act_cols * 2, TK, BM * msub,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    if (sc_bytes <= 1024)
      return msub == 2 ? gemm_variant<BWD, 3, 1024, 2, F32S>(map_a, map_pk, map_sc, a, tiles_n, stream, launch, S, cost)
                       : gemm_variant<BWD, 5, 1024, 1, F32S>(map_a, map_pk, map_sc, a, tiles_n, stream, launch, S, cost);
    if (sc_bytes <= 2048)
      return msub == 2 ? gemm_variant<BWD, 3, 2048, 2, F32S>(map_a, map_pk, map_sc, a, tiles_n, stream, launch, S, cost)
                       : gemm_variant<BWD, 4, 2048, 1, F32S>(map_a, map_pk, map_sc, a, tiles_n, stream, launch, S, cost);
    return gemm_variant<BWD, 4, 4096, 1, F32S>(map_a, map_pk, map_sc, a, tiles_n, stream, launch, S, cost);
  };
  int msub = one_acc_only ? 1 : forced_msub();
  int S = 1;
  double cost = 0;
  cudaError_t e = cudaSuccess;
  if (msub == 0) {
    int S1 = 1, S2 = 1;
    double c1 = 0, c2 = 0;
    e = run(1, false, &S1, &c1);
    if (e == cudaSuccess) e = run(2, false, &S2, &c2);
    if (e != cudaSuccess) return e;
    msub = (M > BM && c2 < c1) ? 2 : 1;
  }
  e = run(msub, true, &S, &cost);
  const int st = msub == 2 ? 3 : (sc_bytes <= 1024 ? 5 : 4);
  if (route)
    snprintf(route, route_len, "tcgen05_gemm_%s launches=1 tile=%dx%dx%d stages=%d+%d grid=%dx%dx%d",
             BWD ? "bwd" : "fwd", BM * msub, BN, TK, st, WST, tiles_n, (M + BM * msub - 1) / (BM * msub), S);
  return e;
}

}  // namespace q4gsw

#include "q4gsw_embedding.cuh"
#include "q4gsw_gemm_ts.cuh"
#include "q4gsw_gemv_tma.cuh"
#include "q4gsw_dq8ca_tma.cuh"

namespace q4gsw {

// Route between the two GEMM kernels.  Up to 512 tokens the weight tile lives
// in tensor memory (its shared-memory traffic is lowest); above, the
// shared-memory route with two 128-token accumulators per CTA re-reads each
// activation tile half as often from L2 and wins (measured on B200 at 1024 and
// 4096 tokens).  q4gsw_debug_pin_routes can pin either route.
static bool use_ss_route(int M) {
  const int g = route_pins().gemm;
  if (g == kGemmTs) return false;
  if (g == kGemmSs || g == kGemmSs1 || g == kGemmSs2) return true;
  return M > 512;
}

cudaError_t launch_gemm_fwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* x, int M, OutSplit out,
                            cudaStream_t stream, char* route, int route_len) {
  if (use_ss_route(M))
    return f32s ? launch_gemm_impl<false, true>(packed, N, K, gs, x, M, out, stream, route, route_len)
                : launch_gemm_impl<false, false>(packed, N, K, gs, x, M, out, stream, route, route_len);
  return f32s ? launch_gemm_ts_impl<false, true>(packed, N, K, gs, x, M, out, stream, route, route_len)
              : launch_gemm_ts_impl<false, false>(packed, N, K, gs, x, M, out, stream, route, route_len);
}

cudaError_t launch_gemm_adapter(bool bwd, const void* packed, int N, int K, int gs, const uint16_t* act, int M,
                                float* out, const AdapterRef& ad, cudaStream_t stream, char* route, int route_len) {
  // the adapter stage exists in the tensor-memory route, which takes any M
  if (bwd)
    return launch_gemm_ts_impl<true, false>(packed, N, K, gs, act, M, single_output(out, K), stream, route, route_len,
                                            &ad);
  return launch_gemm_ts_impl<false, false>(packed, N, K, gs, act, M, single_output(out, N), stream, route, route_len,
                                           &ad);
}

cudaError_t launch_gemm_bwd(const void* packed, int N, int K, int gs, bool f32s, const uint16_t* d_out, int M,
                            float* d_x, cudaStream_t stream, char* route, int route_len) {
  const OutSplit o = single_output(d_x, K);
  if (use_ss_route(M))
    return f32s ? launch_gemm_impl<true, true>(packed, N, K, gs, d_out, M, o, stream, route, route_len)
                : launch_gemm_impl<true, false>(packed, N, K, gs, d_out, M, o, stream, route, route_len);
  return f32s ? launch_gemm_ts_impl<true, true>(packed, N, K, gs, d_out, M, o, stream, route, route_len)
              : launch_gemm_ts_impl<true, false>(packed, N, K, gs, d_out, M, o, stream, route, route_len);
}

__global__ void q4gsw_error_exchange_kernel(unsigned int slot) {
  g_error_snapshot[slot] = atomicExch(&g_device_error, 0u);
}

// A wait on a barrier that nothing completes, bounded by limit_ns: the
// failure path of every kernel's waits, run on purpose and without a fault.
__global__ void q4gsw_wait_probe_kernel(unsigned long long limit_ns) {
  using namespace sm100;
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, &g_device_error, 0x200u, limit_ns);
}

cudaError_t launch_wait_probe(unsigned int limit_us, cudaStream_t stream) {
  q4gsw_wait_probe_kernel<<<1, 32, 0, stream>>>(1000ull * limit_us);
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(cudaStream_t stream, unsigned int* host_value) {
  // The swap is one atomic on the device, so a bit that a kernel on another
  // stream sets after it stays in the word for the next check.
  static std::atomic<unsigned int> next_slot{0};
  const unsigned int slot = next_slot.fetch_add(1, std::memory_order_relaxed) % kErrorSlots;
  q4gsw_error_exchange_kernel<<<1, 1, 0, stream>>>(slot);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbolAsync(host_value, g_error_snapshot, sizeof(unsigned int), slot * sizeof(unsigned int),
                                cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(stream);
}

}  // namespace q4gsw
