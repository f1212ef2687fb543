// q4gsw_gemm_ts.cuh - tcgen05 GEMM route with the dequantised weight tile in
// tensor memory (sm_100a).  Included once, by q4gsw_gemm_sm100.cu, which owns
// the device error word and the tensor-map helpers.
//
// The same two products as the shared-memory route, transposed so that the
// weight is the MMA's M side:
//   forward   y^T[n, m]   = sum_k w[n, k]   x[m, k]        (A = w tile,   B = x tile)
//   backward  d_x^T[k, m] = sum_n w^T[k, n] d_out[m, n]    (A = w^T tile, B = d_out tile)
// with w[n, k] = (code[n, k] - 8) * s[k / gs, n] ("[ExecuTorch][Vulkan] Add
// et_vk.linear_q4gsw_backward kernel (4-bit input-grad)", PR description).
//
// Why transposed: the dequantisation warps write the fp16 weight tile straight
// into tensor memory (tcgen05.st), where tcgen05.mma reads it as the A operand.
// Only the activation tile and the 4-bit codes pass through shared memory, so
// per 128 x 256 x 64 step the shared-memory traffic is the 32 KB activation
// copy in, the MMA's 32 KB read of it and 4 KB of codes, against 112 KB when
// the dequantised tile is stored to and re-read from shared memory.
//
// One CTA computes 128 weight rows (output features) x bt tokens (bt <= 256,
// a multiple of 16, chosen per launch to balance the token tiles), optionally
// for one slice of the contraction (split-K, reduced in a cluster through
// distributed shared memory).  Warp roles:
//   warp 0       TMA producer: activation tile [bt][64] fp16 (128-byte
//                swizzle), packed codes and scale rows of each 64-deep stage;
//   warp 1       allocates tensor memory (fp32 accumulator in columns 0..255,
//                after it one 32-column slot of dequantised weights per
//                shared-memory stage) and issues tcgen05.mma from one thread;
//   warps 2..17  warp w writes TMEM lanes 32 (w % 4) .. +31 (weight rows) of
//                every fourth stage (stages (w - 2) / 4 + 4 i, each into the
//                slot of its shared-memory stage), then runs the epilogue for
//                the same lanes.
// A parity wait is only sound while its barrier is at most one phase behind
// the phase waited for; each wait below states why that holds.
#pragma once

namespace q4gsw {
namespace ts {

constexpr int BW = 128;                    // weight rows per tile (MMA M)
constexpr int BT_MAX = 256;                // tokens per tile (MMA N)
constexpr int TK = 64;                     // contraction depth per stage
constexpr int kMaxST = 8;                  // shared-memory stages (and TMEM slots) at most
constexpr int kDequantWarps = 16;
constexpr int kThreads = 32 * (2 + kDequantWarps);
constexpr int X_BYTES = BT_MAX * TK * 2;   // activation tile, 32 KB
constexpr int P_BYTES = BW / 2 * TK;       // packed codes of one stage, 4 KB
constexpr int CTL_BYTES = 256;
constexpr int ACC_COLS = 256;              // fp32 accumulator columns (tokens)
constexpr int A_COLS = TK / 2;             // one dequantised stage: 64 fp16 per lane = 32 columns
constexpr int TMEM_COLS = 512;
static_assert(ACC_COLS + kMaxST * A_COLS <= TMEM_COLS, "tensor memory budget");

// ST stages; SCB bytes of scale rows per stage (1 KB for fp16 scales, 2 KB for
// fp32 scales, packed layout version 2).
template <int ST, int SCB>
struct Smem {
  static constexpr int SC_BYTES = SCB;
  static constexpr int OFF_X = 0;
  static constexpr int OFF_P = OFF_X + ST * X_BYTES;
  static constexpr int OFF_SC = OFF_P + ST * P_BYTES;
  static constexpr int OFF_CTL = OFF_SC + ST * SCB;
  static constexpr int BYTES = OFF_CTL + CTL_BYTES + 1024;
  static_assert(OFF_P % 1024 == 0 && OFF_SC % 1024 == 0, "1024-byte aligned regions");
  static_assert((BT_MAX + 7) * BW * 4 <= OFF_SC, "split-K receive slots must fit below the scale slots");
  static_assert(BYTES <= 232448, "shared memory per CTA");
};

struct Args {
  OutSplit out;
  int M, N, K, gs;
  int rows_out;       // weight-side extent of the output: N (forward) or K (backward)
  int stages_total;
  int sc_bytes;       // bytes of the scale box of one stage
  int bt;             // tokens per tile
  int tma_out;        // outputs written by one tensor store (map_y*; no split-K), else by threads
  // Low-rank adapter stage (ad_r > 0): one more 64-deep stage of the last
  // split whose weight operand is the adapter matrix (forward: rows of B
  // [N, r]; backward: columns of A [r, K]; leading dimension ad_ld) and whose
  // activation operand is the fp16 intermediate [M][64] (map_ad).
  const __half* ad_mat;
  int ad_r;
  int ad_ld;
};

struct Ctl {
  uint64_t full[kMaxST];       // stage s loaded (TMA transaction bytes)
  uint64_t consumed[kMaxST];   // the MMAs of the stage in slot s completed (one commit per stage)
  uint64_t wready[kMaxST];     // dequantised stage in TMEM slot s written (one warp per lane quadrant)
  uint64_t accfull;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Ctl) <= CTL_BYTES, "control block");

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// (1024 + lo nibble, 1024 + nibble at bits 16..19) -> exact (c - 8) half2
__device__ __forceinline__ uint32_t nibbles_minus8(uint32_t v) {
  const __half2 kSub = u32_as_h2(0x64086408u);   // 1032, 1032
  return h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(v, 0x000F000Fu, 0x64006400u)), kSub));
}

// Rows [row_b, row_e) of the tile, summed over the S partial tiles in rank
// order and written as float4 to the output.  pushed: the partials sit in
// this CTA's shared memory, rank qq's at stage_f32 + qq * slot_floats with
// rows relative to row_b; otherwise each rank's whole [token][128] tile is
// parked in its own shared memory and read through the cluster window.  Each
// thread first issues the loads of up to kPer items (S each), then adds and
// stores: remote loads are latency-bound, and one item at a time left ~4 of
// those latencies in a row per thread.
template <int S>
__device__ __forceinline__ void copy_out(const float* stage_f32, bool pushed, int slot_floats, int row_b, int row_e,
                                         int t0, int f0, const Args& args) {
  using namespace sm100;
  constexpr int kPer = S == 1 ? 8 : (12 / S > 0 ? 12 / S : 1);   // at most 12 float4 in flight
  const OutSplit& o = args.out;
  uint32_t src[S];   // rank qq's partial rows, in the cluster's shared window
#pragma unroll
  for (int qq = 0; qq < S; ++qq)
    src[qq] = pushed ? smem_u32(stage_f32 + qq * slot_floats)
                     : (S == 1 ? smem_u32(stage_f32) : mapa_u32(smem_u32(stage_f32), (uint32_t)qq));
  const int r0 = pushed ? 0 : row_b;   // row of row_b in the source layout
  const int total = (row_e - row_b) * (BW / 4);
  for (int base = threadIdx.x; base < total; base += kThreads * kPer) {
    float4 part[kPer][S];
    bool ok[kPer];
    int offs[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = base + u * kThreads;
      const int row = idx / (BW / 4), c4 = idx % (BW / 4);   // row relative to row_b
      offs[u] = row * BW + 4 * c4;
      ok[u] = idx < total && t0 + row_b + row < args.M && f0 + 4 * c4 < args.rows_out;
      if (ok[u]) {
        const uint32_t o4 = 4u * (uint32_t)((r0 + row) * BW + 4 * c4);
#pragma unroll
        for (int qq = 0; qq < S; ++qq)
          part[u][qq] = S == 1 ? *reinterpret_cast<const float4*>(stage_f32 + (r0 + row) * BW + 4 * c4)
                               : ld_dsmem_v4(src[qq] + o4);
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (!ok[u]) continue;
      float4 acc = part[u][0];
#pragma unroll
      for (int qq = 1; qq < S; ++qq) {
        acc.x += part[u][qq].x;
        acc.y += part[u][qq].y;
        acc.z += part[u][qq].z;
        acc.w += part[u][qq].w;
      }
      const int m = t0 + row_b + offs[u] / BW, f = f0 + offs[u] % BW;
      float* dst;
      if (f < o.n1) dst = o.y0 + (size_t)m * o.n1 + f;
      else if (f < o.n2) dst = o.y1 + (size_t)m * (o.n2 - o.n1) + (f - o.n1);
      else dst = o.y2 + (size_t)m * (o.N - o.n2) + (f - o.n2);
      *reinterpret_cast<float4*>(dst) = acc;
    }
  }
}

template <bool BWD, int ST, bool F32S>
__global__ void __launch_bounds__(kThreads, 1)
q4gsw_gemm_ts_kernel(const __grid_constant__ CUtensorMap map_act, const __grid_constant__ CUtensorMap map_pk,
                     const __grid_constant__ CUtensorMap map_sc, const __grid_constant__ CUtensorMap map_y0,
                     const __grid_constant__ CUtensorMap map_y1, const __grid_constant__ CUtensorMap map_y2,
                     const __grid_constant__ CUtensorMap map_ad, const Args args) {
  using namespace sm100;
  static_assert(ST <= kMaxST, "barrier arrays and TMEM slots");
  using SM = Smem<ST, F32S ? 2048 : 1024>;
  constexpr int SC_BYTES = SM::SC_BYTES;
  constexpr int SB = F32S ? 4 : 2;   // bytes per scale
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + SM::OFF_CTL);
  volatile int* abort_flag = &ctl->abort;
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f0 = blockIdx.x * BW;          // first weight row (output feature) of the tile
  const int t0 = blockIdx.y * args.bt;     // first token of the tile
  const int S = gridDim.z, split = blockIdx.z;
  const int st_begin = (int)((long long)split * args.stages_total / S);
  const int st_end = (int)((long long)(split + 1) * args.stages_total / S);
  const int nit = st_end - st_begin;          // stages of the packed weight
  const int nitx = nit + ((args.ad_r > 0 && split == S - 1) ? 1 : 0);   // plus the adapter stage
  const int gsl = __ffs(args.gs) - 1;

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->consumed[i], 1);
      mbar_init(&ctl->wready[i], 4);   // one warp per lane quadrant
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
      const uint32_t tx = (uint32_t)args.bt * TK * 2 + P_BYTES + args.sc_bytes;
      auto load_weights = [&](int it) {
        const int s = it % ST;
        const int kc = (st_begin + it) * TK;
        uint8_t* pk = smem + SM::OFF_P + s * P_BYTES;
        uint8_t* sc = smem + SM::OFF_SC + s * SC_BYTES;
        if (!BWD) {
          tma_load_2d(pk, &map_pk, &ctl->full[s], kc, f0 / 2);       // [64 pairs][64 B]
          tma_load_2d(sc, &map_sc, &ctl->full[s], f0, kc >> gsl);    // [rows][128 n]
        } else {
          tma_load_2d(pk, &map_pk, &ctl->full[s], f0, kc / 2);       // [32 pairs][128 B]
          tma_load_2d(sc, &map_sc, &ctl->full[s], kc, f0 >> gsl);    // [rows][64 n]
        }
      };
      auto load_act = [&](int it) {
        const int s = it % ST;
        if (it < nit)
          tma_load_2d(smem + SM::OFF_X + s * X_BYTES, &map_act, &ctl->full[s], (st_begin + it) * TK, t0);
        else   // the adapter stage: the low-rank intermediate of the tile's tokens
          tma_load_2d(smem + SM::OFF_X + s * X_BYTES, &map_ad, &ctl->full[s], 0, t0);
      };
      const uint32_t tx_ad = (uint32_t)args.bt * TK * 2;
      // The packed weight is constant: the first stages' codes and scales are
      // requested before waiting for the previous kernel of the stream, which
      // may still be producing the activations.
      const int pre = nitx < ST ? nitx : ST;
      for (int it = 0; it < pre; ++it) {
        mbar_arrive_expect_tx(&ctl->full[it], it < nit ? tx : tx_ad);
        if (it < nit) load_weights(it);
      }
      griddep_wait();
      for (int it = 0; it < pre; ++it) load_act(it);
      int issued = pre;
      for (int it = pre; it < nitx; ++it) {
        const int s = it % ST;
        if (!mbar_wait(&ctl->consumed[s], ((it / ST) - 1) & 1, abort_flag, &g_device_error, 1u)) break;
        mbar_arrive_expect_tx(&ctl->full[s], it < nit ? tx : tx_ad);
        if (it < nit) load_weights(it);
        load_act(it);
        issued = it + 1;
      }
      // never leave with copies in flight: wait for the last fill of each stage
      for (int it = (issued > ST ? issued - ST : 0); it < issued; ++it)
        mbar_wait_teardown(&ctl->full[it % ST], (it / ST) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Every cycle this thread spends between stages is a bubble of the tensor
    // pipe, and the MMAs issue at the pipe's rate only from straight-line code
    // whose operand addresses are fixed offsets: measured on B200 with the
    // stage and slot indices taken modulo at run time, four MMAs and their
    // commit took ~570 cycles at every token width, against ~330 (64 tokens)
    // and 512 (256 tokens, the MMA's own time) from the unrolled form below.
    // So the loop runs in blocks of ST stages, in which stage j of the block
    // uses shared-memory stage and TMEM slot j as constants; the last nitx mod
    // ST stages take the generic loop.  Each stage waits on wready alone (each
    // dequantisation warp saw the stage's full barrier before arriving, so
    // wready covers the activation tile too) and commits once.
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(BW, args.bt, false);
      // The descriptor's start address field is address / 16 in its low 14
      // bits (shared addresses stay below 256 KB), so the descriptor of the
      // activation tile of stage s at depth 16 ks is the stage-0 descriptor
      // plus (s X_BYTES + 32 ks) / 16: an immediate add, no register per stage.
      const uint64_t d0 = smem_desc_sw128(sbase + SM::OFF_X, 16, 1024);
      const uint32_t ab = tmem + ACC_COLS;
      auto issue = [&](uint32_t s, bool first) {
#pragma unroll
        for (int ks = 0; ks < TK / 16; ++ks)
          mma_f16_ts(tmem, ab + s * A_COLS + 8 * ks, d0 + ((s * X_BYTES + 32 * ks) >> 4), idesc,
                     (first && ks == 0) ? 0u : 1u);
      };
      bool ok = true;
      const int nblk = nitx / ST;
      for (int b = 0; b < nblk && ok; ++b) {
        const uint32_t ph = (uint32_t)b & 1u;
#pragma unroll
        for (int j = 0; j < ST; ++j) {
          if (!mbar_try_wait(&ctl->wready[j], ph) &&
              !mbar_wait(&ctl->wready[j], ph, abort_flag, &g_device_error, 4u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue(j, b == 0 && j == 0);
          mma_commit(&ctl->consumed[j]);
        }
      }
      for (int it = nblk * ST; it < nitx && ok; ++it) {
        const int s = it % ST;
        if (!mbar_wait(&ctl->wready[s], (it / ST) & 1, abort_flag, &g_device_error, 4u)) break;
        tc_fence_after();
        issue(s, it == 0);
        mma_commit(&ctl->consumed[s]);
      }
      mma_commit(&ctl->accfull);
      mma_commit(&ctl->drain);
      mbar_wait_teardown(&ctl->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ dequantisation
    // Thread = weight row r of the tile (its TMEM lane 32 q + lane).  The
    // four warps of lane quadrant q take whole stages in turn: warp kq
    // dequantises stages kq, kq + 4, kq + 8, ... (all 64 contraction columns,
    // i.e. the 32 TMEM columns of the slot of the stage's shared-memory ring
    // index; two fp16 per column, lower index in the low half).  A warp thus
    // pays the latency of its barrier wait (~140 cycles, measured, even on a
    // completed phase) once per four stages; with every warp on every stage
    // that chain bounded the stage rate at ~650 cycles.
    //
    // A warp sees only every fourth phase of a stage's barriers, so before
    // waiting for stage it's full phase it first waits for the commit of
    // stage it - ST's MMAs (consumed): those MMAs followed the wready of all
    // four quadrant warps of stage it - ST, each of which had seen that
    // stage's full phase, so full[s] is then at most one phase behind.
    // (Without it, a load of stage it - ST landing after this warp's stage
    // it - 4 left full[s] two phases behind: the parity test passed on the
    // older phase, and the wready counts shifted until a warp waited on its
    // own arrival.)  consumed[s] itself is at most one phase behind: this
    // warp's stage it - 4 needed full(it - 4), which the producer issued
    // after the commit of stage it - 4 - ST >= the one before it - ST.  The
    // same commit frees the stage's TMEM slot, last read by those MMAs.
    static_assert(kDequantWarps == 16, "four warps per lane quadrant");
    const int q = warp & 3, kq = (warp - 2) >> 2;
    const int r = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    uint32_t off[4] = {0u, 0u, 0u, 0u};
    uint32_t sc_off[4] = {0u, 0u, 0u, 0u};
    uint32_t shift = 0, boff = 0, sc_base = 0;
    if (!BWD) {
      // Row r = 2 p + odd of pair p.  Word c of the 16-byte chunk t of the
      // pair row holds columns 16 c + 4 t + (0, 2, 1, 3) in its byte slots;
      // the chunk sits at 16 (t ^ ((p >> 1) & 3)) under the 64-byte swizzle.
      const int p = r >> 1;
      shift = 4 * (r & 1);
#pragma unroll
      for (int t = 0; t < 4; ++t) off[t] = p * 64 + 16 * (t ^ ((p >> 1) & 3));
      // columns 16 c .. 16 c + 15 share one scale: row (16 c) >> gsl of the
      // stage's box (stages start on 64-column boundaries)
#pragma unroll
      for (int c = 0; c < 4; ++c) sc_off[c] = (args.gs < 64 ? ((16 * c) >> gsl) : 0) * BW * SB + SB * r;
    } else {
      // Row r = output feature k = f0 + r.  Pair row p (contraction rows 2p,
      // 2p+1) holds it in byte column_offset(r) of its 128-byte box row; the
      // scales of pair p sit at 2 SB p of scale row ((f0 mod gs) + r) >> gsl.
      boff = (uint32_t)column_offset(r);
      sc_base = (uint32_t)((((f0 & (args.gs - 1)) + r) >> gsl) * TK * SB);
    }
    for (int it = kq; it < nitx; it += 4) {
      const int s = it % ST;
      if (it >= ST && !mbar_wait(&ctl->consumed[s], ((it / ST) - 1) & 1, abort_flag, &g_device_error, 32u)) break;
      if (!mbar_wait(&ctl->full[s], (it / ST) & 1, abort_flag, &g_device_error, 8u)) break;
      tc_fence_after();
      const uint32_t slot = tmem + lane_base + (uint32_t)(ACC_COLS + s * A_COLS);
      const uint32_t pk = sbase + SM::OFF_P + s * P_BYTES;
      const uint32_t sc = sbase + SM::OFF_SC + s * SC_BYTES;
      uint32_t v[8];
      if (it >= nit) {
        // The adapter stage: rank columns j = 0 .. 63 of this thread's output
        // feature, straight from the fp16 adapter matrix (forward B[f][j],
        // backward A[j][f]; zero past the rank or the extent).
        const int f = f0 + r;
        const bool fin = f < args.rows_out;
        const unsigned short* am = reinterpret_cast<const unsigned short*>(args.ad_mat);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int j = 16 * c + 2 * m;
            uint32_t lo = 0u, hi = 0u;
            if (fin && j < args.ad_r)
              lo = BWD ? __ldg(am + (size_t)j * args.ad_ld + f) : __ldg(am + (size_t)f * args.ad_ld + j);
            if (fin && j + 1 < args.ad_r)
              hi = BWD ? __ldg(am + (size_t)(j + 1) * args.ad_ld + f) : __ldg(am + (size_t)f * args.ad_ld + j + 1);
            v[m] = lo | (hi << 16);
          }
          tmem_st_32x32b_x8(slot + 8 * c, v);
        }
      } else if (!BWD) {
        uint4 wv[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) wv[t] = lds128_u32addr(pk + off[t]);
        uint32_t sraw[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) sraw[c] = F32S ? lds32(sc + sc_off[c]) : lds_u16(sc + sc_off[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const uint32_t word = c == 0 ? wv[t].x : c == 1 ? wv[t].y : c == 2 ? wv[t].z : wv[t].w;
            const uint32_t W = word >> shift;   // this row's nibbles
            if (F32S) {
              const float sf = __uint_as_float(sraw[c]);
              v[2 * t] = weight_pair_f32s(u32_as_h2(nibbles_minus8(W)), sf, sf);          // columns 4t, 4t+1
              v[2 * t + 1] = weight_pair_f32s(u32_as_h2(nibbles_minus8(W >> 8)), sf, sf); // 4t+2, 4t+3
            } else {
              const __half2 s2 = u32_as_h2(sraw[c] | (sraw[c] << 16));
              v[2 * t] = h2_as_u32(__hmul2(u32_as_h2(nibbles_minus8(W)), s2));            // columns 4t, 4t+1
              v[2 * t + 1] = h2_as_u32(__hmul2(u32_as_h2(nibbles_minus8(W >> 8)), s2));   // 4t+2, 4t+3
            }
          }
          tmem_st_32x32b_x8(slot + 8 * c, v);
        }
      } else {
        // four slices of 8 pairs (16 contraction rows), each slice's 8 code
        // bytes and their scales loaded before any is used (fp32 scales: one
        // slice at a time, within the register budget)
#pragma unroll (F32S ? 1 : 4)
        for (int c = 0; c < 4; ++c) {
          uint32_t b[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) b[j] = lds_u8(pk + (8 * c + j) * 128 + boff);   // pair p = 8 c + j: code[2p, k] | code[2p+1, k] << 4
          constexpr int NV = F32S ? 4 : 2;   // 16-byte scale vectors of 8 pairs
          uint4 sv[NV];
#pragma unroll
          for (int u = 0; u < NV; ++u) sv[u] = lds128_u32addr(sc + sc_base + 2 * SB * 8 * c + 16 * u);
          const uint32_t* sw = reinterpret_cast<const uint32_t*>(sv);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const __half2 c2 = u32_as_h2(nibbles_minus8(b[j] * 0x1001u));
            if (F32S)   // s32[g, 2p], s32[g, 2p+1]
              v[j] = weight_pair_f32s(c2, __uint_as_float(sw[2 * j]), __uint_as_float(sw[2 * j + 1]));
            else        // s[g, 2p], s[g, 2p+1]
              v[j] = h2_as_u32(__hmul2(c2, u32_as_h2(sw[j])));
          }
          tmem_st_32x32b_x8(slot + 8 * c, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->wready[s]);
    }
  }

  // ---------------------------------------------------------------- epilogue
  // Warp w (2..17) reads TMEM lanes 32 (w % 4) .. +31 (weight rows) and the
  // token columns [64 c, 64 c + 64) with c = (w - 2) / 4, and parks them in
  // shared memory (the operand ring is idle by now) as [token][128 features].
  const bool epi = warp >= 2;
  griddep_wait();   // outputs may still be read by the previous kernel of the stream
  bool have_acc = false;
  if (epi) {
    have_acc = mbar_wait(&ctl->accfull, 0, abort_flag, &g_device_error, 16u);
    have_acc = __all_sync(0xffffffffu, have_acc);
    if (have_acc) tc_fence_after();
  }
  const OutSplit& o = args.out;
  float* stage_f32 = reinterpret_cast<float*>(smem);   // the operand ring, idle by now
  // Park the tile in this CTA's shared memory as [token][128 features].
  auto park = [&] {
    if (!(epi && have_acc)) return;
    const int q = warp & 3, cb = (warp - 2) >> 2;
    const int r = 32 * q + lane;
#pragma unroll 1
    for (int c32 = 0; c32 < 2; ++c32) {
      const int col = 64 * cb + 32 * c32;
      if (col >= args.bt) break;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)col, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) stage_f32[(col + j) * BW + r] = __uint_as_float(v[j]);
    }
  };
  if (S == 1) {
    // One tensor store of the [bt][128] fp32 tile (rows past M and features
    // past the output clipped by the map), or the threads' copy-out.
    park();
    if (args.tma_out) {
      const CUtensorMap* my = f0 < o.n1 ? &map_y0 : (f0 < o.n2 ? &map_y1 : &map_y2);
      const int c0 = f0 < o.n1 ? f0 : (f0 < o.n2 ? f0 - o.n1 : f0 - o.n2);
      fence_proxy_async_smem();
      __syncthreads();
      if (threadIdx.x == 0 && !*abort_flag) {
        tma_store_2d(my, stage_f32, c0, t0);
        bulk_commit();
        bulk_wait_read_all();
      }
    } else {
      __syncthreads();
      if (!*abort_flag) copy_out<1>(stage_f32, false, 0, 0, args.bt, t0, f0, args);
    }
  } else {
    // Split-K: rank rk owns token rows [rk bt / S, (rk + 1) bt / S) and adds
    // the S partial tiles' rows in rank order.  Two ways to bring them over,
    // chosen by the tile's width (measured on B200, M=512 MLP projections and
    // Q/K/V):
    //  - wide tiles (bt >= 192): once every CTA of the cluster is past its main
    //    loop (first barrier: all operand rings idle), each CTA stores its
    //    partial rows straight from tensor memory into the owner's receive
    //    slot for its rank (remote stores are posted, no round trip); after the
    //    second barrier each owner adds its slots from its own shared memory.
    //    This spares parking the 128 KB tile and reading 3/4 of it remotely
    //    (4-way split, 256 tokens: 21.0 -> 19.9 us);
    //  - narrower tiles: each CTA parks its tile before the first barrier,
    //    overlapping the cluster's slowest main loop, and the owners read the
    //    other ranks' rows through the cluster window; after the second barrier
    //    no CTA reads another's shared memory, so any may leave.
    // Every thread of every CTA of the cluster passes both barriers, aborted or not.
    cg::cluster_group cluster = cg::this_cluster();
    const int me = (int)cluster.block_rank();
    const int row_b = me * args.bt / S, row_e = (me + 1) * args.bt / S;
    const bool push = args.bt >= 192;
    const int rmax = (args.bt + S - 1) / S;   // rows of the largest owner's range: one receive slot
    if (!push) park();
    cluster_barrier();
    const bool aborted = cluster_any_abort(cluster, &ctl->abort, S);
    if (push) {
      if (epi && have_acc && !aborted) {
        const int q = warp & 3, cb = (warp - 2) >> 2;
        const int r = 32 * q + lane;
        const uint32_t mine = smem_u32(stage_f32) + 4u * (uint32_t)(me * rmax * BW + r);   // my slot, my feature
#pragma unroll 1
        for (int c32 = 0; c32 < 2; ++c32) {
          const int col = 64 * cb + 32 * c32;
          if (col >= args.bt) break;
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)col, v);
          tmem_wait_ld();
          int owner = ((col + 1) * S - 1) / args.bt;          // largest rank with rank bt / S <= col
          int ob = owner * args.bt / S, oe = (owner + 1) * args.bt / S;
          uint32_t dst = mapa_u32(mine, (uint32_t)owner);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = col + j;
            if (t >= args.bt) break;
            if (t >= oe) {   // the next owner's rows (uniform over the warp)
              ++owner;
              ob = oe;
              oe = (owner + 1) * args.bt / S;
              dst = mapa_u32(mine, (uint32_t)owner);
            }
            st_dsmem_f32(dst + 4u * (uint32_t)((t - ob) * BW), __uint_as_float(v[j]));
          }
        }
      }
      cluster_barrier();   // every partial row delivered
    }
    if (!aborted) {
      switch (S) {
        case 2: copy_out<2>(stage_f32, push, rmax * BW, row_b, row_e, t0, f0, args); break;
        case 3: copy_out<3>(stage_f32, push, rmax * BW, row_b, row_e, t0, f0, args); break;
        case 4: copy_out<4>(stage_f32, push, rmax * BW, row_b, row_e, t0, f0, args); break;
        case 5: copy_out<5>(stage_f32, push, rmax * BW, row_b, row_e, t0, f0, args); break;
        case 6: copy_out<6>(stage_f32, push, rmax * BW, row_b, row_e, t0, f0, args); break;
        case 7: copy_out<7>(stage_f32, push, rmax * BW, row_b, row_e, t0, f0, args); break;
        default: copy_out<8>(stage_f32, push, rmax * BW, row_b, row_e, t0, f0, args); break;
      }
    }
    if (!push) cluster_barrier();   // no CTA leaves while another reads its tile
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace ts

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <bool BWD, bool F32S>
static cudaError_t launch_gemm_ts_impl(const void* packed, int N, int K, int gs, const uint16_t* act, int M,
                                       OutSplit out, cudaStream_t stream, char* route, int route_len,
                                       const AdapterRef* ad = nullptr) {
  using namespace ts;
  constexpr int ST = F32S ? 5 : 6;
  constexpr int SB = F32S ? 4 : 2;
  constexpr int SC_BYTES = Smem<ST, F32S ? 2048 : 1024>::SC_BYTES;
  const CUtensorMapDataType sdt = F32S ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  const Layout L = layout_of(N, K, gs, SB);
  const void* scales = pk + L.scales_offset;
  const int G = K / gs;
  Args a;
  a.out = out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.gs = gs;
  a.rows_out = BWD ? K : N;
  const int contraction = BWD ? N : K;
  a.stages_total = (contraction + TK - 1) / TK;
  // token tiles: as few as fit 256 tokens, balanced, rounded up to 16 (one
  // more may be taken below, once the split is known)
  int tiles_t = (M + BT_MAX - 1) / BT_MAX;
  a.bt = (((M + tiles_t - 1) / tiles_t) + 15) / 16 * 16;
  const int tiles_f = (a.rows_out + BW - 1) / BW;

  CUtensorMap map_act, map_pk, map_sc;
  bool ok = make_map_2d(&map_act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, act, (uint64_t)contraction, M,
                        (uint64_t)contraction * 2, TK, a.bt, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!BWD) {
    const int rows = TK / gs > 1 ? TK / gs : 1;   // scale groups of one 64-column stage
    a.sc_bytes = rows * BW * SB;
    ok = ok && make_map_2d(&map_pk, CU_TENSOR_MAP_DATA_TYPE_UINT8, pk, K, N / 2, K, TK, BW / 2,
                           CU_TENSOR_MAP_SWIZZLE_64B) &&
         make_map_2d(&map_sc, sdt, scales, N, G, (uint64_t)N * SB, BW, rows, CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    const int rows = BW / gs > 1 ? BW / gs : 1;   // scale groups of one 128-feature tile
    a.sc_bytes = rows * TK * SB;
    ok = ok && make_map_2d(&map_pk, CU_TENSOR_MAP_DATA_TYPE_UINT8, pk, K, N / 2, K, BW, TK / 2,
                           CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_map_2d(&map_sc, sdt, scales, N, G, (uint64_t)N * SB, TK, rows, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (!ok || a.sc_bytes > SC_BYTES) return cudaErrorInvalidValue;

  // Output tensor maps [M][width] fp32, box [bt][128]: usable when every
  // buffer starts 16-byte aligned and no 128-feature tile straddles two of
  // them; otherwise the threads write the outputs.
  CUtensorMap map_y[3];
  auto make_out_maps = [&](int bt) -> bool {
    const int nb[3] = {0, out.n1, out.n2};
    const int ne[3] = {out.n1, out.n2, out.N};
    float* const yb[3] = {out.y0, out.y1, out.y2};
    bool tma_out = (out.n1 % BW == 0 || out.n1 == out.N) && (out.n2 % BW == 0 || out.n2 == out.N);
    for (int i = 0; i < 3 && tma_out; ++i) {
      const int width = ne[i] - nb[i];
      if (width <= 0) {
        map_y[i] = map_y[0];
        continue;
      }
      tma_out = (reinterpret_cast<uintptr_t>(yb[i]) % 16 == 0) &&
                make_map_2d(&map_y[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, yb[i], (uint64_t)width, M,
                            (uint64_t)width * 4, BW, bt, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (!tma_out) map_y[0] = map_y[1] = map_y[2] = map_act;   // never read
    return tma_out;
  };
  a.tma_out = make_out_maps(a.bt) ? 1 : 0;

  // adapter stage: the intermediate [M][64] fp16 as the activation operand
  CUtensorMap map_ad = map_act;   // never read without an adapter
  a.ad_mat = nullptr;
  a.ad_r = 0;
  a.ad_ld = 0;
  if (ad) {
    if (!make_map_2d(&map_ad, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ad->inter, 64, M, 128, TK, a.bt,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    a.ad_mat = reinterpret_cast<const __half*>(ad->mat);
    a.ad_r = ad->r;
    a.ad_ld = BWD ? K : ad->r;
  }
  auto kern = q4gsw_gemm_ts_kernel<BWD, ST, F32S>;
  constexpr int smem = Smem<ST, SC_BYTES>::BYTES;
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

  // Split-K S: each candidate costs waves(S) * (stages / S + fixed overhead:
  // 2 stages, or 8 with the cluster reduction), where waves(S) uses how many
  // S-CTA clusters the device can hold at once.
  const int tiles = tiles_f * tiles_t;
  int best_S = 1;
  double best_cost = 1e30;
  for (int S = 1; S <= 8; ++S) {
    if (S > 1 && a.stages_total / S < 4) break;
    int n = max_clusters[d][S].load(std::memory_order_relaxed);
    if (n == 0) {   // not measured yet on this device (concurrent callers store the same value)
      attr[0].val.clusterDim.z = S;
      cfg.gridDim = dim3(tiles_f, tiles_t, S);
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) n = -1;
      max_clusters[d][S].store(n, std::memory_order_relaxed);
    }
    if (n < 1) continue;
    const double waves = ceil((double)tiles / n);
    const double cost = waves * ((double)a.stages_total / S + (S > 1 ? 8.0 : 2.0));
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best_S = S;
    }
  }
  // With split-K the threads sum the S partial tiles through distributed
  // shared memory and write the outputs (fixed order), instead of rank 0's
  // tensor store followed, once it has completed, by the other ranks'
  // reduce-adds.
  if (best_S > 1) a.tma_out = 0;
  // One more token tile at the same split when the tiles stay at least 128
  // tokens wide and the grid still fits in one wave of clusters: the CTAs keep
  // their stage count, and a stage costs nearly the same at 176 tokens as at
  // 256 (measured, M=512 Q/K/V 3072x2048: 14.7 -> 13.8 us with 3 x 176 tokens).
  {
    const int tt = tiles_t + 1;
    const int bt = (((M + tt - 1) / tt) + 15) / 16 * 16;
    const int n = max_clusters[d][best_S].load(std::memory_order_relaxed);
    if (bt >= 128 && n >= 1 && tiles_f * tt <= n) {
      // every map whose box follows the tile's token count
      const bool ok2 = make_map_2d(&map_act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, act, (uint64_t)contraction, M,
                                   (uint64_t)contraction * 2, TK, bt, CU_TENSOR_MAP_SWIZZLE_128B) &&
                       (!ad || make_map_2d(&map_ad, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ad->inter, 64, M, 128, TK, bt,
                                           CU_TENSOR_MAP_SWIZZLE_128B));
      if (!ok2) return cudaErrorInvalidValue;
      if (a.tma_out && !make_out_maps(bt)) a.tma_out = 0;
      if (!a.tma_out) map_y[0] = map_y[1] = map_y[2] = map_act;   // never read
      tiles_t = tt;
      a.bt = bt;
    }
  }
  attr[0].val.clusterDim.z = best_S;
  cfg.gridDim = dim3(tiles_f, tiles_t, best_S);
  if (route)
    snprintf(route, route_len, "tcgen05_ts_gemm_%s launches=1 tile=%dx%dx%d stages=%d+%d grid=%dx%dx%d out=%s%s",
             BWD ? "bwd" : "fwd", BW, a.bt, TK, ST, ST, tiles_f, tiles_t, best_S, a.tma_out ? "tma" : "st",
             ad ? " adapter_stage=1" : "");
  return cudaLaunchKernelEx(&cfg, kern, map_act, map_pk, map_sc, map_y[0], map_y[1], map_y[2], map_ad, a);
}

}  // namespace q4gsw
